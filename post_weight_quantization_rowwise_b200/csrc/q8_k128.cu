// q8_k128.cu -- Q8_K_128 activation quantization on sm_100a.
//
// Page "ik_llama.cpp 量化精度修复实录：用 Q8_K_128 替代 Q8_1 根治 IQ1_S_R4 /
// IQ1_M_R4 的 fp16 溢出" (www.hnwysp.cn/news/39281), 修复方案: blocks of 128
// values, a binary32 scale, int8 codes and one int16 sum of the codes per 32
// values, not multiplied by d, so that no fp16 quantity can overflow.
//
// Per block: amax = max|x|, d = amax/127, id = amax > 0 ? 127/amax : 0,
// q = clamp(rint(x*id), -127, 127) with a NaN product giving 0, and
// bsums[i] = sum of q over values 32i..32i+31.  Block layout (140 bytes, LE):
// float d | int8 qs[128] | int16 bsums[4].
//
// Mapping: one warp per 128-value block; lane t holds values 4t..4t+3 (one
// 16-byte load, so a warp reads 512 contiguous bytes), writes qs[4t..4t+3]
// as one 32-bit store (a warp writes 128 contiguous bytes), and lanes 0, 8,
// 16, 24 write the four sums.  The work is HBM bound (4 B read + 140/128 B
// written per value); each warp keeps four blocks in flight, and the two IEEE
// divisions of the four blocks (d and 1/d) run once, lane u taking block u.
#include "common.cuh"

namespace {

#ifndef IQQ_Q8_UNROLL
#define IQQ_Q8_UNROLL 4  // 128-value blocks in flight per warp
#endif
#ifndef IQQ_Q8_CTAS
#define IQQ_Q8_CTAS 16   // CTAs of 256 threads per SM in the grid (8 resident: two waves; measured best of 4-16)
#endif
constexpr int kThreads = 256;
constexpr int kUnroll = IQQ_Q8_UNROLL;

// rint with the cvt.rni saturating conversion: +-Inf -> INT_MAX / INT_MIN,
// NaN -> 0; then the symmetric int8 clamp.
__device__ __forceinline__ int code_of(float x, float id)
{
    const float p = __fmul_rn(x, id);
    int q = __float2int_rn(p);
    q = max(-127, min(127, q));
    return q;
}

__global__ void __launch_bounds__(kThreads)
q8_k128_kernel(const float4* __restrict__ x, uint8_t* __restrict__ out, int64_t nblocks,
               uint32_t* __restrict__ flags)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
    uint32_t bad = 0u;

    for (int64_t g0 = warp * kUnroll; g0 < nblocks; g0 += nwarps * kUnroll) {
        float4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t g = g0 + u;
            v[u] = g < nblocks ? iqq::ld_stream_f4(x + g * 32 + lane) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        // amax of every block in flight (all lanes hold all of them)
        float amax[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const float4 a = v[u];
            // NaN/Inf detection: x*0 is NaN exactly for non-finite x
            const float z = __fmul_rn(a.x, 0.f) + __fmul_rn(a.y, 0.f) + __fmul_rn(a.z, 0.f) +
                            __fmul_rn(a.w, 0.f);
            if (z != z) bad |= IQQ_FLAG_NONFINITE_INPUT;
            float m = fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(a.z), fabsf(a.w)));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            amax[u] = m;
        }
        // d = amax/127 and id = 127/amax of block u are computed by lane u (one pass of the
        // two IEEE divisions for all the blocks in flight), then broadcast
        float am = amax[0];
#pragma unroll
        for (int u = 1; u < kUnroll; ++u)
            if (lane == u) am = amax[u];
        const float dl = __fdiv_rn(am, 127.0f);
        const float idl = am > 0.f ? __fdiv_rn(127.0f, am) : 0.f;
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t g = g0 + u;
            const float d = __shfl_sync(0xffffffffu, dl, u);
            const float id = __shfl_sync(0xffffffffu, idl, u);
            if (g >= nblocks) break;  // warp-uniform
            const float4 a = v[u];
            const int q0 = code_of(a.x, id), q1 = code_of(a.y, id);
            const int q2 = code_of(a.z, id), q3 = code_of(a.w, id);
            const uint32_t packed = (static_cast<uint32_t>(q0) & 0xffu) |
                                    ((static_cast<uint32_t>(q1) & 0xffu) << 8) |
                                    ((static_cast<uint32_t>(q2) & 0xffu) << 16) |
                                    (static_cast<uint32_t>(q3) << 24);
            int s = q0 + q1 + q2 + q3;
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            s += __shfl_xor_sync(0xffffffffu, s, 2);
            s += __shfl_xor_sync(0xffffffffu, s, 4);
            uint8_t* blk = out + g * IQQ_Q8_K128_BLOCK_BYTES;
            reinterpret_cast<uint32_t*>(blk + 4)[lane] = packed;
            if ((lane & 7) == 0)
                reinterpret_cast<int16_t*>(blk + 132)[lane >> 3] = static_cast<int16_t>(s);
            if (lane == 0) *reinterpret_cast<float*>(blk) = d;
        }
    }
    iqq::raise_flags(flags, bad);
}

}  // namespace

extern "C" iqq_status iqq_quantize_q8_k128(const float* x, void* out, int64_t nrows,
                                           int64_t n_per_row, uint32_t* d_flags, void* stream)
{
    if (!iqq::size_ok(nrows, n_per_row, 4)) return IQQ_ERR_SHAPE;
    if (n_per_row % IQQ_Q8_K128_BLOCK_VALUES != 0) return IQQ_ERR_SHAPE;
    if (nrows == 0 || n_per_row == 0) return IQQ_OK;
    if (x == nullptr || out == nullptr) return IQQ_ERR_NULL;
    if (!iqq::aligned(x, 16) || !iqq::aligned(out, 4) || (d_flags && !iqq::aligned(d_flags, 4)))
        return IQQ_ERR_ALIGN;
    const int64_t nblocks = nrows * (n_per_row / IQQ_Q8_K128_BLOCK_VALUES);
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t warps_needed = (nblocks + kUnroll - 1) / kUnroll;
    const int64_t ctas_needed = (warps_needed + (kThreads / 32) - 1) / (kThreads / 32);
    const int64_t cap = static_cast<int64_t>(sms) * IQQ_Q8_CTAS;
    const int grid = static_cast<int>(ctas_needed < cap ? ctas_needed : cap);
    q8_k128_kernel<<<grid, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const float4*>(x), static_cast<uint8_t*>(out), nblocks, d_flags);
    return iqq::launch_status();
}
