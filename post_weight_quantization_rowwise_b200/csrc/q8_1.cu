// q8_1.cu -- Q8_1 activation quantization (the overflowing format) on sm_100a.
//
// Page "ik_llama.cpp 量化精度修复实录：用 Q8_K_128 替代 Q8_1 根治 IQ1_S_R4 /
// IQ1_M_R4 的 fp16 溢出" (www.hnwysp.cn/news/39281), 修复前的数值隐患: Q8_1 keeps,
// per 32 activations, a binary16 scale d = x_max/127 and a binary16 sum
// s = d * sum(q); s can overflow binary16 while d fits, which breaks the
// subtract-the-sum correction of the 1-bit dot products.  This kernel exists to
// show and count that failure next to Q8_K_128 (which stores int16 sums).
//
// Per block: amax = max|x|, d = amax/127, id = amax > 0 ? 127/amax : 0,
// q = clamp(rint(x*id), -127, 127) (a NaN product gives 0), s = d*sum(q) in
// binary32; d and s stored as binary16 (RNE).  Layout: half d | half s |
// int8 qs[32] = 36 bytes.  The count of blocks whose stored s is +-Inf while d
// is finite is added to a caller-owned 64-bit counter.
//
// Mapping: one warp per 4 consecutive blocks (128 values, one 16-byte load per
// lane); the 8 lanes of a block reduce amax and the sum with 3 shuffles.
#include <cuda_fp16.h>

#include "common.cuh"

namespace {

constexpr int kThreads = 256;
constexpr int kBlockBytes = 36;

__device__ __forceinline__ int code_of(float x, float id)
{
    int q = __float2int_rn(__fmul_rn(x, id));  // cvt.rni: +-Inf saturates, NaN -> 0
    return max(-127, min(127, q));
}

__global__ void __launch_bounds__(kThreads)
q8_1_kernel(const float4* __restrict__ x, uint8_t* __restrict__ out, int64_t nblocks,
            unsigned long long* __restrict__ overflow, uint32_t* __restrict__ flags)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
    uint32_t bad = 0u;
    unsigned long long nover = 0ull;
    for (int64_t g4 = warp * 4; g4 < nblocks; g4 += nwarps * 4) {
        const int64_t g = g4 + (lane >> 3);  // this lane's block
        const bool valid = g < nblocks;
        const float4 a = valid ? iqq::ld_stream_f4(x + g4 * 8 + lane) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float z = __fmul_rn(a.x, 0.f) + __fmul_rn(a.y, 0.f) + __fmul_rn(a.z, 0.f) + __fmul_rn(a.w, 0.f);
        if (z != z) bad |= IQQ_FLAG_NONFINITE_INPUT;
        float amax = fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(a.z), fabsf(a.w)));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
        const float d = __fdiv_rn(amax, 127.0f);
        const float id = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;
        const int q0 = code_of(a.x, id), q1 = code_of(a.y, id), q2 = code_of(a.z, id), q3 = code_of(a.w, id);
        int sum = q0 + q1 + q2 + q3;
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
        sum += __shfl_xor_sync(0xffffffffu, sum, 4);
        if (valid) {
            uint8_t* blk = out + g * kBlockBytes;
            const uint32_t packed = (static_cast<uint32_t>(q0) & 0xffu) | ((static_cast<uint32_t>(q1) & 0xffu) << 8) |
                                    ((static_cast<uint32_t>(q2) & 0xffu) << 16) | (static_cast<uint32_t>(q3) << 24);
            reinterpret_cast<uint32_t*>(blk + 4)[lane & 7] = packed;
            if ((lane & 7) == 0) {
                const uint16_t hd = __half_as_ushort(__float2half_rn(d));
                const uint16_t hs = __half_as_ushort(__float2half_rn(__fmul_rn(d, static_cast<float>(sum))));
                *reinterpret_cast<uint32_t*>(blk) = static_cast<uint32_t>(hd) | (static_cast<uint32_t>(hs) << 16);
                if ((hs & 0x7fffu) == 0x7c00u && (hd & 0x7fffu) != 0x7c00u) ++nover;
            }
        }
    }
    iqq::raise_flags(flags, bad);
    if (overflow != nullptr) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) nover += __shfl_xor_sync(0xffffffffu, nover, o);
        if (lane == 0 && nover != 0ull) atomicAdd(overflow, nover);
    }
}

}  // namespace

extern "C" iqq_status iqq_quantize_q8_1(const float* x, void* out, int64_t nrows, int64_t n_per_row,
                                        unsigned long long* d_overflow, uint32_t* d_flags, void* stream)
{
    if (!iqq::size_ok(nrows, n_per_row, 4)) return IQQ_ERR_SHAPE;
    if (n_per_row % 32 != 0) return IQQ_ERR_SHAPE;
    if (nrows == 0 || n_per_row == 0) return IQQ_OK;
    if (x == nullptr || out == nullptr) return IQQ_ERR_NULL;
    if (!iqq::aligned(x, 16) || !iqq::aligned(out, 4) || (d_flags && !iqq::aligned(d_flags, 4)) ||
        (d_overflow && !iqq::aligned(d_overflow, 8)))
        return IQQ_ERR_ALIGN;
    const int64_t nblocks = nrows * (n_per_row / 32);
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t warps = (nblocks + 3) / 4;
    const int64_t need = (warps + kThreads / 32 - 1) / (kThreads / 32);
    const int64_t cap = static_cast<int64_t>(sms) * 8;
    const int grid = static_cast<int>(need < cap ? need : cap);
    q8_1_kernel<<<grid, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const float4*>(x), static_cast<uint8_t*>(out), nblocks, d_overflow, d_flags);
    return iqq::launch_status();
}
