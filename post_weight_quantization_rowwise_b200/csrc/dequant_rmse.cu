// dequant_rmse.cu -- Q4_0 dequantization and the round-trip weighted RMSE on sm_100a.
//
// Block format (written by q4_0_w.cu): bytes 0-1 binary16 d (LE), byte 2+i holds
// code i + 8 in its low nibble and code i+16 + 8 in its high nibble.  A value
// decodes to fp16(d) * (nibble - 8), exact in binary32.
//
// The weighted RMSE follows the quantize-stats statistics named on page
// "量化方法论实证：为什么 LQER/L²QER 难以改进 ik_llama.cpp 的 k-quants 与
// i-quants" (www.0539edu.com/news/4792009) §3.2 (rmse and maxerr), weighted by
// the imatrix entries qw: with e = x - y rounded to binary32 it adds
// {sum qw e^2, sum qw, sum e^2} in binary64 and takes max|e|.  The decoded y
// never goes to memory.
//
// Both kernels are HBM bound.  Thread mapping: one thread per 4 consecutive
// values (a "quad"); 8 quads make a block, so the 8 threads of a block share
// its 18 bytes through L1 and every warp reads/writes 512 contiguous bytes of
// float data per access.
#include <cuda_fp16.h>

#include "common.cuh"

namespace {

constexpr int kThreads = 256;

struct Quad {
    float d;        // block scale
    uint32_t nib4;  // four 4-bit codes (biased by 8), value k in bits 4k..4k+3
};

// The 4 nibbles of quad qd (values 4qd..4qd+3) of the 18-byte block at blk.
__device__ __forceinline__ Quad load_quad(const uint8_t* blk, int qd)
{
    const uint16_t* h = reinterpret_cast<const uint16_t*>(blk);
    const uint16_t d16 = __ldg(h);
    const int j = 1 + 2 * (qd & 3);  // u16 index of qs[4*(qd&3)]
    const uint32_t b = static_cast<uint32_t>(__ldg(h + j)) | (static_cast<uint32_t>(__ldg(h + j + 1)) << 16);
    // b holds qs bytes 4m..4m+3; values < 16 sit in low nibbles, values >= 16 in high nibbles
    const uint32_t sel = qd < 4 ? b : (b >> 4);
    const uint32_t n = (sel & 0xfu) | ((sel >> 4) & 0xf0u) | ((sel >> 8) & 0xf00u) | ((sel >> 12) & 0xf000u);
    Quad q;
    q.d = __half2float(__ushort_as_half(d16));
    q.nib4 = n;
    return q;
}

__device__ __forceinline__ float code_value(uint32_t nib4, int k)
{
    return static_cast<float>(static_cast<int>((nib4 >> (4 * k)) & 0xfu) - 8);
}

__global__ void __launch_bounds__(kThreads)
dequant_q4_0_kernel(const uint8_t* __restrict__ blocks, float4* __restrict__ y, int64_t nquads)
{
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; t < nquads; t += stride) {
        const int64_t g = t >> 3;
        const int qd = static_cast<int>(t & 7);
        const Quad q = load_quad(blocks + g * IQQ_Q4_0_BLOCK_BYTES, qd);
        float4 o;
        o.x = __fmul_rn(q.d, code_value(q.nib4, 0));
        o.y = __fmul_rn(q.d, code_value(q.nib4, 1));
        o.z = __fmul_rn(q.d, code_value(q.nib4, 2));
        o.w = __fmul_rn(q.d, code_value(q.nib4, 3));
        __stcs(y + t, o);  // streaming store: the output is not re-read here
    }
}

// Rows [blockIdx.y*rows_per_cta, ...) x column quad blockIdx.x*kThreads + threadIdx.x.
__global__ void __launch_bounds__(kThreads)
weighted_rmse_kernel(const float* __restrict__ x, const uint8_t* __restrict__ blocks,
                     const float* __restrict__ qw, int64_t nrows, int64_t n_per_row,
                     int64_t rows_per_qw, int rows_per_cta, double* __restrict__ acc)
{
    const int64_t nq = n_per_row / 4;
    const int64_t nb = n_per_row / IQQ_Q4_0_BLOCK_VALUES;
    const int64_t cq = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
    const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_cta;
    const int64_t r1 = min(nrows, r0 + rows_per_cta);

    double sw = 0.0, sq = 0.0, se = 0.0;
    float emax = 0.0f;
    if (cq < nq) {
        const int64_t b = cq >> 3;
        const int qd = static_cast<int>(cq & 7);
        double col[4] = {0.0, 0.0, 0.0, 0.0};
        double qd4[4] = {1.0, 1.0, 1.0, 1.0};
        int64_t cur = -1, nrow_cur = 0;
        for (int64_t r = r0; r < r1; ++r) {
            const int64_t qrow = rows_per_qw > 0 ? r / rows_per_qw : 0;
            if (qrow != cur) {
                if (cur >= 0) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        sw = fma(qd4[k], col[k], sw);
                        se += col[k];
                        sq = fma(qd4[k], static_cast<double>(nrow_cur), sq);
                        col[k] = 0.0;
                    }
                }
                if (qw != nullptr) {
                    const float4 w = __ldg(reinterpret_cast<const float4*>(qw + qrow * n_per_row) + cq);
                    qd4[0] = w.x; qd4[1] = w.y; qd4[2] = w.z; qd4[3] = w.w;
                }
                cur = qrow;
                nrow_cur = 0;
            }
            const float4 xv = iqq::ld_stream_f4(reinterpret_cast<const float4*>(x + r * n_per_row) + cq);
            const Quad q = load_quad(blocks + (r * nb + b) * IQQ_Q4_0_BLOCK_BYTES, qd);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float xk = k == 0 ? xv.x : k == 1 ? xv.y : k == 2 ? xv.z : xv.w;
                const float e = __fsub_rn(xk, __fmul_rn(q.d, code_value(q.nib4, k)));
                emax = fmaxf(emax, fabsf(e));
                const double ed = static_cast<double>(e);
                col[k] = fma(ed, ed, col[k]);
            }
            ++nrow_cur;
        }
        if (cur >= 0) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                sw = fma(qd4[k], col[k], sw);
                se += col[k];
                sq = fma(qd4[k], static_cast<double>(nrow_cur), sq);
            }
        }
    }

    // CTA reduction, then one atomic per quantity per CTA
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        sw += __shfl_xor_sync(0xffffffffu, sw, o);
        sq += __shfl_xor_sync(0xffffffffu, sq, o);
        se += __shfl_xor_sync(0xffffffffu, se, o);
        emax = fmaxf(emax, __shfl_xor_sync(0xffffffffu, emax, o));
    }
    __shared__ double s_w[kThreads / 32], s_q[kThreads / 32], s_e[kThreads / 32];
    __shared__ float s_m[kThreads / 32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) { s_w[warp] = sw; s_q[warp] = sq; s_e[warp] = se; s_m[warp] = emax; }
    __syncthreads();
    if (threadIdx.x == 0) {
        double a = 0.0, bq = 0.0, c = 0.0;
        float m = 0.0f;
        for (int w = 0; w < kThreads / 32; ++w) { a += s_w[w]; bq += s_q[w]; c += s_e[w]; m = fmaxf(m, s_m[w]); }
        atomicAdd(acc + 0, a);
        atomicAdd(acc + 1, bq);
        atomicAdd(acc + 2, c);
        // non-negative binary64 values order like their bit patterns
        atomicMax(reinterpret_cast<unsigned long long*>(acc + 3),
                  static_cast<unsigned long long>(__double_as_longlong(static_cast<double>(m))));
    }
}

int sm_count()
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

}  // namespace

extern "C" iqq_status iqq_dequant_q4_0(const void* blocks, float* y, int64_t nrows, int64_t n_per_row,
                                       void* stream)
{
    if (!iqq::size_ok(nrows, n_per_row, 4)) return IQQ_ERR_SHAPE;
    if (n_per_row % IQQ_Q4_0_BLOCK_VALUES != 0) return IQQ_ERR_SHAPE;
    if (nrows == 0 || n_per_row == 0) return IQQ_OK;
    if (blocks == nullptr || y == nullptr) return IQQ_ERR_NULL;
    if (!iqq::aligned(blocks, 2) || !iqq::aligned(y, 16)) return IQQ_ERR_ALIGN;
    const int64_t nquads = nrows * n_per_row / 4;
    const int64_t need = (nquads + kThreads - 1) / kThreads;
    const int64_t cap = static_cast<int64_t>(sm_count()) * 16;
    const int grid = static_cast<int>(need < cap ? need : cap);
    dequant_q4_0_kernel<<<grid, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint8_t*>(blocks), reinterpret_cast<float4*>(y), nquads);
    return iqq::launch_status();
}

extern "C" iqq_status iqq_weighted_rmse(const float* x, const void* blocks, const float* qw,
                                        int64_t nrows, int64_t n_per_row, int64_t rows_per_qw,
                                        double* d_acc, void* stream)
{
    if (!iqq::size_ok(nrows, n_per_row, 4) || rows_per_qw < 0) return IQQ_ERR_SHAPE;
    if (n_per_row % IQQ_Q4_0_BLOCK_VALUES != 0) return IQQ_ERR_SHAPE;
    if (nrows == 0 || n_per_row == 0) return IQQ_OK;
    if (x == nullptr || blocks == nullptr || d_acc == nullptr) return IQQ_ERR_NULL;
    if (!iqq::aligned(x, 16) || !iqq::aligned(blocks, 2) || (qw && !iqq::aligned(qw, 16)) ||
        !iqq::aligned(d_acc, 8))
        return IQQ_ERR_ALIGN;
    const int64_t nq = n_per_row / 4;
    const int64_t gx = (nq + kThreads - 1) / kThreads;
    // about 16 resident CTAs' worth per SM, at least 8 rows per CTA
    const int64_t target = static_cast<int64_t>(sm_count()) * 16;
    int64_t gy = target / gx;
    if (gy < 1) gy = 1;
    int64_t rpc = (nrows + gy - 1) / gy;
    if (rpc < 8) rpc = 8;
    gy = (nrows + rpc - 1) / rpc;
    if (gx > 0x7fffffff || gy > 65535) return IQQ_ERR_SHAPE;
    dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
    weighted_rmse_kernel<<<grid, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        x, static_cast<const uint8_t*>(blocks), qw, nrows, n_per_row, rows_per_qw,
        static_cast<int>(rpc), d_acc);
    return iqq::launch_status();
}
