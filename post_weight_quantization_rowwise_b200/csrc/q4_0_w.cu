// q4_0_w.cu -- imatrix-weighted Q4_0 quantization on sm_100a.
//
// Page "ik_llama.cpp 量化权重之谜：weight[j] = qw[j] * sqrtf(sigma2 +
// xb[j]*xb[j])的由来与原理" (www.dpshk.com/news/4810665), §一: per row
// sigma2 = sum_x2 / n_per_row; per 32-value block weight[j] = qw[j] *
// sqrtf(sigma2 + xb[j]*xb[j]) (or qw[j], §一/§二), then make_qx_quants(QK4_0,
// 8, ...): a weighted least-squares scale with sumlx = sum w*x*l,
// suml2 = sum w*l*l, d = sumlx/suml2, refined by greedy code moves driven by
// g = d*w*(x - d*l).  The candidate set, tie rule, stopping rule, rounding
// modes and byte layout are the readings the library documents in iqq.h:
//   iscale_k = -c_k/xmax, c_k = (float)(80+k)/10, k = -9..9;
//   l = clamp(rint(iscale_k*x), -8, 7); sums sequential over j with fmaf;
//   best score sumlx^2/suml2, ties to the lowest k;
//   <= 5 Gauss-Seidel passes, a +-1 move accepted iff the score rises;
//   final sums recomputed, d = sumlx/suml2 -> binary16 (RNE);
//   block = d16 (LE) | qs[i] = (l[i]+8) | (l[i+16]+8) << 4.
//
// This is ALU bound (about 150 binary32 operations per value against
// 4.6 bytes of HBM traffic), so the design is about instruction count:
//  - one thread owns one 32-value block with all of its state in registers,
//    so every sum is a private sequential fmaf chain in exactly the order the
//    definition fixes (no shuffles, no reordering: bit-exact by construction);
//  - the candidate sweep runs on |x| with the sign folded out: for candidate k
//    the code magnitude is m = min(rint(a_k*|x_j|), B_j) with a_k = c_k/|xmax|
//    and B_j = 8 when x_j has the sign of xmax (code <= 0, clamp at -8) and 7
//    otherwise.  Every term w*x*l then has the sign of -xmax, so
//    |sumlx| = sum fmaf(|wx_j|, m_j, .) bit for bit (round-to-nearest is
//    sign-symmetric) and the score needs only that magnitude;
//  - rint of 0 <= v < 2^22 is (v + 1.5*2^23) - 1.5*2^23, two full-rate adds,
//    and the clamp is a single min against M + B_j;
//  - sigma2 is a binary64 CTA reduction over the row (exact squares), the one
//    place where the summation order differs from the sequential definition.
//
// CTA = 128 threads = 128 consecutive blocks of one row ("chunk"); each CTA
// reduces sigma2 over its whole row (the row is read from HBM once and from L2
// by the row's other chunks).  Built with -fmad=false: no contraction except
// the explicit __fmaf_rn calls.
#include <cuda_fp16.h>

#include "common.cuh"

namespace {

constexpr int QK = IQQ_Q4_0_BLOCK_VALUES;
constexpr int kThreads = 128;
constexpr int kCand = 19;
constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23

// c_k = (float)(80 + k) / 10 for k = -9..9, each the IEEE quotient.
__constant__ float c_cand[kCand] = {
    71.0f / 10.0f, 72.0f / 10.0f, 73.0f / 10.0f, 74.0f / 10.0f, 75.0f / 10.0f,
    76.0f / 10.0f, 77.0f / 10.0f, 78.0f / 10.0f, 79.0f / 10.0f, 80.0f / 10.0f,
    81.0f / 10.0f, 82.0f / 10.0f, 83.0f / 10.0f, 84.0f / 10.0f, 85.0f / 10.0f,
    86.0f / 10.0f, 87.0f / 10.0f, 88.0f / 10.0f, 89.0f / 10.0f};

// rint(v) for |v| < 2^22, half to even.
__device__ __forceinline__ float rint_small(float v) { return __fsub_rn(__fadd_rn(v, kMagic), kMagic); }

__device__ __forceinline__ float clamp_code(float r) { return fminf(fmaxf(r, -8.0f), 7.0f); }

__device__ __forceinline__ double block_reduce_sum(double v, double* s_red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) s_red[warp] = v;
    __syncthreads();
    double t = 0.0;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) t += s_red[w];
    __syncthreads();
    return t;
}

constexpr unsigned kFull = 0xffffffffu;
constexpr int kRow = QK + 1;                 // padded smem row: conflict-free both ways
constexpr int kWarpSmemFloats = 3 * 32 * kRow;  // x, w, l of the warp's 32 blocks

// One candidate's sums over the block in the folded form: |sumlx| and suml2.
#define IQQ_SWEEP_TERM(a, s, t, j)                                                  \
    {                                                                               \
        const float v_ = __fmul_rn(a, fabsf(xv[j]));                                \
        const float m_ = __fsub_rn(fminf(__fadd_rn(v_, kMagic), ub[j]), kMagic);    \
        s = __fmaf_rn(awx[j], m_, s);                                               \
        t = __fmaf_rn(w[j], __fmul_rn(m_, m_), t);                                  \
    }

// Running arg-max of sumlx^2/suml2 over the candidates, strictly greater wins.
__device__ __forceinline__ void keep_best(float s, float t, int k, float& best, int& kbest)
{
    const float score = t > 0.0f ? __fdiv_rn(__fmul_rn(s, s), t) : -INFINITY;
    if (score > best) {
        best = score;
        kbest = k;
    }
}

// Candidate sweep of one block: returns the winning k index (0..18) and its score.
__device__ __forceinline__ void sweep_block(const float (&xv)[QK], const float (&w)[QK],
                                            const float (&awx)[QK], const float (&ub)[QK],
                                            float amax, float& best, int& kbest)
{
    best = -INFINITY;
    kbest = 0;
#pragma unroll 1
    for (int k = 0; k + 1 < kCand; k += 2) {
        const float a0 = __fdiv_rn(c_cand[k], amax);      // |iscale_k|
        const float a1 = __fdiv_rn(c_cand[k + 1], amax);
        float s0 = 0.0f, t0 = 0.0f, s1 = 0.0f, t1 = 0.0f;
#pragma unroll
        for (int j = 0; j < QK; ++j) {
            IQQ_SWEEP_TERM(a0, s0, t0, j)
            IQQ_SWEEP_TERM(a1, s1, t1, j)
        }
        keep_best(s0, t0, k, best, kbest);
        keep_best(s1, t1, k + 1, best, kbest);
    }
    {
        const float a0 = __fdiv_rn(c_cand[kCand - 1], amax);
        float s0 = 0.0f, t0 = 0.0f;
#pragma unroll
        for (int j = 0; j < QK; ++j) IQQ_SWEEP_TERM(a0, s0, t0, j)
        keep_best(s0, t0, kCand - 1, best, kbest);
    }
}

// Greedy refinement of the warp's 32 blocks, one block at a time, lane j holding
// element j.  All trial moves of a pass that precede the next accepted move see
// the same (sumlx, suml2, score), so they are evaluated together; the lowest
// accepting lane is the move the sequential pass accepts first.  The state then
// advances and the scan resumes after that element, so the sequence of accepted
// moves and every rounding is that of the sequential Gauss-Seidel passes.
__device__ __forceinline__ void greedy_warp(float* sx, float* sw, float* sl, float sumlx,
                                            float suml2, float score, bool active)
{
    const int lane = threadIdx.x & 31;
#pragma unroll 1
    for (int bb = 0; bb < 32; ++bb) {
        if (!__shfl_sync(kFull, static_cast<int>(active), bb)) continue;
        float lx = __shfl_sync(kFull, sumlx, bb);
        float l2 = __shfl_sync(kFull, suml2, bb);
        float sc = __shfl_sync(kFull, score, bb);
        const float xj = sx[bb * kRow + lane];
        const float wj = sw[bb * kRow + lane];
        float lj = sl[bb * kRow + lane];
        const float wxj = __fmul_rn(wj, xj);
        float d = __fdiv_rn(lx, l2);
        int passes = 1, start = 0;
        bool changed = false;
#pragma unroll 1
        while (true) {
            const float g = __fmul_rn(d, __fmul_rn(wj, __fsub_rn(xj, __fmul_rn(d, lj))));
            const float sg = g > 0.0f ? 1.0f : -1.0f;
            const float ln = __fadd_rn(lj, sg);
            const float nlx = __fadd_rn(lx, __fmul_rn(sg, wxj));
            const float nl2 = __fmaf_rn(wj, __fadd_rn(__fmul_rn(__fmul_rn(2.0f, sg), lj), 1.0f), l2);
            bool ok = lane >= start && (g > 0.0f || g < 0.0f) && ln >= -8.0f && ln <= 7.0f && nl2 > 0.0f;
            float ns = 0.0f;
            if (ok) {
                ns = __fdiv_rn(__fmul_rn(nlx, nlx), nl2);
                ok = ns > sc;
            }
            const unsigned m = __ballot_sync(kFull, ok);
            if (m == 0u) {                       // the rest of this pass accepts nothing
                if (!changed || passes == 5) break;
                ++passes;
                changed = false;
                start = 0;
                continue;
            }
            const int j0 = __ffs(m) - 1;
            if (lane == j0) lj = ln;
            lx = __shfl_sync(kFull, nlx, j0);
            l2 = __shfl_sync(kFull, nl2, j0);
            sc = __shfl_sync(kFull, ns, j0);
            d = __fdiv_rn(lx, l2);
            changed = true;
            start = j0 + 1;
            if (start == QK) {                   // the pass ended on an accepted move
                if (passes == 5) break;
                ++passes;
                changed = false;
                start = 0;
            }
        }
        sl[bb * kRow + lane] = lj;
    }
}

__global__ void __launch_bounds__(kThreads, 3)
q4_0_w_kernel(const float* __restrict__ x, const float* __restrict__ qw, uint8_t* __restrict__ out,
              int64_t nrows, int64_t n_per_row, int64_t rows_per_qw, int weight_mode,
              int chunks_per_row, uint32_t* __restrict__ flags)
{
    extern __shared__ float smem[];
    __shared__ double s_red[kThreads / 32];
    const int lane = threadIdx.x & 31;
    float* sx = smem + (threadIdx.x >> 5) * kWarpSmemFloats;
    float* sw = sx + 32 * kRow;
    float* sl = sw + 32 * kRow;
    const int64_t nb = n_per_row / QK;
    const int64_t nwork = nrows * chunks_per_row;

    for (int64_t cta = blockIdx.x; cta < nwork; cta += gridDim.x) {
        const int64_t row = cta / chunks_per_row;
        const int chunk = static_cast<int>(cta - row * chunks_per_row);
        const float* xr = x + row * n_per_row;
        const int64_t qrow = rows_per_qw > 0 ? row / rows_per_qw : 0;
        const float* qr = qw != nullptr ? qw + qrow * n_per_row : nullptr;
        uint32_t bad = 0u;

        // sigma2: binary64 sum of exact squares over the whole row
        double acc = 0.0;
        float nf = 0.0f;
        const float4* xr4 = reinterpret_cast<const float4*>(xr);
        for (int64_t i = threadIdx.x; i < n_per_row / 4; i += kThreads) {
            const float4 v = __ldg(xr4 + i);
            acc = fma(static_cast<double>(v.x), static_cast<double>(v.x), acc);
            acc = fma(static_cast<double>(v.y), static_cast<double>(v.y), acc);
            acc = fma(static_cast<double>(v.z), static_cast<double>(v.z), acc);
            acc = fma(static_cast<double>(v.w), static_cast<double>(v.w), acc);
            nf = __fmaf_rn(v.x, 0.0f, nf);  // becomes NaN on any Inf/NaN
            nf = __fmaf_rn(v.y, 0.0f, nf);
            nf = __fmaf_rn(v.z, 0.0f, nf);
            nf = __fmaf_rn(v.w, 0.0f, nf);
        }
        if (chunk == 0 && nf != nf) bad |= IQQ_FLAG_NONFINITE_INPUT;
        const double sum = block_reduce_sum(acc, s_red);
        const float sigma2 = static_cast<float>(sum / static_cast<double>(n_per_row));
        const bool check_qw = qr != nullptr && (rows_per_qw > 0 ? row % rows_per_qw == 0 : row == 0);

        // ---- per thread: one block (lanes past the row's end idle but join the warp steps)
        const int64_t b = static_cast<int64_t>(chunk) * kThreads + threadIdx.x;
        const bool valid = b < nb;
        float xv[QK], w[QK];
        int mode = 0;  // 0: nothing to search (all-zero or no block), 1: fallback, 2: search
        float sumlx = 0.0f, suml2 = 0.0f, score = 0.0f, dfb = 0.0f;
        {
            float l[QK];
            if (valid) {
                const float4* xb4 = reinterpret_cast<const float4*>(xr + b * QK);
#pragma unroll
                for (int i = 0; i < QK / 4; ++i) {
                    const float4 v = __ldg(xb4 + i);
                    xv[4 * i] = v.x; xv[4 * i + 1] = v.y; xv[4 * i + 2] = v.z; xv[4 * i + 3] = v.w;
                }
                if (qr != nullptr) {
                    const float4* qb4 = reinterpret_cast<const float4*>(qr + b * QK);
#pragma unroll
                    for (int i = 0; i < QK / 4; ++i) {
                        const float4 v = __ldg(qb4 + i);
                        w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
                    }
                    if (check_qw) {
                        float qmin = w[0], qnf = 0.0f;
#pragma unroll
                        for (int j = 0; j < QK; ++j) { qmin = fminf(qmin, w[j]); qnf = __fmaf_rn(w[j], 0.0f, qnf); }
                        if (qnf != qnf) bad |= IQQ_FLAG_NONFINITE_INPUT;
                        if (qmin < 0.0f) bad |= IQQ_FLAG_NEG_QW;
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < QK; ++j) w[j] = 1.0f;
                }
            } else {
#pragma unroll
                for (int j = 0; j < QK; ++j) { xv[j] = 0.0f; w[j] = 0.0f; }
            }
            // importance weights (binary32, one rounding per operation)
            if (weight_mode == 0) {
#pragma unroll
                for (int j = 0; j < QK; ++j) {
                    const float u = __fadd_rn(sigma2, __fmul_rn(xv[j], xv[j]));
                    w[j] = __fmul_rn(w[j], __fsqrt_rn(u));
                }
            }
            // xmax: signed value of the first element of largest |x|
            float amax = 0.0f, xmax = 0.0f;
#pragma unroll
            for (int j = 0; j < QK; ++j) {
                const float a = fabsf(xv[j]);
                if (a > amax) { amax = a; xmax = xv[j]; }
            }
            if (amax > 0.0f) {
                float best;
                int kbest;
                {
                    float awx[QK], ub[QK];
                    const uint32_t sxm = __float_as_uint(xmax);
#pragma unroll
                    for (int j = 0; j < QK; ++j) {
                        awx[j] = fabsf(__fmul_rn(w[j], xv[j]));
                        // clamp bound in the magic domain: M + 8 when x_j has the sign of
                        // xmax (its code is <= 0, clamped at -8), M + 7 otherwise
                        ub[j] = __uint_as_float(0x4B400008u - ((__float_as_uint(xv[j]) ^ sxm) >> 31));
                    }
                    sweep_block(xv, w, awx, ub, amax, best, kbest);
                }
                if (best == -INFINITY) {
                    // no candidate has positive weighted code energy: codes of k = 0, d = 1/iscale_0
                    const float iscale0 = __fdiv_rn(-8.0f, xmax);
#pragma unroll
                    for (int j = 0; j < QK; ++j) l[j] = clamp_code(rint_small(__fmul_rn(iscale0, xv[j])));
                    dfb = __fdiv_rn(1.0f, iscale0);
                    mode = 1;
                } else {
                    const float iscale = __fdiv_rn(-c_cand[kbest], xmax);
#pragma unroll
                    for (int j = 0; j < QK; ++j) {
                        l[j] = clamp_code(rint_small(__fmul_rn(iscale, xv[j])));
                        sumlx = __fmaf_rn(__fmul_rn(w[j], xv[j]), l[j], sumlx);
                        suml2 = __fmaf_rn(w[j], __fmul_rn(l[j], l[j]), suml2);
                    }
                    score = best;
                    mode = 2;
                }
            } else {
#pragma unroll
                for (int j = 0; j < QK; ++j) l[j] = 0.0f;
            }
            // stage x, w and the codes for the warp's greedy step
#pragma unroll
            for (int j = 0; j < QK; ++j) {
                sx[lane * kRow + j] = xv[j];
                sw[lane * kRow + j] = w[j];
                sl[lane * kRow + j] = l[j];
            }
        }
        __syncwarp();
        greedy_warp(sx, sw, sl, sumlx, suml2, score, mode == 2);
        __syncwarp();

        uint16_t d16 = 0;
        uint32_t nib[QK / 2];
        {
            float l[QK];
#pragma unroll
            for (int j = 0; j < QK; ++j) l[j] = sl[lane * kRow + j];
            float d = dfb;
            if (mode == 2) {
                sumlx = 0.0f;
                suml2 = 0.0f;
#pragma unroll
                for (int j = 0; j < QK; ++j) {
                    sumlx = __fmaf_rn(__fmul_rn(w[j], xv[j]), l[j], sumlx);
                    suml2 = __fmaf_rn(w[j], __fmul_rn(l[j], l[j]), suml2);
                }
                d = __fdiv_rn(sumlx, suml2);
            }
            if (mode != 0) {
                d16 = __half_as_ushort(__float2half_rn(d));
                if ((d16 & 0x7fffu) == 0x7c00u && isfinite(d)) bad |= IQQ_FLAG_SCALE_OVERFLOW;
            }
#pragma unroll
            for (int i = 0; i < QK / 2; ++i) {
                const uint32_t lo = static_cast<uint32_t>(static_cast<int>(l[i]) + 8);
                const uint32_t hi = static_cast<uint32_t>(static_cast<int>(l[i + QK / 2]) + 8);
                nib[i] = lo | (hi << 4);
            }
        }
        if (valid) {
            uint16_t* o16 = reinterpret_cast<uint16_t*>(out + (row * nb + b) * IQQ_Q4_0_BLOCK_BYTES);
            o16[0] = d16;
#pragma unroll
            for (int i = 0; i < QK / 4; ++i) o16[1 + i] = static_cast<uint16_t>(nib[2 * i] | (nib[2 * i + 1] << 8));
        }
        iqq::raise_flags(flags, bad);
        __syncwarp();  // the warp's staging area is rewritten by the next row
    }
}

constexpr size_t kDynSmem = sizeof(float) * kWarpSmemFloats * (kThreads / 32);

}  // namespace

extern "C" iqq_status iqq_quantize_q4_0_w(const float* x, const float* qw, void* out, int64_t nrows,
                                          int64_t n_per_row, int64_t rows_per_qw, int weight_mode,
                                          uint32_t* d_flags, void* stream)
{
    if (!iqq::size_ok(nrows, n_per_row, 4) || rows_per_qw < 0) return IQQ_ERR_SHAPE;
    if (n_per_row % QK != 0) return IQQ_ERR_SHAPE;
    if (weight_mode != 0 && weight_mode != 1) return IQQ_ERR_ARG;
    if (nrows == 0 || n_per_row == 0) return IQQ_OK;
    if (x == nullptr || out == nullptr) return IQQ_ERR_NULL;
    if (!iqq::aligned(x, 16) || (qw && !iqq::aligned(qw, 16)) || !iqq::aligned(out, 2) ||
        (d_flags && !iqq::aligned(d_flags, 4)))
        return IQQ_ERR_ALIGN;
    const int64_t nb = n_per_row / QK;
    const int64_t chunks = (nb + kThreads - 1) / kThreads;
    if (chunks > 0x7fffffff) return IQQ_ERR_SHAPE;
    const int64_t nwork = nrows * chunks;
    const int grid = static_cast<int>(nwork < 0x7fffffff ? nwork : 0x7fffffff);
    static thread_local int configured_device = -1;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return iqq::launch_status();
    if (configured_device != dev) {
        if (cudaFuncSetAttribute(q4_0_w_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kDynSmem)) != cudaSuccess)
            return iqq::launch_status();
        configured_device = dev;
    }
    q4_0_w_kernel<<<grid, kThreads, kDynSmem, static_cast<cudaStream_t>(stream)>>>(
        x, qw, static_cast<uint8_t*>(out), nrows, n_per_row, rows_per_qw, weight_mode,
        static_cast<int>(chunks), d_flags);
    return iqq::launch_status();
}
