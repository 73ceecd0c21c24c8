// qx_0_w.cu -- imatrix-weighted Q4_0 (and Q5_0, Q6_0, Q8_0) quantization on sm_100a.
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
// The same search serves the family's other 32-value formats (§一 names
// quantize_row_q5_0_impl, ..._q6_0_impl): nmax = 16, 32, 128, codes in
// [-nmax, nmax-1], candidates c_k = (float)(nmax*(80+k))/80 (the Q4_0 set for
// nmax = 8); the kernel is a template on the bit width.
//
// The work is ALU bound (about 150 binary32 operations per value against
// 4.6 bytes of HBM traffic), so the design is about instruction count and
// issue efficiency:
//  - one thread owns one 32-value block, so every sum is a private sequential
//    fmaf chain in exactly the order the definition fixes (no shuffles, no
//    reordering: bit-exact by construction);
//  - the candidate sweep runs on |x| with the sign folded out: for candidate k
//    the code magnitude is m = min(rint(a_k*|x_j|), B_j) with a_k = c_k/|xmax|
//    and B_j = 8 when x_j has the sign of xmax (code <= 0, clamped at -8) and
//    7 otherwise.  With w >= 0 every term w*x*l then has the sign of -xmax, so
//    |sumlx| = sum fmaf(|wx_j|, m_j, .) bit for bit (round to nearest is
//    sign-symmetric) and the score needs only that magnitude;
//  - rint of 0 <= v < 2^22 is either cvt.rni (one conversion-pipe op) or
//    (v + 1.5*2^23) - 1.5*2^23 (two FMA-pipe adds); the sweep mixes the two
//    to balance the pipes, and the clamp is one min against B_j;
//  - greedy pass 1 runs per thread (sequential, as defined, two trials evaluated per
//    state); the few blocks whose first pass moved a code finish passes 2..5
//    warp-cooperatively;
//  - sigma2 is a binary64 CTA reduction over the row (exact squares), the one
//    place where the summation order differs from the sequential definition; rows
//    spanning 4 or more CTAs may take it from a per-row pass into a workspace.
//
// CTA = 128 threads = 128 consecutive blocks of one row ("chunk"); each CTA
// reduces sigma2 over its whole row (the row is read from HBM once and from L2
// by the row's other chunks).  Per warp, shared memory holds the weights w of
// its 32 blocks and a scratch area used first by the sweep (|wx| and the clamp
// bounds) and then by the later steps (x and the codes), whose per-value loops
// then need no registers per value and stay rolled (small code, fewer
// registers).  Built with -fmad=false: no
// contraction except the explicit __fmaf_rn calls.
#include <cuda_fp16.h>

#include <type_traits>

#include "common.cuh"

namespace {

constexpr int QK = IQQ_Q4_0_BLOCK_VALUES;
constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kCand = 19;
constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
constexpr unsigned kFull = 0xffffffffu;

// Per-warp shared memory (floats).  Rows of 36 keep LDS.128/STS.128 16-byte
// aligned and conflict-free (8 lanes per phase hit 8 distinct 4-bank groups);
// rows of 33 keep scalar column accesses conflict-free.
constexpr int kRow4 = QK + 4;
constexpr int kRow1 = QK + 1;
#ifndef IQQ_SWEEP_CPI
#define IQQ_SWEEP_CPI 2  // candidates per sweep iteration
#endif
#ifndef IQQ_SWEEP_CVT_MASK
#define IQQ_SWEEP_CVT_MASK 1  // bit c set: candidate c of a group rounds with cvt.rni
#endif
constexpr int kW = 0;                    // w[32][36]
constexpr int kScratch = 32 * kRow4;     // sweep: |wx|[32][36], B[32][36]; later: x[32][33], l[32][33]
constexpr int kAwx = kScratch;
constexpr int kUb = kAwx + 32 * kRow4;
constexpr int kWarpFloats = kUb + 32 * kRow4;
static_assert(kScratch + 2 * 32 * kRow1 <= kWarpFloats, "staging fits in the sweep area");

#ifndef IQQ_PASS1_SPEC
#define IQQ_PASS1_SPEC 2  // greedy pass 1: trials evaluated together against one state (measured: 2 best of 1-8)
#endif
#ifndef IQQ_Q4_MIN_CTAS
#define IQQ_Q4_MIN_CTAS 4  // resident CTAs per SM the register budget is sized for
#endif

// Formats: bits -> nmax (codes in [-nmax, nmax-1]) and block bytes.
template <int BITS> struct Fmt;
template <> struct Fmt<4> { static constexpr int nmax = 8, bytes = 18, fi = 0; };
template <> struct Fmt<5> { static constexpr int nmax = 16, bytes = 22, fi = 1; };
template <> struct Fmt<6> { static constexpr int nmax = 32, bytes = 26, fi = 2; };
template <> struct Fmt<8> { static constexpr int nmax = 128, bytes = 34, fi = 3; };

// c_k = (float)(nmax * (80 + k)) / 80 for k = -9..9, each the IEEE quotient (for
// nmax = 8 these are (80 + k)/10).
#define IQQ_C(n, k) (static_cast<float>((n) * (80 + (k))) / 80.0f)
#define IQQ_CROW(n)                                                                                   \
    {IQQ_C(n, -9), IQQ_C(n, -8), IQQ_C(n, -7), IQQ_C(n, -6), IQQ_C(n, -5), IQQ_C(n, -4), IQQ_C(n, -3), \
     IQQ_C(n, -2), IQQ_C(n, -1), IQQ_C(n, 0),  IQQ_C(n, 1),  IQQ_C(n, 2),  IQQ_C(n, 3),  IQQ_C(n, 4),  \
     IQQ_C(n, 5),  IQQ_C(n, 6),  IQQ_C(n, 7),  IQQ_C(n, 8),  IQQ_C(n, 9)}
__constant__ float c_cand_all[4][kCand] = {IQQ_CROW(8), IQQ_CROW(16), IQQ_CROW(32), IQQ_CROW(128)};
#undef IQQ_CROW
#undef IQQ_C

// rint(v) for |v| < 2^22, half to even.
__device__ __forceinline__ float rint_small(float v) { return __fsub_rn(__fadd_rn(v, kMagic), kMagic); }

template <int NMAX>
__device__ __forceinline__ float clamp_code(float r)
{
    return fminf(fmaxf(r, static_cast<float>(-NMAX)), static_cast<float>(NMAX - 1));
}

__device__ __forceinline__ double block_reduce_sum(double v, double* s_red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) s_red[warp] = v;
    __syncthreads();
    double t = 0.0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) t += s_red[w];
    __syncthreads();
    return t;
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


// N candidates k0..k0+N-1 over the block.  Per value and candidate: v = a_k*|x|,
// the code magnitude m = min(rint(v), B) -- rint either by cvt.rni, or as
// min(v + M, M + B) - M -- then the two sequential sums |sumlx| += |wx|*m and
// suml2 += w*m*m.  |wx|, B, M + B and w stream from this thread's rows of the
// warp's shared memory (LDS.128).
template <int BITS, int N>
__device__ __forceinline__ void sweep_group(int k0, const float (&xv)[QK], const float* __restrict__ my_w,
                                            const float* __restrict__ my_awx,
                                            const float* __restrict__ my_ub, float amax,
                                            float& best, int& kbest)
{
    constexpr int kMask = IQQ_SWEEP_CVT_MASK & ((1 << N) - 1);
    float a[N], s[N], t[N];
#pragma unroll
    for (int c = 0; c < N; ++c) {
        a[c] = __fdiv_rn(c_cand_all[Fmt<BITS>::fi][k0 + c], amax);  // |iscale_k|
        s[c] = 0.0f;
        t[c] = 0.0f;
    }
#pragma unroll
    for (int j4 = 0; j4 < QK; j4 += 4) {
        const float4 aw = *reinterpret_cast<const float4*>(my_awx + j4);
        const float4 ub = *reinterpret_cast<const float4*>(my_ub + j4);
        const float4 ww = *reinterpret_cast<const float4*>(my_w + j4);
        const float awv[4] = {aw.x, aw.y, aw.z, aw.w};
        const float ubv[4] = {ub.x, ub.y, ub.z, ub.w};
        const float wv[4] = {ww.x, ww.y, ww.z, ww.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
#pragma unroll
            for (int c = 0; c < N; ++c) {
                const float v = __fmul_rn(a[c], fabsf(xv[j4 + q]));
                // rint(v): one conversion-pipe op, or two FMA-pipe adds
                const float r = ((kMask >> c) & 1) ? rintf(v) : rint_small(v);
                const float m = fminf(r, ubv[q]);
                s[c] = __fmaf_rn(awv[q], m, s[c]);
                t[c] = __fmaf_rn(wv[q], __fmul_rn(m, m), t[c]);
            }
        }
        // compiler-only fence: keeps each group's shared-memory loads beside its
        // arithmetic instead of hoisting all of them (which costs registers)
        asm volatile("" ::: "memory");
    }
#pragma unroll
    for (int c = 0; c < N; ++c) keep_best(s[c], t[c], k0 + c, best, kbest);
}

// Greedy passes 2..5 for the warp's blocks whose first pass changed a code (bit
// set in `pending`), one block at a time, lane j holding element j.  All trial
// moves of a pass that precede the next accepted move see the same (sumlx,
// suml2, score), so they are evaluated together; the lowest accepting lane is the
// move the sequential pass accepts first.  The state then advances and the scan
// resumes after that element, so the sequence of accepted moves and every
// rounding is that of the sequential Gauss-Seidel passes.
template <int NMAX>
__device__ __forceinline__ void greedy_warp(const float* sX, const float* sW, float* sL, unsigned pending,
                                            float sumlx, float suml2, float score)
{
    const int lane = threadIdx.x & 31;
#pragma unroll 1
    while (pending != 0u) {
        const int bb = __ffs(pending) - 1;
        pending &= pending - 1u;
        float lx = __shfl_sync(kFull, sumlx, bb);
        float l2 = __shfl_sync(kFull, suml2, bb);
        float sc = __shfl_sync(kFull, score, bb);
        const float xj = sX[bb * kRow1 + lane];
        const float wj = sW[bb * kRow4 + lane];
        float lj = sL[bb * kRow1 + lane];
        const float wxj = __fmul_rn(wj, xj);
        float d = __fdiv_rn(lx, l2);
        int passes = 2, start = 0;
        bool changed = false;
#pragma unroll 1
        while (true) {
            const float g = __fmul_rn(d, __fmul_rn(wj, __fsub_rn(xj, __fmul_rn(d, lj))));
            const float sg = g > 0.0f ? 1.0f : -1.0f;
            const float ln = __fadd_rn(lj, sg);
            const float nlx = __fadd_rn(lx, __fmul_rn(sg, wxj));
            const float nl2 = __fmaf_rn(wj, __fadd_rn(__fmul_rn(__fmul_rn(2.0f, sg), lj), 1.0f), l2);
            bool ok = lane >= start && (g > 0.0f || g < 0.0f) && ln >= static_cast<float>(-NMAX) &&
                      ln <= static_cast<float>(NMAX - 1) && nl2 > 0.0f;
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
        sL[bb * kRow1 + lane] = lj;
    }
}

// EPI: the epilogue of the blocks just written may also (y_out) store their dequantized
// values y = fp16(d) * l (exact in binary32, the dequantization's bits) and (acc_out)
// accumulate their round trip exactly as the weighted-RMSE reduction does: with e = x - y
// in binary32, {sum qw e^2, sum qw, sum e^2} in binary64 and max |e|, one set of atomics
// per warp (no CTA barrier).
template <int BITS, bool EPI, typename XT>
__global__ void __launch_bounds__(kThreads, IQQ_Q4_MIN_CTAS)
qx_0_w_kernel(const XT* __restrict__ x, const float* __restrict__ qw, uint8_t* __restrict__ out,
              int64_t nrows, int64_t n_per_row, int64_t rows_per_qw, int weight_mode, float fudge,
              int chunks_per_row, const float* __restrict__ row_sigma2, float* __restrict__ y_out,
              double* __restrict__ acc_out, uint32_t* __restrict__ flags)
{
    extern __shared__ float smem[];
    __shared__ double s_red[kWarps];
    const int lane = threadIdx.x & 31;
    float* const warp_smem = smem + (threadIdx.x >> 5) * kWarpFloats;
    float* const sW = warp_smem + kW;
    float* const my_w = sW + lane * kRow4;
    float* const my_awx = warp_smem + kAwx + lane * kRow4;
    float* const my_ub = warp_smem + kUb + lane * kRow4;
    float* const sX = warp_smem + kScratch;             // x and the codes, after the sweep
    float* const sL = warp_smem + kScratch + 32 * kRow1;
    float* const my_x = sX + lane * kRow1;
    float* const my_l = sL + lane * kRow1;
    constexpr int NMAX = Fmt<BITS>::nmax;
    const int64_t nb = n_per_row / QK;
    const int64_t nwork = nrows * chunks_per_row;

    for (int64_t cta = blockIdx.x; cta < nwork; cta += gridDim.x) {
        const int64_t row = cta / chunks_per_row;
        const int chunk = static_cast<int>(cta - row * chunks_per_row);
        const XT* xr = x + row * n_per_row;
        const int64_t qrow = rows_per_qw > 0 ? row / rows_per_qw : 0;
        const float* qr = qw != nullptr ? qw + qrow * n_per_row : nullptr;
        uint32_t bad = 0u;

        // this thread's block (lanes past the row's end idle but join the warp steps);
        // its loads are issued first so that they overlap the row reduction below
        const int64_t b = static_cast<int64_t>(chunk) * kThreads + threadIdx.x;
        const bool valid = b < nb;
        float xv[QK];
        float4 q4[QK / 4];
        if (valid) {
            const XT* xb = xr + b * QK;
#pragma unroll
            for (int i = 0; i < QK / 4; ++i) {
                const float4 v = iqq::ld4(xb + 4 * i);
                xv[4 * i] = v.x; xv[4 * i + 1] = v.y; xv[4 * i + 2] = v.z; xv[4 * i + 3] = v.w;
            }
            if (qr != nullptr) {
                const float4* qb4 = reinterpret_cast<const float4*>(qr + b * QK);
#pragma unroll
                for (int i = 0; i < QK / 4; ++i) q4[i] = __ldg(qb4 + i);
            } else {
#pragma unroll
                for (int i = 0; i < QK / 4; ++i) q4[i] = make_float4(1.0f, 1.0f, 1.0f, 1.0f);
            }
        } else {
#pragma unroll
            for (int j = 0; j < QK; ++j) xv[j] = 0.0f;
#pragma unroll
            for (int i = 0; i < QK / 4; ++i) q4[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }

        // sigma2: binary64 sum of exact squares over the whole row -- reduced here, or
        // read from the per-row pass (which also reports non-finite x)
        float sigma2;
        if (row_sigma2 != nullptr) {
            sigma2 = __ldg(row_sigma2 + row);
        } else {
            double acc = 0.0;
            float nf = 0.0f;
            for (int64_t i = threadIdx.x; i < n_per_row / 4; i += kThreads) {
                const float4 v = iqq::ld4(xr + 4 * i);
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
            sigma2 = static_cast<float>(sum / static_cast<double>(n_per_row));
        }
        // the importance's correction factor on the sigma2 term (1: none)
        sigma2 = __fmul_rn(fudge, sigma2);

        if (valid && qr != nullptr && (rows_per_qw > 0 ? row % rows_per_qw == 0 : row == 0)) {
            float qmin = q4[0].x, qnf = 0.0f;
#pragma unroll
            for (int i = 0; i < QK / 4; ++i) {
                qmin = fminf(fminf(qmin, q4[i].x), fminf(q4[i].y, fminf(q4[i].z, q4[i].w)));
                qnf = __fmaf_rn(q4[i].x, 0.0f, qnf); qnf = __fmaf_rn(q4[i].y, 0.0f, qnf);
                qnf = __fmaf_rn(q4[i].z, 0.0f, qnf); qnf = __fmaf_rn(q4[i].w, 0.0f, qnf);
            }
            if (qnf != qnf) bad |= IQQ_FLAG_NONFINITE_INPUT;
            if (qmin < 0.0f) bad |= IQQ_FLAG_NEG_QW;
        }

        // importance weights (binary32, one rounding per operation) -> shared memory:
        // mode 0 qw*sqrt(sigma2 + x*x), 1 qw, 2 qw*(x*x), 3 qw*|x|, 4 qw*(sigma2 + x*x),
        // 5 qw*(sqrt(sigma2) + |x|); then xmax (signed value of the first largest |x|)
        const float sigma = weight_mode == 5 ? __fsqrt_rn(sigma2) : 0.0f;
#pragma unroll
        for (int i = 0; i < QK / 4; ++i) {
            float4 w4 = q4[i];
            float* wp[4] = {&w4.x, &w4.y, &w4.z, &w4.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float xj = xv[4 * i + k];
                const float t = __fmul_rn(xj, xj);
                float m;
                switch (weight_mode) {
                case 0: m = __fsqrt_rn(__fadd_rn(sigma2, t)); break;
                case 2: m = t; break;
                case 3: m = fabsf(xj); break;
                case 4: m = __fadd_rn(sigma2, t); break;
                case 5: m = __fadd_rn(sigma, fabsf(xj)); break;
                default: m = 1.0f; break;
                }
                if (weight_mode != 1) *wp[k] = __fmul_rn(*wp[k], m);
            }
            *reinterpret_cast<float4*>(my_w + 4 * i) = w4;
        }
        float amax = 0.0f, xmax = 0.0f;
#pragma unroll
        for (int j = 0; j < QK; ++j) {
            const float a = fabsf(xv[j]);
            if (a > amax) { amax = a; xmax = xv[j]; }
        }

        // candidate sweep
        float best = -INFINITY;
        int kbest = 0;
        {
            const uint32_t sxm = __float_as_uint(xmax);
#pragma unroll
            for (int j4 = 0; j4 < QK; j4 += 4) {
                const float4 w4 = *reinterpret_cast<const float4*>(my_w + j4);
                // |wx| and the clamp bound B: nmax when x_j has the sign of xmax (its code
                // is <= 0, clamped at -nmax), nmax - 1 otherwise
#define IQQ_DIFF(j) ((__float_as_uint(xv[j]) ^ sxm) >> 31)
                *reinterpret_cast<float4*>(my_awx + j4) =
                    make_float4(fabsf(__fmul_rn(w4.x, xv[j4])), fabsf(__fmul_rn(w4.y, xv[j4 + 1])),
                                fabsf(__fmul_rn(w4.z, xv[j4 + 2])), fabsf(__fmul_rn(w4.w, xv[j4 + 3])));
                constexpr float kB0 = static_cast<float>(NMAX), kB1 = static_cast<float>(NMAX - 1);
                *reinterpret_cast<float4*>(my_ub + j4) =
                    make_float4(IQQ_DIFF(j4) ? kB1 : kB0, IQQ_DIFF(j4 + 1) ? kB1 : kB0,
                                IQQ_DIFF(j4 + 2) ? kB1 : kB0, IQQ_DIFF(j4 + 3) ? kB1 : kB0);
#undef IQQ_DIFF
            }
            if (amax > 0.0f) {
                constexpr int N = IQQ_SWEEP_CPI;
                int k0 = 0;
#pragma unroll 1
                for (; k0 + N <= kCand; k0 += N)
                    sweep_group<BITS, N>(k0, xv, my_w, my_awx, my_ub, amax, best, kbest);
#pragma unroll 1
                for (; k0 < kCand; ++k0) sweep_group<BITS, 1>(k0, xv, my_w, my_awx, my_ub, amax, best, kbest);
            }
        }
        __syncwarp();  // the sweep area becomes the x / code staging area
#pragma unroll
        for (int j = 0; j < QK; ++j) my_x[j] = xv[j];

        // codes of the winner (or of k = 0 for the fallback) and the greedy state
        int mode = 0;  // 0: nothing to search (all-zero or no block), 1: fallback, 2: search
        float sumlx = 0.0f, suml2 = 0.0f, score = 0.0f, dfb = 0.0f;
        {
            float iscale = 0.0f;
            if (amax > 0.0f) {
                if (best == -INFINITY) {
                    // no candidate has positive weighted code energy: codes of k = 0, d = 1/iscale_0
                    iscale = __fdiv_rn(static_cast<float>(-NMAX), xmax);
                    dfb = __fdiv_rn(1.0f, iscale);
                    mode = 1;
                } else {
                    iscale = __fdiv_rn(-c_cand_all[Fmt<BITS>::fi][kbest], xmax);
                    score = best;
                    mode = 2;
                }
            }
#pragma unroll 4
            for (int j = 0; j < QK; ++j) {
                const float xj = my_x[j], wj = my_w[j];
                const float l = clamp_code<NMAX>(rint_small(__fmul_rn(iscale, xj)));
                my_l[j] = l;
                sumlx = __fmaf_rn(__fmul_rn(wj, xj), l, sumlx);
                suml2 = __fmaf_rn(wj, __fmul_rn(l, l), suml2);
            }
        }
        // greedy pass 1: this thread's block, sequential over j, exactly as defined.  The
        // state (sumlx, suml2, score, d) changes only when a move is accepted, so the trials
        // of IQQ_PASS1_SPEC consecutive elements are evaluated together against the current
        // state; the first one that passes the cheap rejection test is then decided exactly
        // as the sequential pass decides it, and the scan resumes after it.  The sequence of
        // accepted moves and every rounding are those of the element-by-element pass.
        bool changed = false;
        if (mode == 2) {
            float d = __fdiv_rn(sumlx, suml2);
            constexpr int U = IQQ_PASS1_SPEC;
            int j = 0;
#pragma unroll 1
            while (j < QK) {
                float t_ln[U], t_nlx[U], t_nl2[U], t_a2[U];
                int first = U;
#pragma unroll
                for (int u = U - 1; u >= 0; --u) {
                    const int jj = j + u < QK ? j + u : QK - 1;  // past the end: recomputes the last, unused
                    const float xj = my_x[jj], wj = my_w[jj], lj = my_l[jj];
                    const float g = __fmul_rn(d, __fmul_rn(wj, __fsub_rn(xj, __fmul_rn(d, lj))));
                    const float sg = g > 0.0f ? 1.0f : -1.0f;
                    t_ln[u] = __fadd_rn(lj, sg);
                    t_nlx[u] = __fadd_rn(sumlx, __fmul_rn(sg, __fmul_rn(wj, xj)));
                    t_nl2[u] = __fmaf_rn(wj, __fadd_rn(__fmul_rn(__fmul_rn(2.0f, sg), lj), 1.0f), suml2);
                    t_a2[u] = __fmul_rn(t_nlx[u], t_nlx[u]);
                    // rejected for certain when fl(nlx^2) <= thr = fl(fl(score*nl2)*(1 - 2^-22)):
                    // with no underflow or overflow (thr in [1e-30, 1e30]) thr < score*nl2, so
                    // then nlx^2/nl2 < score exactly and its rounded quotient cannot exceed score
                    const float thr = __fmul_rn(__fmul_rn(score, t_nl2[u]), 0.99999976158142089844f);
                    const bool maybe = !(t_a2[u] <= thr && thr >= 1e-30f && thr <= 1e30f);
                    const bool cand = maybe && (g > 0.0f || g < 0.0f) && t_ln[u] >= static_cast<float>(-NMAX) &&
                                      t_ln[u] <= static_cast<float>(NMAX - 1) && t_nl2[u] > 0.0f && j + u < QK;
                    if (cand) first = u;  // descending u: the lowest candidate wins
                }
                if (first == U) {
                    j += U;
                    continue;
                }
                // element j + first: the sequential pass's decision, from the same state
                float ln = t_ln[0], nlx = t_nlx[0], nl2 = t_nl2[0], a2 = t_a2[0];
#pragma unroll
                for (int u = 1; u < U; ++u)
                    if (first == u) { ln = t_ln[u]; nlx = t_nlx[u]; nl2 = t_nl2[u]; a2 = t_a2[u]; }
                const float ns = __fdiv_rn(a2, nl2);
                if (ns > score) {
                    my_l[j + first] = ln;
                    sumlx = nlx;
                    suml2 = nl2;
                    score = ns;
                    d = __fdiv_rn(sumlx, suml2);
                    changed = true;
                }
                j += first + 1;
            }
        }
        // passes 2..5, warp-cooperatively, for the blocks whose first pass moved a code
        const unsigned pending = __ballot_sync(kFull, changed);
        if (pending != 0u) {
            __syncwarp();
            greedy_warp<NMAX>(sX, sW, sL, pending, sumlx, suml2, score);
        }
        __syncwarp();

        // final sums from the final codes, d, and the packed block
        uint16_t d16 = 0;
        {
            float d = dfb;
            if (mode == 2) {
                float sfx = 0.0f, sf2 = 0.0f;
#pragma unroll 4
                for (int j = 0; j < QK; ++j) {
                    const float xj = my_x[j], wj = my_w[j], lj = my_l[j];
                    sfx = __fmaf_rn(__fmul_rn(wj, xj), lj, sfx);
                    sf2 = __fmaf_rn(wj, __fmul_rn(lj, lj), sf2);
                }
                d = __fdiv_rn(sfx, sf2);
            }
            if (mode != 0) {
                d16 = __half_as_ushort(__float2half_rn(d));
                if ((d16 & 0x7fffu) == 0x7c00u && isfinite(d)) bad |= IQQ_FLAG_SCALE_OVERFLOW;
            }
        }
        if (valid) {
            // biased code n = l + nmax: the low byte of (l + nmax + 1.5*2^23)
            auto biased = [&](int j) -> uint32_t {
                return __float_as_uint(__fadd_rn(my_l[j], kMagic + static_cast<float>(NMAX))) & 0xffu;
            };
            uint16_t* o16 = reinterpret_cast<uint16_t*>(out + (row * nb + b) * Fmt<BITS>::bytes);
            o16[0] = d16;
            if (BITS == 8) {
                // int8 codes: the low byte of (l + 1.5*2^23) is l in two's complement
#pragma unroll
                for (int i = 0; i < QK / 2; ++i) {
                    const uint32_t lo = __float_as_uint(__fadd_rn(my_l[2 * i], kMagic)) & 0xffu;
                    const uint32_t hi = __float_as_uint(__fadd_rn(my_l[2 * i + 1], kMagic)) & 0xffu;
                    o16[1 + i] = static_cast<uint16_t>(lo | (hi << 8));
                }
            } else {
                constexpr int kHighWords = BITS == 4 ? 0 : (BITS == 5 ? 2 : 4);  // 16-bit words of qh
                if (BITS != 4) {
                    uint32_t qh[2] = {0u, 0u};
#pragma unroll
                    for (int j = 0; j < QK; ++j) {
                        const uint32_t n = biased(j);
                        if (BITS == 5) qh[0] |= ((n >> 4) & 1u) << j;
                        else qh[j >> 4] |= ((n >> 4) & 3u) << (2 * (j & 15));
                    }
#pragma unroll
                    for (int i = 0; i < kHighWords; ++i)
                        o16[1 + i] = static_cast<uint16_t>(qh[i >> 1] >> (16 * (i & 1)));
                }
#pragma unroll
                for (int i = 0; i < QK / 4; ++i) {
                    // bytes 2i, 2i+1 of qs: low nibbles of codes 2i, 2i+1 and 2i+16, 2i+17
                    const uint32_t b0 = (biased(2 * i) & 15u) | ((biased(2 * i + 16) & 15u) << 4);
                    const uint32_t b1 = (biased(2 * i + 1) & 15u) | ((biased(2 * i + 17) & 15u) << 4);
                    o16[1 + kHighWords + i] = static_cast<uint16_t>(b0 | (b1 << 8));
                }
            }
        }
        if (EPI) {
            const bool want_acc = acc_out != nullptr;  // uniform
            double ew = 0.0, eq = 0.0, ee = 0.0;
            float em = 0.0f;
            if (valid) {
                const float dq = __half2float(__ushort_as_half(d16));
                float4* yb = y_out != nullptr ? reinterpret_cast<float4*>(y_out + row * n_per_row + b * QK) : nullptr;
                // the imatrix row again (recomputed rather than kept live across the sweep)
                const float* qre = qw != nullptr ? qw + (rows_per_qw > 0 ? row / rows_per_qw : 0) * n_per_row
                                                 : nullptr;
                const float4* q4p = qre != nullptr ? reinterpret_cast<const float4*>(qre + b * QK) : nullptr;
#pragma unroll 2
                for (int i = 0; i < QK / 4; ++i) {
                    float yk[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) yk[k] = __fmul_rn(dq, my_l[4 * i + k]);
                    if (yb != nullptr) __stcs(yb + i, make_float4(yk[0], yk[1], yk[2], yk[3]));
                    if (want_acc) {
                        const float4 qv = q4p != nullptr ? __ldg(q4p + i) : make_float4(1.0f, 1.0f, 1.0f, 1.0f);
                        const float qk[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const float e = __fsub_rn(my_x[4 * i + k], yk[k]);
                            const double ed = static_cast<double>(e);
                            const double e2 = ed * ed;  // exact
                            ew = fma(static_cast<double>(qk[k]), e2, ew);
                            eq += static_cast<double>(qk[k]);
                            ee += e2;
                            em = fmaxf(em, fabsf(e));
                        }
                    }
                }
            }
            if (want_acc) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    ew += __shfl_xor_sync(kFull, ew, o);
                    eq += __shfl_xor_sync(kFull, eq, o);
                    ee += __shfl_xor_sync(kFull, ee, o);
                    em = fmaxf(em, __shfl_xor_sync(kFull, em, o));
                }
                if (lane == 0) {
                    atomicAdd(acc_out + 0, ew);
                    atomicAdd(acc_out + 1, eq);
                    atomicAdd(acc_out + 2, ee);
                    // non-negative binary64 values order like their bit patterns
                    atomicMax(reinterpret_cast<unsigned long long*>(acc_out + 3),
                              static_cast<unsigned long long>(__double_as_longlong(static_cast<double>(em))));
                }
            }
        }
        iqq::raise_flags(flags, bad);
        __syncwarp();  // the warp's shared memory is rewritten by the next row
    }
}

constexpr size_t kDynSmem = sizeof(float) * kWarpFloats * kWarps;

// Rows spanning at least this many CTAs take sigma2 from a separate per-row pass when the
// caller provides a workspace: below it the fused reduction's re-reads of the row (from L2,
// once per chunk) cost less than a second pass over the tensor.
#ifndef IQQ_PREPASS_CHUNKS
#define IQQ_PREPASS_CHUNKS 4
#endif
constexpr int64_t kPrepassChunks = IQQ_PREPASS_CHUNKS;
constexpr int kPrepassThreads = 256;

// sigma2 of each row (the same binary64 sum of exact squares and rounding as the fused
// reduction), one CTA per row, and the non-finite check of x.
template <typename XT>
__global__ void __launch_bounds__(kPrepassThreads)
row_sigma2_kernel(const XT* __restrict__ x, int64_t nrows, int64_t n_per_row, float* __restrict__ out,
                  uint32_t* __restrict__ flags)
{
    __shared__ double s_red[kPrepassThreads / 32];
    for (int64_t row = blockIdx.x; row < nrows; row += gridDim.x) {
        const XT* xr = x + row * n_per_row;
        double acc = 0.0;
        float nf = 0.0f;
        for (int64_t i = threadIdx.x; i < n_per_row / 4; i += kPrepassThreads) {
            const float4 v = iqq::ld4_stream(xr + 4 * i);
            acc = fma(static_cast<double>(v.x), static_cast<double>(v.x), acc);
            acc = fma(static_cast<double>(v.y), static_cast<double>(v.y), acc);
            acc = fma(static_cast<double>(v.z), static_cast<double>(v.z), acc);
            acc = fma(static_cast<double>(v.w), static_cast<double>(v.w), acc);
            nf = __fmaf_rn(v.x, 0.0f, nf);
            nf = __fmaf_rn(v.y, 0.0f, nf);
            nf = __fmaf_rn(v.z, 0.0f, nf);
            nf = __fmaf_rn(v.w, 0.0f, nf);
        }
        iqq::raise_flags(flags, nf != nf ? IQQ_FLAG_NONFINITE_INPUT : 0u);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        if (lane == 0) s_red[warp] = acc;
        __syncthreads();
        if (threadIdx.x == 0) {
            double t = 0.0;
#pragma unroll
            for (int w = 0; w < kPrepassThreads / 32; ++w) t += s_red[w];
            out[row] = static_cast<float>(t / static_cast<double>(n_per_row));
        }
        __syncthreads();
    }
}

int64_t chunks_of(int64_t n_per_row) { return (n_per_row / QK + kThreads - 1) / kThreads; }

// Library-owned sigma2 rows for iqq_quantize_qx_0_w_static (one copy per device; calls that
// use it are ordered by their stream, so concurrent calls on different streams must not
// share a device).
static __device__ __align__(256) float g_static_sigma2[IQQ_STATIC_WS_ROWS];

int64_t workspace_bytes_for(int64_t nrows, int64_t n_per_row)
{
    if (nrows <= 0 || n_per_row <= 0 || chunks_of(n_per_row) < kPrepassChunks) return 0;
    return (nrows * 4 + 255) / 256 * 256;
}

template <int BITS, bool EPI, typename XT>
iqq_status launch_qx(const XT* x, const float* qw, void* out, int64_t nrows, int64_t n_per_row,
                     int64_t rows_per_qw, int weight_mode, float fudge, const float* row_sigma2, float* y_out,
                     double* acc, uint32_t* d_flags, void* stream)
{
    const int64_t nb = n_per_row / QK;
    const int64_t chunks = (nb + kThreads - 1) / kThreads;
    if (chunks > 0x7fffffff) return IQQ_ERR_SHAPE;
    const int64_t nwork = nrows * chunks;
    const int grid = static_cast<int>(nwork < 0x7fffffff ? nwork : 0x7fffffff);
    static thread_local int configured_device = -1;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return iqq::launch_status();
    if (configured_device != dev) {
        if (cudaFuncSetAttribute(qx_0_w_kernel<BITS, EPI, XT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kDynSmem)) != cudaSuccess)
            return iqq::launch_status();
        configured_device = dev;
    }
    qx_0_w_kernel<BITS, EPI, XT><<<grid, kThreads, kDynSmem, static_cast<cudaStream_t>(stream)>>>(
        x, qw, static_cast<uint8_t*>(out), nrows, n_per_row, rows_per_qw, weight_mode, fudge,
        static_cast<int>(chunks), row_sigma2, y_out, acc, d_flags);
    return iqq::launch_status();
}

template <int BITS, typename XT>
iqq_status launch_bits(const XT* x, const float* qw, void* out, int64_t nrows, int64_t n_per_row,
                       int64_t rows_per_qw, int weight_mode, float fudge, const float* rs, float* y_out,
                       double* acc, uint32_t* d_flags, void* stream)
{
    if (acc != nullptr || y_out != nullptr)
        return launch_qx<BITS, true, XT>(x, qw, out, nrows, n_per_row, rows_per_qw, weight_mode, fudge, rs, y_out,
                                     acc, d_flags, stream);
    return launch_qx<BITS, false, XT>(x, qw, out, nrows, n_per_row, rows_per_qw, weight_mode, fudge, rs, nullptr,
                                  nullptr, d_flags, stream);
}

// workspace == nullptr: the fused reduction.  Otherwise it holds at least
// workspace_bytes_for(nrows, n_per_row) bytes (checked by the caller).  acc: optional
// round-trip error accumulator (8-byte aligned, checked by the caller).
template <typename XT>
iqq_status quantize_qx(int bits, const XT* x, const float* qw, void* out, int64_t nrows,
                       int64_t n_per_row, int64_t rows_per_qw, int weight_mode, void* workspace,
                       uint32_t* d_flags, void* stream, double* acc = nullptr, float* y_out = nullptr,
                       float fudge = 1.0f, bool direct = false)
{
    if (bits != 4 && bits != 5 && bits != 6 && bits != 8) return IQQ_ERR_ARG;
    if (!iqq::size_ok(nrows, n_per_row, 4) || rows_per_qw < 0) return IQQ_ERR_SHAPE;
    if (n_per_row % QK != 0) return IQQ_ERR_SHAPE;
    if (weight_mode < 0 || weight_mode > 5) return IQQ_ERR_ARG;
    if (nrows == 0 || n_per_row == 0) return IQQ_OK;
    if (x == nullptr || out == nullptr) return IQQ_ERR_NULL;
    if (!iqq::aligned(x, 16) || (qw && !iqq::aligned(qw, 16)) || !iqq::aligned(out, 2) ||
        (d_flags && !iqq::aligned(d_flags, 4)))
        return IQQ_ERR_ALIGN;
    // Q4_0: the transition-based sweep (q4_0_w.cu), which computes each row's sigma2 itself
    // and needs no workspace; binary32 x with or without the epilogue outputs, bf16 x without
    if (bits == 4 && !direct && iqq::q4_0_w_fits(n_per_row)) {
        if constexpr (std::is_same<XT, float>::value)
            return iqq::launch_q4_0_w(x, qw, out, nrows, n_per_row, rows_per_qw, weight_mode, fudge, d_flags, stream,
                                      y_out, acc);
        else if (acc == nullptr && y_out == nullptr)
            return iqq::launch_q4_0_w(x, qw, out, nrows, n_per_row, rows_per_qw, weight_mode, fudge, d_flags, stream);
    }
    const float* rs = nullptr;
    if (workspace != nullptr && workspace_bytes_for(nrows, n_per_row) > 0) {
        float* ws = static_cast<float*>(workspace);
        const int64_t g = nrows < 0x7fffffff ? nrows : 0x7fffffff;
        row_sigma2_kernel<XT><<<static_cast<int>(g), kPrepassThreads, 0, static_cast<cudaStream_t>(stream)>>>(
            x, nrows, n_per_row, ws, d_flags);
        const iqq_status st = iqq::launch_status();
        if (st != IQQ_OK) return st;
        rs = ws;
    }
    switch (bits) {
    case 4: return launch_bits<4, XT>(x, qw, out, nrows, n_per_row, rows_per_qw, weight_mode, fudge, rs, y_out, acc, d_flags, stream);
    case 5: return launch_bits<5, XT>(x, qw, out, nrows, n_per_row, rows_per_qw, weight_mode, fudge, rs, y_out, acc, d_flags, stream);
    case 6: return launch_bits<6, XT>(x, qw, out, nrows, n_per_row, rows_per_qw, weight_mode, fudge, rs, y_out, acc, d_flags, stream);
    default: return launch_bits<8, XT>(x, qw, out, nrows, n_per_row, rows_per_qw, weight_mode, fudge, rs, y_out, acc, d_flags, stream);
    }
}

}  // namespace

extern "C" iqq_status iqq_quantize_q4_0_w(const float* x, const float* qw, void* out, int64_t nrows,
                                          int64_t n_per_row, int64_t rows_per_qw, int weight_mode,
                                          uint32_t* d_flags, void* stream)
{
    return quantize_qx(4, x, qw, out, nrows, n_per_row, rows_per_qw, weight_mode, nullptr, d_flags, stream);
}

extern "C" iqq_status iqq_quantize_q4_0_w_batch(const iqq_q4_0_problem* problems, int64_t count, int weight_mode,
                                                float fudge, uint32_t* d_flags, void* stream)
{
    if (count < 0) return IQQ_ERR_SHAPE;
    if (count > 0 && problems == nullptr) return IQQ_ERR_NULL;
    if (weight_mode < 0 || weight_mode > 5) return IQQ_ERR_ARG;
    if (!(fudge >= 0.0f) || !isfinite(fudge)) return IQQ_ERR_ARG;
    if (!iqq::aligned(d_flags, 4)) return IQQ_ERR_ALIGN;
    for (int64_t i = 0; i < count; ++i) {
        const iqq_q4_0_problem& q = problems[i];
        if (!iqq::size_ok(q.nrows, q.n_per_row, 4) || q.rows_per_qw < 0 || q.n_per_row % QK != 0)
            return IQQ_ERR_SHAPE;
        if (q.nrows == 0 || q.n_per_row == 0) continue;
        if (!iqq::q4_0_w_fits(q.n_per_row)) return IQQ_ERR_SHAPE;
        if (q.x == nullptr || q.out == nullptr) return IQQ_ERR_NULL;
        if (!iqq::aligned(q.x, 16) || (q.qw && !iqq::aligned(q.qw, 16)) || !iqq::aligned(q.out, 2))
            return IQQ_ERR_ALIGN;
    }
    return iqq::launch_q4_0_w_batch(problems, count, weight_mode, fudge, d_flags, stream);
}

extern "C" iqq_status iqq_quantize_q4_0_w_direct(const float* x, const float* qw, void* out, int64_t nrows,
                                                 int64_t n_per_row, int64_t rows_per_qw, int weight_mode,
                                                 uint32_t* d_flags, void* stream)
{
    return quantize_qx(4, x, qw, out, nrows, n_per_row, rows_per_qw, weight_mode, nullptr, d_flags, stream, nullptr,
                       nullptr, 1.0f, true);
}

extern "C" iqq_status iqq_quantize_qx_0_w(int bits, const float* x, const float* qw, void* out,
                                          int64_t nrows, int64_t n_per_row, int64_t rows_per_qw,
                                          int weight_mode, uint32_t* d_flags, void* stream)
{
    return quantize_qx(bits, x, qw, out, nrows, n_per_row, rows_per_qw, weight_mode, nullptr, d_flags, stream);
}

extern "C" iqq_status iqq_quantize_qx_0_w_static(int bits, const float* x, const float* qw, void* out,
                                                 int64_t nrows, int64_t n_per_row, int64_t rows_per_qw,
                                                 int weight_mode, uint32_t* d_flags, void* stream)
{
    if (bits != 4 && bits != 5 && bits != 6 && bits != 8) return IQQ_ERR_ARG;
    if (!iqq::size_ok(nrows, n_per_row, 4) || rows_per_qw < 0 || n_per_row % QK != 0) return IQQ_ERR_SHAPE;
    if (workspace_bytes_for(nrows, n_per_row) == 0)  // no per-row pass: the fused path
        return quantize_qx(bits, x, qw, out, nrows, n_per_row, rows_per_qw, weight_mode, nullptr, d_flags,
                           stream);
    if (weight_mode < 0 || weight_mode > 5) return IQQ_ERR_ARG;
    if (x == nullptr || out == nullptr) return IQQ_ERR_NULL;
    if (!iqq::aligned(x, 16) || (qw && !iqq::aligned(qw, 16)) || !iqq::aligned(out, 2) ||
        (d_flags && !iqq::aligned(d_flags, 4)))
        return IQQ_ERR_ALIGN;  // every host check before the first CUDA call
    void* ws = nullptr;
    if (cudaGetSymbolAddress(&ws, g_static_sigma2) != cudaSuccess) return iqq::launch_status();
    // row batches that fit the static rows; each batch is a tensor of its own rows.  With one
    // imatrix row per rows_per_qw rows, a batch is a whole number of imatrix groups, so that
    // it starts on an imatrix-row boundary and takes its imatrix rows from there; only a
    // group larger than the array itself is split, one part of one group per batch.
    const int64_t bb = bits == 4 ? Fmt<4>::bytes : bits == 5 ? Fmt<5>::bytes : bits == 6 ? Fmt<6>::bytes : Fmt<8>::bytes;
    const bool grouped = qw != nullptr && rows_per_qw > 0;
    const int64_t batch = grouped && rows_per_qw <= IQQ_STATIC_WS_ROWS
                              ? (IQQ_STATIC_WS_ROWS / rows_per_qw) * rows_per_qw
                              : IQQ_STATIC_WS_ROWS;
    for (int64_t r0 = 0; r0 < nrows;) {
        int64_t nr = nrows - r0 < batch ? nrows - r0 : batch;
        const float* qb = qw;
        int64_t rpq = rows_per_qw;
        if (grouped) {
            const int64_t q = r0 / rows_per_qw;
            qb = qw + q * n_per_row;
            if (rows_per_qw > IQQ_STATIC_WS_ROWS) {
                // a part of one imatrix group: it ends at the group's end at the latest
                const int64_t group_end = (q + 1) * rows_per_qw;
                if (r0 + nr > group_end) nr = group_end - r0;
                rpq = 0;
            }
        }
        const iqq_status st = quantize_qx(bits, x + r0 * n_per_row, qb,
                                          static_cast<uint8_t*>(out) + r0 * (n_per_row / QK) * bb, nr, n_per_row,
                                          rpq, weight_mode, ws, d_flags, stream);
        if (st != IQQ_OK) return st;
        r0 += nr;
    }
    return IQQ_OK;
}

extern "C" iqq_status iqq_quantize_qx_0_w_ex(int bits, const float* x, const float* qw, void* out,
                                             int64_t nrows, int64_t n_per_row, int64_t rows_per_qw,
                                             int weight_mode, float fudge, void* workspace,
                                             size_t workspace_bytes, float* y_out, double* d_acc,
                                             uint32_t* d_flags, void* stream)
{
    if (bits != 4 && bits != 5 && bits != 6 && bits != 8) return IQQ_ERR_ARG;
    if (!iqq::size_ok(nrows, n_per_row, 4) || rows_per_qw < 0 || n_per_row % QK != 0) return IQQ_ERR_SHAPE;
    const int64_t need = workspace_bytes_for(nrows, n_per_row);
    void* ws = nullptr;
    if (need > 0 && workspace != nullptr) {
        if (workspace_bytes < static_cast<size_t>(need)) return IQQ_ERR_SHAPE;
        if (!iqq::aligned(workspace, 16)) return IQQ_ERR_ALIGN;
        ws = workspace;
    }
    if (!iqq::aligned(d_acc, 8) || !iqq::aligned(y_out, 16)) return IQQ_ERR_ALIGN;
    if (!(fudge >= 0.0f) || !isfinite(fudge)) return IQQ_ERR_ARG;
    return quantize_qx(bits, x, qw, out, nrows, n_per_row, rows_per_qw, weight_mode, ws, d_flags, stream, d_acc,
                       y_out, fudge);
}

extern "C" size_t iqq_quantize_qx_0_w_workspace_bytes(int64_t nrows, int64_t n_per_row)
{
    return static_cast<size_t>(workspace_bytes_for(nrows, n_per_row));
}

extern "C" iqq_status iqq_quantize_qx_0_w_ws(int bits, const float* x, const float* qw, void* out,
                                             int64_t nrows, int64_t n_per_row, int64_t rows_per_qw,
                                             int weight_mode, void* workspace, size_t workspace_bytes,
                                             uint32_t* d_flags, void* stream)
{
    if (bits != 4 && bits != 5 && bits != 6 && bits != 8) return IQQ_ERR_ARG;
    if (!iqq::size_ok(nrows, n_per_row, 4) || rows_per_qw < 0 || n_per_row % QK != 0) return IQQ_ERR_SHAPE;
    const int64_t need = workspace_bytes_for(nrows, n_per_row);
    if (need > 0) {
        if (workspace == nullptr) return IQQ_ERR_NULL;
        if (workspace_bytes < static_cast<size_t>(need)) return IQQ_ERR_SHAPE;
        if (!iqq::aligned(workspace, 16)) return IQQ_ERR_ALIGN;
    }
    return quantize_qx(bits, x, qw, out, nrows, n_per_row, rows_per_qw, weight_mode,
                       need > 0 ? workspace : nullptr, d_flags, stream);
}

extern "C" iqq_status iqq_quantize_qx_0_w_bf16(int bits, const void* x, const float* qw, void* out,
                                               int64_t nrows, int64_t n_per_row, int64_t rows_per_qw,
                                               int weight_mode, void* workspace, size_t workspace_bytes,
                                               uint32_t* d_flags, void* stream)
{
    if (bits != 4 && bits != 5 && bits != 6 && bits != 8) return IQQ_ERR_ARG;
    if (!iqq::size_ok(nrows, n_per_row, 4) || rows_per_qw < 0 || n_per_row % QK != 0) return IQQ_ERR_SHAPE;
    const int64_t need = workspace_bytes_for(nrows, n_per_row);
    void* ws = nullptr;
    if (need > 0 && workspace != nullptr) {
        if (workspace_bytes < static_cast<size_t>(need)) return IQQ_ERR_SHAPE;
        if (!iqq::aligned(workspace, 16)) return IQQ_ERR_ALIGN;
        ws = workspace;
    }
    return quantize_qx(bits, static_cast<const __nv_bfloat16*>(x), qw, out, nrows, n_per_row, rows_per_qw,
                       weight_mode, ws, d_flags, stream);
}
