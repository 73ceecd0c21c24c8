// q4_0_w.cu -- imatrix-weighted Q4_0 quantization (nmax = 8) on sm_100a with a
// transition-based candidate sweep.
//
// Page "ik_llama.cpp 量化权重之谜：weight[j] = qw[j] * sqrtf(sigma2 +
// xb[j]*xb[j])的由来与原理" (www.dpshk.com/news/4810665), §一: per row
// sigma2 = sum_x2 / n_per_row, per 32-value block weight[j] = qw[j] *
// sqrtf(sigma2 + xb[j]^2), then make_qx_quants(QK4_0, 8, ...): the weighted
// least-squares scale search (sumlx = sum w*x*l, suml2 = sum w*l*l,
// d = sumlx/suml2) and greedy code moves driven by g = d*w*(x - d*l).  The
// candidate set, tie rule, stopping rule, rounding and byte layout are the
// library's readings (iqq.h): iscale_k = -c_k/xmax, c_k = (float)(80+k)/10,
// k = -9..9; l = clamp(rint(iscale_k*x), -8, 7); fmaf sums sequential over j;
// the strictly best sumlx^2/suml2 wins (ties to the lowest k); <= 5
// Gauss-Seidel greedy passes; final d = sumlx/suml2 -> binary16.
//
// The result is bit for bit that of the direct definition.  What changes is how
// the winning candidate is found, since evaluating all 19 candidates' sequential
// sums costs about 130 operations per value:
//
//  1. Magnitudes.  With a_k = fl(c_k/|xmax|), |l| = min(rint(a_k*|x|), 8 or 7) (the
//     bound is 8 where x has the sign of xmax), because fl(-c_k/xmax) = -sign(xmax)*a_k
//     and rounding is sign symmetric; every term w*x*l of sumlx has the sign of -xmax, so
//     a candidate's sums are sums of nonnegative magnitudes.
//  2. Transitions.  |l| as a function of k is a nondecreasing step function.  Per
//     value the kernel evaluates it exactly at the first and last candidate (at
//     most two steps lie between them for nmax = 8) and places each step at the
//     first candidate whose code is larger, from a real-valued estimate of where
//     a_k*|xs| crosses the rounding boundary.  An estimate closer than 2^-10 of a
//     candidate to the boundary (exact ties included) is settled by evaluating
//     the code there exactly.  Each step adds |w*xs| and w*(2m+1) to per-candidate
//     difference sums.
//  3. Filter.  Prefix sums of the differences give candidate k's sums with a
//     relative error below (max(10, steps) + 1 + k)*2^-24; the exact sequential sums
//     are within 33*2^-24 of the same real values.  A candidate whose approximate
//     score lies further below the best approximate score than the two bounds
//     allow cannot be the exact winner, and a candidate with no step has the same
//     sums as its predecessor, so it cannot win the tie either.  The surviving
//     candidates (usually one) get their exact sequential sums, spread over the
//     warp's lanes.  Blocks outside the range where the bounds hold (tiny, huge or
//     non-finite values, empty weights) take the direct sweep.
//
// Work layout: a launch serves up to 64 tensors, whose blocks, each tensor in row-major
// order, are cut into 32-block tiles laid end to end; a persistent grid (one CTA per SM)
// splits the tiles into equal ranges, one per CTA, which walks the tensors its range
// touches.  Eighteen consumer warps take tiles from a shared counter (one block per lane);
// one more, producer, warp computes each row's sigma2 (binary64 sum of exact squares)
// just ahead of them, which also brings the rows into L2 before the consumers load their
// blocks.  A tile may span rows; every lane finds its own row.  Rows of any width are
// balanced to a tile per CTA, so short rows (64 blocks) and rows that are not a multiple
// of 32 blocks (344) leave no lanes idle.  Every wait is bounded.  A variant of the kernel
// (EPI) also writes each block's dequantized values and accumulates its round trip.
#include <cuda_fp16.h>

#include "common.cuh"

namespace iqq {

namespace {

constexpr int QK = IQQ_Q4_0_BLOCK_VALUES;
constexpr int kNmax = 8;
constexpr int kCand = 19;
#ifndef IQQ_Q4_CONSUMERS
#define IQQ_Q4_CONSUMERS 18     // consumer warps per CTA: 18 fill an SM's shared memory (one CTA per SM)
#endif
constexpr int kConsumers = IQQ_Q4_CONSUMERS;
constexpr int kThreads = (kConsumers + 1) * 32; // plus one producer warp
constexpr int kRowS = QK + 4;                   // code row stride: 16-byte rows, LDS.128 conflict-free
constexpr int kMaxRows = 256;                   // sigma2 rows per chunk of a CTA's range
constexpr int kLeadRows = 4;                    // rows the producer may run ahead of the consumers
constexpr float kMagic = 12582912.0f;           // 1.5 * 2^23
constexpr unsigned kFull = 0xffffffffu;
constexpr float kEta = 0.0009765625f;           // 2^-10: estimate closer than this to a candidate -> exact
constexpr long long kWaitCycles = 4000000000LL; // about 2 s at 2 GHz

// Unroll factors of the per-block loops over 4-value groups (larger: more latency hidden per
// warp, more code for the instruction cache); values measured on the layer set.
#ifndef IQQ_Q4_T_UNROLL
#define IQQ_Q4_T_UNROLL 1       // transitions
#endif
#ifndef IQQ_Q4_X_UNROLL
#define IQQ_Q4_X_UNROLL 1       // exact sums of a candidate
#endif
#ifndef IQQ_Q4_S_UNROLL
#define IQQ_Q4_S_UNROLL 1       // weights, codes, greedy screen, final sums
#endif
#ifndef IQQ_Q4_PDL
#define IQQ_Q4_PDL 1            // programmatic dependent launch between consecutive launches
#endif
#define IQQ_PRAGMA(x) _Pragma(#x)
#define IQQ_UNROLL(n) IQQ_PRAGMA(unroll n)

// Per consumer warp: x and w of its 32 blocks, chunk-interleaved (the 16-byte chunk c of lane
// L's block at float 128c + 4L, so that the lanes of a quarter warp loading the same chunk of
// their blocks hit distinct banks, without padding), and an area used in turn by the
// per-candidate difference sums (float2 [18][32]), the survivors' exact scores (float2 [32])
// and the codes (float [32][36], padded rows).  18 warps fill an SM's shared memory:
// 18 x 12.5 KB.
struct WarpSmem {
    float x[32 * QK];
    float w[32 * QK];
    union {
        float2 diff[18 * 32];
        float2 res[32];  // (score, k) of an exact check
        float l[32 * kRowS];
    } u;
};
constexpr size_t kDynSmem = sizeof(WarpSmem) * kConsumers;

// Offset of value j of a block in the chunk-interleaved x and w areas, from the block's base
// (area + 4 * lane).
__device__ __forceinline__ int xoff(int j) { return ((j & ~3) << 5) | (j & 3); }

__device__ __forceinline__ float rcp_approx(float v)
{
    float r;
    asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}

__device__ __forceinline__ float clamp8(float r) { return fminf(fmaxf(r, -8.0f), 7.0f); }

// Bounded wait until *p >= target; returns false on expiry.
__device__ __forceinline__ bool wait_at_least(const volatile int* p, int target)
{
    if (*p >= target) return true;
    const long long t0 = clock64();
    unsigned ns = 32;
    while (*p < target) {
        if (clock64() - t0 > kWaitCycles) return false;
        __nanosleep(ns);
        if (ns < 1024) ns <<= 1;
    }
    return true;
}

// The exact sequential sums of the candidate iscale = a over a staged block, and its score.
__device__ __forceinline__ float exact_score(const float* __restrict__ xr, const float* __restrict__ wr, float a)
{
    float s = 0.0f, t = 0.0f;
    IQQ_UNROLL(IQQ_Q4_X_UNROLL)
    for (int j4 = 0; j4 < QK; j4 += 4) {
        const float4 xv4 = *reinterpret_cast<const float4*>(xr + 32 * j4);
        const float4 wv4 = *reinterpret_cast<const float4*>(wr + 32 * j4);
        const float xq[4] = {xv4.x, xv4.y, xv4.z, xv4.w};
        const float wq[4] = {wv4.x, wv4.y, wv4.z, wv4.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float l = clamp8(rintf(__fmul_rn(a, xq[k])));
            s = __fmaf_rn(__fmul_rn(wq[k], xq[k]), l, s);
            t = __fmaf_rn(wq[k], __fmul_rn(l, l), t);
        }
    }
    return t > 0.0f ? __fdiv_rn(__fmul_rn(s, s), t) : -INFINITY;
}

// The greedy passes of the warp's blocks that accepted a move in their first pass (bit set in
// `pending`), from the element after that move on, one block at a time, lane j holding
// element j.  All trial moves of a pass that precede the next accepted move see the same
// (sumlx, suml2, score), so they are evaluated together; the lowest accepting lane is the move
// the sequential pass accepts first.  The state then advances and the scan resumes after that
// element: the accepted moves and every rounding are those of the sequential passes.  Every
// lane's trial is evaluated each time: when the rest of a pass accepts nothing, the next
// pass starts from element 0 in the same state, so the same ballot gives its first move.
__device__ __forceinline__ void greedy_rest(const float* sX, const float* sW, float* sL, unsigned pending,
                                            float sumlx, float suml2, float score, int gstart)
{
    const int lane = threadIdx.x & 31;
    while (pending != 0u) {
        const int bb = __ffs(pending) - 1;
        pending &= pending - 1u;
        float lx = __shfl_sync(kFull, sumlx, bb);
        float l2 = __shfl_sync(kFull, suml2, bb);
        float sc = __shfl_sync(kFull, score, bb);
        int start = __shfl_sync(kFull, gstart, bb);
        const float xj = sX[4 * bb + xoff(lane)];
        const float wj = sW[4 * bb + xoff(lane)];
        float lj = sL[bb * kRowS + lane];
        const float wxj = __fmul_rn(wj, xj);
        float d = __fdiv_rn(lx, l2);
        int passes = 1;
        bool changed = true;  // pass 1 accepted the move before `start`
        for (int guard = 0; guard < 5 * (QK + 1); ++guard) {  // at most 5 passes of <= 32 moves
            const float g = __fmul_rn(d, __fmul_rn(wj, __fsub_rn(xj, __fmul_rn(d, lj))));
            const float sg = g > 0.0f ? 1.0f : -1.0f;
            const float ln = __fadd_rn(lj, sg);
            const float nlx = __fadd_rn(lx, __fmul_rn(sg, wxj));
            // 2*sg*lj + 1 is a small integer: exact in one fma, as in the definition's three steps
            const float nl2 = __fmaf_rn(wj, __fmaf_rn(g > 0.0f ? 2.0f : -2.0f, lj, 1.0f), l2);
            const float a2 = __fmul_rn(nlx, nlx);
            // rejected for certain when fl(nlx^2) <= fl(fl(sc*nl2)*(1 - 2^-22)) with that bound in
            // [1e-30, 1e30]: then nlx^2/nl2 < sc exactly, and so is its rounded quotient
            const float thr = __fmul_rn(__fmul_rn(sc, nl2), 0.99999976158142089844f);
            bool ok = (g > 0.0f || g < 0.0f) && ln >= -8.0f && ln <= 7.0f && nl2 > 0.0f &&
                      !(a2 <= thr && thr >= 1e-30f && thr <= 1e30f);
            float ns = 0.0f;
            if (ok) {
                ns = __fdiv_rn(a2, nl2);
                ok = ns > sc;
            }
            const unsigned m = __ballot_sync(kFull, ok);
            unsigned mh = start < QK ? m & (kFull << start) : 0u;  // the rest of this pass
            if (mh == 0u) {                      // the rest of this pass accepts nothing
                if (!changed || passes == 5) break;
                ++passes;                        // the next pass, from element 0, same state
                changed = false;
                mh = m;
                if (mh == 0u) break;             // it accepts nothing either
            }
            const int j0 = __ffs(mh) - 1;
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
        sL[bb * kRowS + lane] = lj;
    }
}

// One warp: sigma2 of the row xr into *sig (lane 0 writes): the binary64 sum of exact squares
// over n_per_row; an Inf or NaN in x makes it non-finite (the square of any finite binary32
// value is finite in binary64) and raises the flag.
template <typename XT>
__device__ __forceinline__ void row_sigma2(const XT* __restrict__ xr, int64_t n_per_row, float* sig,
                                           uint32_t* __restrict__ flags)
{
    const int lane = threadIdx.x & 31;
    const int64_t n4 = n_per_row / 4;
    double acc = 0.0;
    int64_t i = lane;
    for (; i + 15 * 32 < n4; i += 16 * 32) {
        float4 v[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) v[u] = iqq::ld4(xr + 4 * (i + 32 * u));
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            acc = fma(static_cast<double>(v[u].x), static_cast<double>(v[u].x), acc);
            acc = fma(static_cast<double>(v[u].y), static_cast<double>(v[u].y), acc);
            acc = fma(static_cast<double>(v[u].z), static_cast<double>(v[u].z), acc);
            acc = fma(static_cast<double>(v[u].w), static_cast<double>(v[u].w), acc);
        }
    }
    for (; i < n4; i += 32) {
        const float4 v = iqq::ld4(xr + 4 * i);
        acc = fma(static_cast<double>(v.x), static_cast<double>(v.x), acc);
        acc = fma(static_cast<double>(v.y), static_cast<double>(v.y), acc);
        acc = fma(static_cast<double>(v.z), static_cast<double>(v.z), acc);
        acc = fma(static_cast<double>(v.w), static_cast<double>(v.w), acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
    if (lane == 0) {
        if (!isfinite(acc)) iqq::raise_flags(flags, IQQ_FLAG_NONFINITE_INPUT);
        *sig = static_cast<float>(acc / static_cast<double>(n_per_row));
    }
}

// The producer warp: sigma2 of rows rA+r0 .. rA+nr-1 in order, published through s_produced.
template <typename XT>
__device__ void produce_rows(const XT* __restrict__ x, int64_t n_per_row, int64_t rA, int r0, int nr, float* s_sig,
                             volatile int* s_produced, const volatile int* s_consumed_row,
                             uint32_t* __restrict__ flags)
{
    for (int rr = r0; rr < nr; ++rr) {
        // stay a few rows ahead of the furthest row a grabbed tile needs, so that the rows read
        // here are still in L2 when the consumers load their blocks (bounded: on expiry go on)
        if (rr > kLeadRows) {
            const long long t0 = clock64();
            while (*s_consumed_row + kLeadRows < rr && clock64() - t0 < kWaitCycles / 4) __nanosleep(256);
        }
        row_sigma2(x + (rA + rr) * n_per_row, n_per_row, &s_sig[rr], flags);
        if ((threadIdx.x & 31) == 0) {
            __threadfence_block();
            *s_produced = rr + 1;
        }
        __syncwarp();
    }
}

// Stages the block's 32 values of x into the lane's interleaved chunks: 16-byte asynchronous
// copies for binary32 storage (no registers held while they are in flight), widened loads for
// bf16.
__device__ __forceinline__ void stage_x(float* dst, const float* src)
{
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
#pragma unroll
    for (int i = 0; i < QK / 4; ++i)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d + 512 * i), "l"(src + 4 * i)
                     : "memory");
}
__device__ __forceinline__ void stage_x(float* dst, const __nv_bfloat16* src)
{
#pragma unroll
    for (int i = 0; i < QK / 4; ++i) *reinterpret_cast<float4*>(dst + 128 * i) = iqq::ld4(src + 4 * i);
}
__device__ __forceinline__ void stage_qw(float* dst, const float* src)
{
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
#pragma unroll
    for (int i = 0; i < QK / 4; ++i)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 16;" ::"r"(d + 512 * i), "l"(src + 4 * i)
                     : "memory");
}
__device__ __forceinline__ void staged_wait() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// The step of code n -> n+1 of a value of magnitude X whose index estimate t (+0.5) lies within
// 2^-10 of candidate ic = round(t - 0.5): it is at ic if the code there is already > n, else at
// ic + 1 (the neighbouring candidates are far from the rounding boundary).
__device__ __forceinline__ int exact_step(float t, float n, float X, float A, const float* s_c)
{
    const int ic = min(max(__float2int_rn(__fsub_rn(t, 0.5f)), 0), 19);
    if (ic <= 0) return 1;
    if (ic >= 18) return 18;
    const float v = rintf(__fmul_rn(__fdiv_rn(s_c[ic], A), X));
    return v >= __fadd_rn(n, 1.0f) ? ic : ic + 1;
}

// Adds a step n -> n+1 of a value (|w*x| = p, weight w) to the difference sums of candidate idx.
__device__ __forceinline__ void add_step(float2* dcol, int idx, float p, float w, float n)
{
    float2* c = dcol + 32 * (min(max(idx, 1), 18) - 1);
    float2 v = *c;
    v.x = __fadd_rn(v.x, p);
    v.y = __fmaf_rn(w, __fmaf_rn(2.0f, n, 1.0f), v.y);
    *c = v;
}

// The round trip of a lane's blocks (the epilogue variant): sum qw e^2, sum qw, sum e^2 in
// binary64 and max |e|.
struct RoundTrip {
    double ew = 0.0, eq = 0.0, ee = 0.0;
    float em = 0.0f;
};

// One tile: blocks g .. g+31 (those below gend) of the chunk whose rows start at rA.  EPI: the
// blocks' dequantized values go to y_out (when given) and their round trip to rt (when
// want_rt).
template <typename XT, bool EPI>
__device__ void consume_tile(const XT* __restrict__ x, const float* __restrict__ qw, uint8_t* __restrict__ out,
                             int64_t nrows, int64_t n_per_row, int64_t rows_per_qw, int weight_mode, float fudge,
                             int64_t g, int64_t gend, int64_t rA, int64_t nb, const float* s_sig,
                             const volatile int* s_produced, int* s_consumed_row, const float* s_c, WarpSmem& ws,
                             volatile int* s_abort, uint32_t* __restrict__ flags, float* __restrict__ y_out,
                             bool want_rt, RoundTrip& rt)
{
    const int lane = threadIdx.x & 31;
    uint32_t bad = 0u;

    // this lane's block: its row (relative to rA) and position in the row; 32-bit arithmetic
    // within the chunk (fewer than kMaxRows rows of nb < 2^22 blocks)
    const int64_t gb = g + lane;
    const bool valid = gb < gend;
    const uint32_t nb32 = static_cast<uint32_t>(nb);
    const uint32_t off = static_cast<uint32_t>((valid ? gb : g) - rA * nb);
    const uint32_t rr = off / nb32;
    const uint32_t b = off - rr * nb32;
    const int64_t row = rA + rr;

    // x and qw of the block into the lane's rows (asynchronous while the row's sigma2 is awaited)
    float* const my_x = ws.x + 4 * lane;
    float* const my_w = ws.w + 4 * lane;
    const int64_t qrow = rows_per_qw > 0 ? row / rows_per_qw : 0;
    const float* qb = qw != nullptr ? qw + qrow * n_per_row + static_cast<int64_t>(b) * QK : nullptr;
    if (valid) {
        stage_x(my_x, x + row * n_per_row + static_cast<int64_t>(b) * QK);
        if (qb != nullptr) stage_qw(my_w, qb);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");

    // the sigma2 of every row of the tile (every lane observes the producer's count)
    {
        const uint32_t last = static_cast<uint32_t>((gend < g + 32 ? gend : g + 32) - 1 - rA * nb) / nb32;
        if (lane == 0 && static_cast<int>(last) > *s_consumed_row) atomicMax(s_consumed_row, static_cast<int>(last));
        const bool ok = __all_sync(kFull, wait_at_least(s_produced, static_cast<int>(last) + 1));
        if (!ok) {
            staged_wait();
            if (lane == 0) {
                iqq::raise_flags(flags, IQQ_FLAG_WAIT_TIMEOUT);
                *s_abort = 1;
            }
            return;
        }
    }
    __threadfence_block();
    const float sigma2 = __fmul_rn(fudge, valid ? s_sig[rr] : 0.0f);
    staged_wait();

    // the imatrix checks on the first row of each imatrix group; importance weights in place of
    // qw (binary32, one rounding per operation): mode 0 qw*sqrt(sigma2 + x*x), 1 qw,
    // 2 qw*(x*x), 3 qw*|x|, 4 qw*(sigma2 + x*x), 5 qw*(sqrt(sigma2) + |x|); |xmax| and xmax
    // (the first element of largest |x|)
    float A = 0.0f, xmax = 0.0f;
    int jmax = 0;
    {
        if (!valid) {
#pragma unroll
            for (int i = 0; i < QK; i += 4) {
                *reinterpret_cast<float4*>(my_x + 32 * i) = make_float4(0.f, 0.f, 0.f, 0.f);
                *reinterpret_cast<float4*>(my_w + 32 * i) = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        } else if (qb == nullptr) {
#pragma unroll
            for (int i = 0; i < QK; i += 4)
                *reinterpret_cast<float4*>(my_w + 32 * i) = make_float4(1.f, 1.f, 1.f, 1.f);
        } else if (rows_per_qw > 0 ? row % rows_per_qw == 0 : row == 0) {
            float qmin = 0.0f, qnf = 0.0f;
#pragma unroll 2
            for (int i = 0; i < QK; i += 4) {
                const float4 q = *reinterpret_cast<const float4*>(my_w + 32 * i);
                qmin = fminf(fminf(qmin, fminf(q.x, q.y)), fminf(q.z, q.w));
                qnf = __fmaf_rn(q.x, 0.0f, __fmaf_rn(q.y, 0.0f, __fmaf_rn(q.z, 0.0f, __fmaf_rn(q.w, 0.0f, qnf))));
            }
            if (qnf != qnf) bad |= IQQ_FLAG_NONFINITE_INPUT;
            if (qmin < 0.0f) bad |= IQQ_FLAG_NEG_QW;
        }
        // |xmax| and xmax, the first element of largest |x|, and its index
        auto track = [&](const float (&xq)[4], int i) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float a = fabsf(xq[k]);
                if (a > A) { A = a; xmax = xq[k]; jmax = i + k; }
            }
        };
        if (weight_mode == 0) {  // the default weights: a loop of their own (compact code)
            IQQ_UNROLL(IQQ_Q4_S_UNROLL)
            for (int i = 0; i < QK; i += 4) {
                const float4 v = *reinterpret_cast<const float4*>(my_x + 32 * i);
                const float4 q = *reinterpret_cast<const float4*>(my_w + 32 * i);
                const float xq[4] = {v.x, v.y, v.z, v.w};
                const float wq[4] = {q.x, q.y, q.z, q.w};
                float wn[4];
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    wn[k] = __fmul_rn(wq[k], __fsqrt_rn(__fadd_rn(sigma2, __fmul_rn(xq[k], xq[k]))));
                track(xq, i);
                *reinterpret_cast<float4*>(my_w + 32 * i) = make_float4(wn[0], wn[1], wn[2], wn[3]);
            }
        } else {
            const float sigma = weight_mode == 5 ? __fsqrt_rn(sigma2) : 0.0f;
#pragma unroll 1
            for (int i = 0; i < QK; i += 4) {
                const float4 v = *reinterpret_cast<const float4*>(my_x + 32 * i);
                const float4 q = *reinterpret_cast<const float4*>(my_w + 32 * i);
                const float xq[4] = {v.x, v.y, v.z, v.w};
                float wq[4] = {q.x, q.y, q.z, q.w};
                if (weight_mode != 1) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float xj = xq[k];
                        const float t = __fmul_rn(xj, xj);
                        float m;
                        switch (weight_mode) {
                        case 2: m = t; break;
                        case 3: m = fabsf(xj); break;
                        case 4: m = __fadd_rn(sigma2, t); break;
                        default: m = __fadd_rn(sigma, fabsf(xj)); break;
                        }
                        wq[k] = __fmul_rn(wq[k], m);
                    }
                }
                track(xq, i);
                *reinterpret_cast<float4*>(my_w + 32 * i) = make_float4(wq[0], wq[1], wq[2], wq[3]);
            }
        }
    }

    // ---------------------------------------------------------------- transitions
    // With iscale_k = -c_k/xmax the codes are l = clamp(rint(iscale_k*x), -8, 7), and
    // |l| = min(rint(fl(c_k/|xmax|)*|x|), 8 or 7): every term w*x*l of sumlx has the sign
    // of -xmax, so the sums of a candidate are sums of nonnegative magnitudes.
    const bool active = A > 0.0f;
    float2* const dcol = ws.u.diff + lane;  // diff[i-1][lane] for candidate i = 1..18
#pragma unroll
    for (int i = 0; i < 18; ++i) dcol[32 * i] = make_float2(0.0f, 0.0f);
    const float a0 = active ? __fdiv_rn(-s_c[0], xmax) : 0.0f;
    const float a18 = active ? __fdiv_rn(-s_c[kCand - 1], xmax) : 0.0f;
    const float kR = __fmul_rn(10.0f, A);  // 80*|xmax|/nmax: the step index scale
    // candidate 0's sums in four interleaved chains (value j in chain j mod 4): a term goes
    // through at most 8 + 2 roundings there, not 32
    float S0k[4] = {0.0f, 0.0f, 0.0f, 0.0f}, T0k[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    float nsteps = 0.0f;
    uint32_t m_unc = 0u, m_two = 0u;
    IQQ_UNROLL(IQQ_Q4_T_UNROLL)
    for (int j4 = 0; j4 < QK; j4 += 4) {
        const float4 xv4 = *reinterpret_cast<const float4*>(my_x + 32 * j4);
        const float4 wv4 = *reinterpret_cast<const float4*>(my_w + 32 * j4);
        const float xq[4] = {xv4.x, xv4.y, xv4.z, xv4.w};
        const float wq[4] = {wv4.x, wv4.y, wv4.z, wv4.w};
        uint32_t unc4 = 0u, two4 = 0u;  // this group's masks (constant shifts)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float xs = xq[k], w = wq[k];
            const float p = fabsf(__fmul_rn(w, xs));
            const float l0 = rintf(__fmul_rn(a0, xs));            // |l0| <= 7: no clamp needed
            const float l18 = clamp8(rintf(__fmul_rn(a18, xs)));
            const float m0 = fabsf(l0);
            S0k[k] = __fmaf_rn(p, m0, S0k[k]);
            T0k[k] = __fmaf_rn(w, __fmul_rn(m0, m0), T0k[k]);
            const float dm = __fsub_rn(fabsf(l18), m0);          // 0, 1 or 2 steps
            nsteps = __fadd_rn(nsteps, dm);
            // t + 0.5, t = (m0 + 0.5)*R - 71: the (real) candidate index of the first step; the
            // step goes to round(t + 0.5) unless t lies within 2^-10 of a candidate (then exact).
            // Computed for every value (no branch); values without a step add zeros.
            const float R = __fmul_rn(kR, rcp_approx(fabsf(xs)));
            const float t = __fmaf_rn(m0, R, __fmaf_rn(0.5f, R, -70.5f));
            const float y = __fadd_rn(t, kMagic);
            const float dist = __fsub_rn(t, __fsub_rn(y, kMagic));
            // candidate index - 1, clamped to [0, 17] (memory safety for any input)
            const uint32_t i1 = min(__float_as_uint(y) - (__float_as_uint(kMagic) + 1u), 17u);
            const bool step = dm > 0.5f;
            const bool sure = step && fabsf(dist) < 0.5f - kEta;
            float2* c = dcol + 32 * i1;
            float2 v = *c;
            v.x = __fadd_rn(v.x, p);
            v.y = __fmaf_rn(w, __fmaf_rn(2.0f, m0, 1.0f), v.y);
            if (sure) *c = v;
            unc4 |= static_cast<uint32_t>(step && !sure) << k;
            two4 |= static_cast<uint32_t>(dm > 1.5f) << k;
        }
        m_unc |= unc4 << j4;
        m_two |= two4 << j4;
    }
    const float S0 = __fadd_rn(__fadd_rn(S0k[0], S0k[1]), __fadd_rn(S0k[2], S0k[3]));
    const float T0 = __fadd_rn(__fadd_rn(T0k[0], T0k[1]), __fadd_rn(T0k[2], T0k[3]));
    // The first largest element (|x| = |xmax|) always has one step, 7 -> 8, and it lies on a
    // rounding tie: at candidate 4 (c = 7.5) when fl(fl(7.5/|xmax|)*|xmax|) >= 7.5 (rint
    // rounds 7.5 to 8), else at candidate 5.  It is placed here, per block, rather than
    // among the uncertain steps below.
    if (active && ((m_unc >> jmax) & 1u)) {
        const float v4 = __fmul_rn(__fdiv_rn(s_c[4], A), A);
        const float w = my_w[xoff(jmax)];
        float2* c = dcol + 32 * (v4 >= 7.5f ? 3 : 4);
        float2 v = *c;
        v.x = __fadd_rn(v.x, fabsf(__fmul_rn(w, xmax)));
        v.y = __fmaf_rn(w, 15.0f, v.y);
        *c = v;
        m_unc &= ~(1u << jmax);
    }
    // the other uncertain first steps and the second steps, per lane from the staged row, one
    // pass over the values that have either
    {
        uint32_t todo = m_unc | m_two;
        while (todo != 0u) {
            const int j = __ffs(todo) - 1;
            todo &= todo - 1u;
            const float xs = my_x[xoff(j)], w = my_w[xoff(j)];
            const float X = fabsf(xs);
            const float p = fabsf(__fmul_rn(w, xs));
            const float m0 = fabsf(rintf(__fmul_rn(a0, xs)));
            const float R = __fmul_rn(kR, rcp_approx(X));
            const float t = __fmaf_rn(m0, R, __fmaf_rn(0.5f, R, -70.5f));  // as in the loop above
            if ((m_unc >> j) & 1u) add_step(dcol, exact_step(t, m0, X, A, s_c), p, w, m0);
            if ((m_two >> j) & 1u) {
                const float t2 = __fadd_rn(t, R);  // the second step
                const float n = __fadd_rn(m0, 1.0f);
                const float y = __fadd_rn(t2, kMagic);
                const float dist = __fsub_rn(t2, __fsub_rn(y, kMagic));
                int idx = static_cast<int>(__float_as_uint(y) - __float_as_uint(kMagic));
                if (!(fabsf(dist) < 0.5f - kEta && idx >= 1 && idx <= 18)) idx = exact_step(t2, n, X, A, s_c);
                add_step(dcol, idx, p, w, n);
            }
        }
    }

    // ---------------------------------------------------------------- approximate scores
    // Prefix sums of the differences; candidate i's approximate score replaces its (consumed)
    // difference sums.  A candidate with no step has its predecessor's sums: dominated (it
    // cannot win the tie).
    uint32_t dom = 0u;
    float S = S0, T = T0;
    float mx = __fmul_rn(__fmul_rn(S, S), rcp_approx(T));
    const float sc0 = mx;
#pragma unroll 2
    for (int i = 1; i < kCand; ++i) {
        float2* c = dcol + 32 * (i - 1);
        const float2 v = *c;
        if (v.x == 0.0f && v.y == 0.0f) dom |= 1u << i;
        S = __fadd_rn(S, v.x);
        T = __fadd_rn(T, v.y);
        const float sci = __fmul_rn(__fmul_rn(S, S), rcp_approx(T));
        c->x = sci;
        mx = fmaxf(mx, sci);
    }
    // Bounds (u = 2^-24, sums of non-negative terms, first order): a term of candidate k's
    // approximate sums goes through at most max(10, steps) + 1 + k roundings (candidate 0's
    // chains 1 + 8 + 2, a difference sum's steps + 1, then k prefix additions), so its score
    // S^2/T is within 3 (max(10, steps) + 1 + k) + 6 u of the real one (6 u: the approximate
    // quotient); an exact score is within 2*33 + 32 + 2 = 100 u (its sequential chains and two
    // roundings).  Candidate i cannot be the exact winner when its approximate score lies
    // below the best approximate score (candidate m) by more than the sum of i's and m's
    // bounds plus twice the exact one: 6 max(10, steps) + 3 i + 3 m + 6 + 12 + 200 u, with
    // m <= 18 and 20 u of slack for the roundings of the threshold itself.
    const bool regular = active && A >= 0x1p-100f && A <= 0x1p100f && S0 >= 0x1p-50f && T0 >= 0x1p-50f &&
                         S <= 0x1p50f && T <= 0x1p50f && mx >= 0x1p-100f && mx <= 0x1p100f;
    uint32_t surv = 0u;
    {
        // threshold of candidate i: mx (1 - (6 max(10, steps) + 3 i + 292) u)
        const float mu = __fmul_rn(mx, 0x1p-24f);
        const float thr0 = __fsub_rn(mx, __fmul_rn(mu, __fmaf_rn(6.0f, fmaxf(nsteps, 10.0f), 292.0f)));
        const float d3 = __fmul_rn(mu, 3.0f);
        if (sc0 >= thr0) surv = 1u;
#pragma unroll
        for (int i = 1; i < kCand; ++i)
            if (dcol[32 * (i - 1)].x >= __fmaf_rn(-d3, static_cast<float>(i), thr0)) surv |= 1u << i;
        surv &= ~dom;
    }
    // blocks outside the bounds: every candidate gets its exact sums (the direct sweep)
    if (!regular) surv = active ? (1u << kCand) - 1u : 0u;
    __syncwarp();  // the difference sums are read: the area now holds the survivors' scores

    // ---------------------------------------------------------------- exact winner
    int kbest = surv != 0u ? __ffs(surv) - 1 : 0;
    float best = -INFINITY;
    {
        const int cnt = __popc(surv);
        const int need = cnt >= 2 ? cnt : 0;
        // exclusive prefix of need over the warp
        int start = need;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(kFull, start, o);
            if (lane >= o) start += v;
        }
        const int total = __shfl_sync(kFull, start, 31);
        start -= need;
        for (int base = 0; base < total; base += 32) {  // warp-uniform
            const int q = base + lane;
            // owner: the last lane whose range starts at or before q
            int lo = 0;
#pragma unroll
            for (int step = 16; step > 0; step >>= 1) {
                const int s = __shfl_sync(kFull, start, lo + step);
                if (s <= q) lo += step;
            }
            const int owner = lo;
            const int ostart = __shfl_sync(kFull, start, owner);
            const uint32_t osurv = __shfl_sync(kFull, surv, owner);
            const float oxmax = __shfl_sync(kFull, xmax, owner);
            float r = -INFINITY;
            int kk = 0;
            if (q < total) {
                // the (q - ostart)-th survivor of the owner: drop that many lowest set bits
                unsigned m = osurv;
                for (int i = q - ostart; i > 0 && m != 0u; --i) m &= m - 1u;
                kk = m != 0u ? min(__ffs(m) - 1, kCand - 1) : kCand - 1;
                r = exact_score(ws.x + 4 * owner, ws.w + 4 * owner, __fdiv_rn(-s_c[kk], oxmax));
            }
            ws.u.res[lane] = make_float2(r, __int_as_float(kk));
            __syncwarp();
            if (need > 0) {
                // this lane's items of the round, in increasing k: strictly better wins
                const int q0 = max(start, base), q1 = min(start + need, base + 32);
                for (int qq = q0; qq < q1; ++qq) {
                    const float2 e = ws.u.res[qq - base];
                    if (e.x > best) {
                        best = e.x;
                        kbest = __float_as_int(e.y);
                    }
                }
            }
            __syncwarp();
        }
    }
    __syncwarp();  // the area now holds the codes

    // ---------------------------------------------------------------- codes and greedy state
    // mode 0: nothing to search (all-zero block or no block), 1: no candidate with positive
    // weighted code energy (codes of iscale = -nmax/xmax, d = 1/iscale), 2: search
    int mode = 0;
    float* const my_l = ws.u.l + lane * kRowS;
    float sumlx = 0.0f, suml2 = 0.0f, score = 0.0f, dfb = 0.0f;
    {
        float a = 0.0f;
        if (active) {
            if (!regular && best == -INFINITY) {
                a = __fdiv_rn(static_cast<float>(-kNmax), xmax);
                dfb = __fdiv_rn(1.0f, a);
                mode = 1;
            } else {
                a = __fdiv_rn(-s_c[kbest], xmax);
                mode = 2;
            }
        }
        IQQ_UNROLL(IQQ_Q4_S_UNROLL)
        for (int j4 = 0; j4 < QK; j4 += 4) {
            const float4 xv4 = *reinterpret_cast<const float4*>(my_x + 32 * j4);
            const float4 wv4 = *reinterpret_cast<const float4*>(my_w + 32 * j4);
            const float xq[4] = {xv4.x, xv4.y, xv4.z, xv4.w};
            const float wq[4] = {wv4.x, wv4.y, wv4.z, wv4.w};
            float lq[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                lq[k] = clamp8(rintf(__fmul_rn(a, xq[k])));
                sumlx = __fmaf_rn(__fmul_rn(wq[k], xq[k]), lq[k], sumlx);
                suml2 = __fmaf_rn(wq[k], __fmul_rn(lq[k], lq[k]), suml2);
            }
            *reinterpret_cast<float4*>(my_l + j4) = make_float4(lq[0], lq[1], lq[2], lq[3]);
        }
        if (mode == 2) score = __fdiv_rn(__fmul_rn(sumlx, sumlx), suml2);
    }

    // greedy pass 1, this lane's block.  Until the first accepted move the state (sumlx =
    // S, suml2 = T, score, d) is that of the sweep, so every element's trial can be screened
    // against it at once.  With r = x/d - l and eps = w (x/d)^2 / T (d = S/T), the trial at
    // an element raises the score (in real arithmetic) by (w/T')(2|r| - 1 + eps) relative,
    // and the binary32 comparison cannot accept it unless that exceeds -7u (u = 2^-24):
    // so it is rejected for certain when w (1 - 2|r| - eps) >= 7u (T + 17 w).  Evaluated
    // with r, eps from q = fl(x * D), D = T/S and 1/T to within 3u (approximate reciprocals;
    // error below 100u in 1 - 2|r| - eps while |q| < 8.5) as
    // fl(w * fl(fl(1 - 2^-15 - 2|r|) - eps)) >= 2^-20 T.  The elements not excluded are tried
    // exactly, in order; at the first accepted move the block is handed to the
    // warp-cooperative passes, which continue from the next element.
    bool changed = false;
    int gstart = 0;
    if (mode == 2) {
        const float invT = rcp_approx(suml2);
        const float D = __fmul_rn(suml2, rcp_approx(sumlx));
        const float thr = __fmul_rn(suml2, 0x1p-20f);
        uint32_t maybe = 0u;
        IQQ_UNROLL(IQQ_Q4_S_UNROLL)
        for (int j4 = 0; j4 < QK; j4 += 4) {
            const float4 xv4 = *reinterpret_cast<const float4*>(my_x + 32 * j4);
            const float4 wv4 = *reinterpret_cast<const float4*>(my_w + 32 * j4);
            const float4 lv4 = *reinterpret_cast<const float4*>(my_l + j4);
            const float xq[4] = {xv4.x, xv4.y, xv4.z, xv4.w};
            const float wq[4] = {wv4.x, wv4.y, wv4.z, wv4.w};
            const float lq[4] = {lv4.x, lv4.y, lv4.z, lv4.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float q = __fmul_rn(xq[k], D);
                const float r = __fsub_rn(q, lq[k]);
                const float eps = __fmul_rn(__fmul_rn(wq[k], __fmul_rn(q, q)), invT);
                const float b = __fsub_rn(__fmaf_rn(-2.0f, fabsf(r), 1.0f - 0x1p-15f), eps);
                const bool sure_reject = __fmul_rn(wq[k], b) >= thr;
                maybe |= static_cast<uint32_t>(!sure_reject) << (j4 + k);
            }
        }
        float d = __fdiv_rn(sumlx, suml2);
        while (maybe != 0u) {
            const int j = __ffs(maybe) - 1;
            maybe &= maybe - 1u;
            const float xj = my_x[xoff(j)], wj = my_w[xoff(j)], lj = my_l[j];
            const float g = __fmul_rn(d, __fmul_rn(wj, __fsub_rn(xj, __fmul_rn(d, lj))));
            const float sg = g > 0.0f ? 1.0f : -1.0f;
            const float ln = __fadd_rn(lj, sg);
            if (!(g > 0.0f || g < 0.0f) || ln < -8.0f || ln > 7.0f) continue;
            const float nlx = __fadd_rn(sumlx, __fmul_rn(sg, __fmul_rn(wj, xj)));
            const float nl2 = __fmaf_rn(wj, __fmaf_rn(g > 0.0f ? 2.0f : -2.0f, lj, 1.0f), suml2);
            if (!(nl2 > 0.0f)) continue;
            const float ns = __fdiv_rn(__fmul_rn(nlx, nlx), nl2);
            if (ns > score) {
                my_l[j] = ln;
                sumlx = nlx;
                suml2 = nl2;
                score = ns;
                changed = true;
                gstart = j + 1;
                break;
            }
        }
    }
    const unsigned pending = __ballot_sync(kFull, changed);
    if (pending != 0u) {
        __syncwarp();
        greedy_rest(ws.x, ws.w, ws.u.l, pending, sumlx, suml2, score, gstart);
    }
    __syncwarp();

    // ---------------------------------------------------------------- final scale and block
    uint16_t d16 = 0;
    {
        float d = dfb;
        if (mode == 2) {
            float sfx = 0.0f, sf2 = 0.0f;
            IQQ_UNROLL(IQQ_Q4_S_UNROLL)
            for (int j4 = 0; j4 < QK; j4 += 4) {
                const float4 xv4 = *reinterpret_cast<const float4*>(my_x + 32 * j4);
                const float4 wv4 = *reinterpret_cast<const float4*>(my_w + 32 * j4);
                const float4 lv4 = *reinterpret_cast<const float4*>(my_l + j4);
                const float xq[4] = {xv4.x, xv4.y, xv4.z, xv4.w};
                const float wq[4] = {wv4.x, wv4.y, wv4.z, wv4.w};
                const float lq[4] = {lv4.x, lv4.y, lv4.z, lv4.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    sfx = __fmaf_rn(__fmul_rn(wq[k], xq[k]), lq[k], sfx);
                    sf2 = __fmaf_rn(wq[k], __fmul_rn(lq[k], lq[k]), sf2);
                }
            }
            d = __fdiv_rn(sfx, sf2);
        }
        if (mode != 0) {
            d16 = __half_as_ushort(__float2half_rn(d));
            if ((d16 & 0x7fffu) == 0x7c00u && isfinite(d)) bad |= IQQ_FLAG_SCALE_OVERFLOW;
        }
    }
    if constexpr (EPI) {
        // the round trip weighs by qw: stage the block's qw again, over its weights (the final
        // sums were their last use), while the block is packed
        if (want_rt && valid && qb != nullptr) {
            stage_qw(my_w, qb);
            asm volatile("cp.async.commit_group;" ::: "memory");
        }
    }
    if (valid) {
        uint16_t* o16 = reinterpret_cast<uint16_t*>(out + (row * nb + b) * IQQ_Q4_0_BLOCK_BYTES);
        o16[0] = d16;
        // biased code n = l + 8: the low byte of (l + 8 + 1.5*2^23)
#pragma unroll 2
        for (int i = 0; i < QK / 4; ++i) {
            const uint32_t n0 = __float_as_uint(__fadd_rn(my_l[2 * i], kMagic + 8.0f)) & 15u;
            const uint32_t n1 = __float_as_uint(__fadd_rn(my_l[2 * i + 1], kMagic + 8.0f)) & 15u;
            const uint32_t n2 = __float_as_uint(__fadd_rn(my_l[2 * i + 16], kMagic + 8.0f)) & 15u;
            const uint32_t n3 = __float_as_uint(__fadd_rn(my_l[2 * i + 17], kMagic + 8.0f)) & 15u;
            o16[1 + i] = static_cast<uint16_t>(n0 | (n2 << 4) | (n1 << 8) | (n3 << 12));
        }
        if constexpr (EPI) {
            // y = fp16(d) * l (the bits of the dequantization) and the round trip e = x - y in
            // binary32, accumulated as the weighted-RMSE reduction does (qw restaged above)
            const float dq = __half2float(__ushort_as_half(d16));
            float4* yb = y_out != nullptr
                             ? reinterpret_cast<float4*>(y_out + row * n_per_row + static_cast<int64_t>(b) * QK)
                             : nullptr;
            if (want_rt) staged_wait();
#pragma unroll 1
            for (int j4 = 0; j4 < QK; j4 += 4) {
                const float4 lv4 = *reinterpret_cast<const float4*>(my_l + j4);
                const float yk[4] = {__fmul_rn(dq, lv4.x), __fmul_rn(dq, lv4.y), __fmul_rn(dq, lv4.z),
                                     __fmul_rn(dq, lv4.w)};
                if (yb != nullptr) __stcs(yb + j4 / 4, make_float4(yk[0], yk[1], yk[2], yk[3]));
                if (want_rt) {
                    const float4 xv4 = *reinterpret_cast<const float4*>(my_x + 32 * j4);
                    const float xq[4] = {xv4.x, xv4.y, xv4.z, xv4.w};
                    const float4 qv = qb != nullptr ? *reinterpret_cast<const float4*>(my_w + 32 * j4)
                                                    : make_float4(1.0f, 1.0f, 1.0f, 1.0f);
                    const float qk[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float e = __fsub_rn(xq[k], yk[k]);
                        const double ed = static_cast<double>(e);
                        const double e2 = ed * ed;  // exact
                        rt.ew = fma(static_cast<double>(qk[k]), e2, rt.ew);
                        rt.eq += static_cast<double>(qk[k]);
                        rt.ee += e2;
                        rt.em = fmaxf(rt.em, fabsf(e));
                    }
                }
            }
        }
    }
    iqq::raise_flags(flags, bad);
    __syncwarp();  // the warp's shared memory is rewritten by the next tile
}

// One tensor of a launch, and a launch: up to kMaxBatch tensors whose 32-block tiles are laid
// end to end (a tile never spans two tensors).
template <typename XT>
struct Prob {
    const XT* x;
    const float* qw;
    uint8_t* out;
    int64_t nrows, n_per_row, rows_per_qw;
};
constexpr int kMaxBatch = 64;
template <typename XT>
struct Batch {
    Prob<XT> p[kMaxBatch];
    int64_t cum[kMaxBatch + 1];  // tiles before tensor i
    int count;
};
static_assert(sizeof(Batch<float>) + 64 <= 4096, "kernel parameters");

// EPI: also the dequantized values (y_out, optional; launches of one tensor) and the
// round-trip accumulator (acc, optional): per lane across its tiles, then one set of atomics
// per CTA.
template <typename XT, bool EPI>
__global__ void __maxnreg__(96)  // one CTA of 608 threads per SM (at most 5 warps of an SMSP's 16K registers)
q4_0_w_kernel(const __grid_constant__ Batch<XT> B, int weight_mode, float fudge, uint32_t* __restrict__ flags,
              float* __restrict__ y_out, double* __restrict__ acc)
{
    extern __shared__ float4 smem4[];
    WarpSmem* const wsm = reinterpret_cast<WarpSmem*>(smem4);
    __shared__ float s_sig[kMaxRows];
    __shared__ float s_c[kCand];
    __shared__ int s_produced, s_next, s_consumed_row, s_abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t tiles = B.cum[B.count];
    // this CTA's tiles: an equal share (+-1) of the launch's
    const int64_t per = tiles / gridDim.x, extra = tiles % gridDim.x;
    const int64_t t0 = blockIdx.x * per + min(static_cast<int64_t>(blockIdx.x), extra);
    const int64_t t1 = t0 + per + (static_cast<int64_t>(blockIdx.x) < extra ? 1 : 0);
    if (threadIdx.x < kCand) s_c[threadIdx.x] = __fdiv_rn(static_cast<float>(kNmax * (71 + threadIdx.x)), 80.0f);
    if (threadIdx.x == 0) s_abort = 0;
    // Programmatic dependent launch: the next kernel of the stream may be scheduled now (its
    // CTAs start as this grid's retire); this grid waits for the previous kernel's completion
    // and memory before its first global access.  (No-ops without the launch attribute.)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    RoundTrip rt;
    int pi = 0;
    while (pi + 1 < B.count && B.cum[pi + 1] <= t0) ++pi;
    for (; pi < B.count && B.cum[pi] < t1; ++pi) {
        // the tensor's blocks [g, gend) in this CTA's share
        const XT* const x = B.p[pi].x;
        const float* const qw = B.p[pi].qw;
        uint8_t* const out = B.p[pi].out;
        const int64_t nrows = B.p[pi].nrows, n_per_row = B.p[pi].n_per_row, rows_per_qw = B.p[pi].rows_per_qw;
        const int64_t nb = n_per_row / QK;
        const int64_t total = nrows * nb;
        int64_t g = (max(t0, B.cum[pi]) - B.cum[pi]) * 32;
        const int64_t gl = (min(t1, B.cum[pi + 1]) - B.cum[pi]) * 32;
        const int64_t gend = gl < total ? gl : total;
        while (g < gend) {
            // a chunk of whole tiles touching at most kMaxRows rows
            const int64_t rA = g / nb;
            int64_t gB = (rA + kMaxRows) * nb / 32 * 32;
            if (gB > gend) gB = gend;
            const int nr = static_cast<int>((gB - 1) / nb - rA + 1);
            // the rows of the first tiles the warps take, one row per warp, side by side; the
            // producer continues after them
            const int64_t need = (g - rA * nb + static_cast<int64_t>(kConsumers) * 32 + nb - 1) / nb;
            const int head =
                static_cast<int>(min(min(static_cast<int64_t>(nr), need), static_cast<int64_t>(kConsumers + 1)));
            __syncthreads();  // every warp is done with the previous chunk
            if (*reinterpret_cast<volatile int*>(&s_abort) != 0) break;  // uniform: a wait ran out
            if (warp < head) row_sigma2(x + (rA + warp) * n_per_row, n_per_row, &s_sig[warp], flags);
            if (threadIdx.x == 0) {
                s_produced = head;
                s_next = 0;
                s_consumed_row = 0;
            }
            __syncthreads();
            if (warp == kConsumers) {
                produce_rows<XT>(x, n_per_row, rA, head, nr, s_sig, &s_produced, &s_consumed_row, flags);
            } else {
                WarpSmem& ws = wsm[warp];
                while (true) {
                    int t = 0;
                    if (lane == 0) t = atomicAdd(&s_next, 1);
                    t = __shfl_sync(kFull, t, 0);
                    const int64_t gt = g + static_cast<int64_t>(t) * 32;
                    if (gt >= gB || *reinterpret_cast<volatile int*>(&s_abort) != 0) break;
                    consume_tile<XT, EPI>(x, qw, out, nrows, n_per_row, rows_per_qw, weight_mode, fudge, gt, gB, rA,
                                          nb, s_sig, &s_produced, &s_consumed_row, s_c, ws, &s_abort, flags, y_out,
                                          acc != nullptr, rt);
                }
            }
            g = gB;
        }
    }
    if constexpr (EPI) {
        if (acc != nullptr) {  // uniform: warp sums, then the CTA's, then one atomic per quantity
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                rt.ew += __shfl_xor_sync(kFull, rt.ew, o);
                rt.eq += __shfl_xor_sync(kFull, rt.eq, o);
                rt.ee += __shfl_xor_sync(kFull, rt.ee, o);
                rt.em = fmaxf(rt.em, __shfl_xor_sync(kFull, rt.em, o));
            }
            __syncthreads();  // every warp is done with its staging area
            double* s_red = reinterpret_cast<double*>(smem4);  // [kConsumers][4]
            if (lane == 0 && warp < kConsumers) {
                s_red[4 * warp + 0] = rt.ew;
                s_red[4 * warp + 1] = rt.eq;
                s_red[4 * warp + 2] = rt.ee;
                s_red[4 * warp + 3] = static_cast<double>(rt.em);
            }
            __syncthreads();
            if (threadIdx.x == 0) {
                double a = 0.0, bq = 0.0, c = 0.0, m = 0.0;
                for (int w = 0; w < kConsumers; ++w) {
                    a += s_red[4 * w + 0];
                    bq += s_red[4 * w + 1];
                    c += s_red[4 * w + 2];
                    m = fmax(m, s_red[4 * w + 3]);
                }
                atomicAdd(acc + 0, a);
                atomicAdd(acc + 1, bq);
                atomicAdd(acc + 2, c);
                // non-negative binary64 values order like their bit patterns
                atomicMax(reinterpret_cast<unsigned long long*>(acc + 3),
                          static_cast<unsigned long long>(__double_as_longlong(m)));
            }
        }
    }
}

template <typename XT, bool EPI>
iqq_status launch(const Batch<XT>& B, int weight_mode, float fudge, uint32_t* d_flags, void* stream, float* y_out,
                  double* acc)
{
    static thread_local int configured_device = -1;
    static thread_local int grid_cap = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return iqq::launch_status();
    if (configured_device != dev) {
        if (cudaFuncSetAttribute(q4_0_w_kernel<XT, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kDynSmem)) != cudaSuccess ||
            cudaFuncSetAttribute(q4_0_w_kernel<XT, EPI>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared) != cudaSuccess)
            return iqq::launch_status();
        int sms = 0, per_sm = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return iqq::launch_status();
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, q4_0_w_kernel<XT, EPI>, kThreads, kDynSmem) !=
            cudaSuccess)
            return iqq::launch_status();
        grid_cap = sms * (per_sm > 0 ? per_sm : 1);
        configured_device = dev;
    }
    const int64_t tiles = B.cum[B.count];
    if (tiles == 0) return IQQ_OK;
    const int grid = static_cast<int>(tiles < grid_cap ? tiles : grid_cap);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kDynSmem;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = IQQ_Q4_PDL;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, q4_0_w_kernel<XT, EPI>, B, weight_mode, fudge, d_flags, y_out, acc) != cudaSuccess)
        return iqq::launch_status();
    return iqq::launch_status();
}

// A launch of one tensor.
template <typename XT, bool EPI>
iqq_status launch_one(const XT* x, const float* qw, void* out, int64_t nrows, int64_t n_per_row, int64_t rows_per_qw,
                      int weight_mode, float fudge, uint32_t* d_flags, void* stream, float* y_out, double* acc)
{
    Batch<XT> B;
    B.count = 1;
    B.p[0] = Prob<XT>{x, qw, static_cast<uint8_t*>(out), nrows, n_per_row, rows_per_qw};
    B.cum[0] = 0;
    B.cum[1] = (nrows * (n_per_row / QK) + 31) / 32;
    return launch<XT, EPI>(B, weight_mode, fudge, d_flags, stream, y_out, acc);
}

}  // namespace

// Whether the kernel above serves a tensor of this width: rows of fewer than 2^22 blocks (the
// chunk arithmetic is 32-bit).
bool q4_0_w_fits(int64_t n_per_row) { return n_per_row / QK < (int64_t(1) << 22); }

iqq_status launch_q4_0_w(const float* x, const float* qw, void* out, int64_t nrows, int64_t n_per_row,
                         int64_t rows_per_qw, int weight_mode, float fudge, uint32_t* d_flags, void* stream,
                         float* y_out, double* acc)
{
    if (y_out != nullptr || acc != nullptr)
        return launch_one<float, true>(x, qw, out, nrows, n_per_row, rows_per_qw, weight_mode, fudge, d_flags, stream,
                                       y_out, acc);
    return launch_one<float, false>(x, qw, out, nrows, n_per_row, rows_per_qw, weight_mode, fudge, d_flags, stream,
                                    nullptr, nullptr);
}

iqq_status launch_q4_0_w(const __nv_bfloat16* x, const float* qw, void* out, int64_t nrows, int64_t n_per_row,
                         int64_t rows_per_qw, int weight_mode, float fudge, uint32_t* d_flags, void* stream)
{
    return launch_one<__nv_bfloat16, false>(x, qw, out, nrows, n_per_row, rows_per_qw, weight_mode, fudge, d_flags,
                                            stream, nullptr, nullptr);
}

// Several binary32 tensors (validated by the caller), kMaxBatch per launch.
iqq_status launch_q4_0_w_batch(const iqq_q4_0_problem* probs, int64_t count, int weight_mode, float fudge,
                               uint32_t* d_flags, void* stream)
{
    Batch<float> B;
    B.count = 0;
    B.cum[0] = 0;
    for (int64_t i = 0; i < count; ++i) {
        const iqq_q4_0_problem& q = probs[i];
        const int64_t tiles = (q.nrows * (q.n_per_row / QK) + 31) / 32;
        if (tiles == 0) continue;
        B.p[B.count] = Prob<float>{q.x, q.qw, static_cast<uint8_t*>(q.out), q.nrows, q.n_per_row, q.rows_per_qw};
        B.cum[B.count + 1] = B.cum[B.count] + tiles;
        if (++B.count == kMaxBatch) {
            const iqq_status st = launch<float, false>(B, weight_mode, fudge, d_flags, stream, nullptr, nullptr);
            if (st != IQQ_OK) return st;
            B.count = 0;
        }
    }
    if (B.count == 0) return IQQ_OK;
    return launch<float, false>(B, weight_mode, fudge, d_flags, stream, nullptr, nullptr);
}

}  // namespace iqq
