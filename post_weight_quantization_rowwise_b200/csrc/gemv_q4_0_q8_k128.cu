// gemv_q4_0_q8_k128.cu -- y[t][r] = dot(dequant(W[r]), dequant(A[t])) for Q4_0 weight rows W
// and Q8_K_128 activation rows A.
//
// Source: "ik_llama.cpp 量化精度修复实录：用 Q8_K_128 替代 Q8_1 根治 IQ1_S_R4 / IQ1_M_R4 的 fp16
// 溢出" (www.hnwysp.cn/news/39281).  修复前的数值隐患: the dot product multiplies UNSIGNED weight
// codes by the int8 activation codes and corrects the result with the activation block sum;
// 修复方案: Q8_K_128 keeps those sums per 32 values as int16, not multiplied by d, so the
// correction is exact.  For Q4_0 the unsigned code is the stored nibble u = l + 8, so per
// 32-value block
//     sum_i l_i q_i = sum_i u_i q_i - 8 * bsum        (exact in int32, |.| < 2^15).
//
// Arithmetic (every block term is exact, only the sums round):
//   isum  = dp4a over the nibbles - 8 * bsum                          int32, exact
//   term  = (double)d8 * ((double)d4 * (double)isum)                  11+15+24 bits: exact
//   y     = binary64 sum of the K/32 terms of the row, rounded once to binary32.
// (acc = fma(d8, d4 * isum, acc) is that exact product plus one rounding of the sum.)  The
// sums run in a fixed order for a given k -- per lane over its pairs of blocks, then a warp
// butterfly -- so results are reproducible and within (K/32 + 16) * 2^-53 * sum|terms| of
// the exact dot product before the final rounding.
//
// Mapping (HBM-bound on the weight stream at small token counts): a launch serves up to 64
// problems (matrices) with one wave of CTAs.  The problems' weights, laid end to end, are
// split into equal byte ranges, one per CTA; a CTA takes the rows that start in its range,
// of one problem or of several in turn (so the wave is balanced to a row whatever the
// problems' sizes).  Every warp of the CTA takes rows r_begin + warp, + 16, ... and streams
// each row through its own shared-memory stages in units of up to 64 pairs of blocks (2304
// bytes), copied with cp.async.bulk and completing on the warp's own mbarriers; lane 0
// keeps D units in flight.  A lane takes up to two pairs of blocks per unit (36 bytes each,
// read as nine 32-bit words: conflict-free because 9 is odd).  Partial sums stay in
// registers across the units of a row; one butterfly per row.  Per problem the CTA
// synchronizes after staging the problem's activations for its token tile (int8 codes with
// a 16-byte-chunk swizzle that keeps the per-lane 128-bit loads conflict-free, the binary32
// scales and the int16 block sums), and once more before staging the next problem's.
//
// Every wait on an mbarrier is bounded by a clock limit; on expiry the warp raises
// IQQ_FLAG_WAIT_TIMEOUT, drains its copies in flight (again bounded) and returns.
#include <cuda_fp16.h>

#include <atomic>

#include "common.cuh"

namespace {

constexpr int kWarps = 16;      // warps per CTA; 32 for one token when one CTA fits per SM
constexpr int kWarpsWide = 32;
constexpr int kUnitPairs = 64;                    // pairs of blocks per streamed unit
constexpr int kUnitBytes = kUnitPairs * 36 + 16;  // + room for the 8-byte start offset
__host__ __device__ constexpr int static_smem(int warps) { return warps * 4 * 8; }  // per-warp range slots
constexpr int kSmemCta = 227 * 1024;              // shared memory per CTA, at most
constexpr int kSmemPerSm = 228 * 1024;
constexpr long long kWaitCycles = 4000000000LL;   // about 2 s at the maximum SM clock
constexpr uint32_t kSuspendHintNs = 100000;
#ifndef IQQ_GEMV_WIDE
#define IQQ_GEMV_WIDE 1  // 32-warp CTAs for one token on very wide rows
#endif
#ifndef IQQ_GEMV_PDL
#define IQQ_GEMV_PDL 1  // launch with programmatic stream serialization
#endif

__device__ __forceinline__ uint32_t smem_addr(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(kSuspendHintNs)
        : "memory");
    return ok != 0u;
}

// Bounded wait for the phase with the given parity to complete.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > kWaitCycles) return false;
    }
    return true;
}

__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ int dp4a_us(uint32_t u, uint32_t s, int c)
{
    int r;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(r) : "r"(u), "r"(s), "r"(c));
    return r;
}

// One matrix-vector problem of a launch (the ABI's iqq_gemv_problem, validated).
struct Problem {
    const uint8_t* w;
    const uint8_t* a;
    float* y;
    int64_t n_out;
    int32_t k;
    int32_t n_tok;
};

constexpr int kMaxBatch = 64;  // problems per launch (kernel parameters stay under 4 KB)

struct Params {
    Problem prob[kMaxBatch];
    int64_t cum_bytes[kMaxBatch + 1];  // weight bytes of the problems before p
    int64_t share_q, share_r;          // B / C and B % C for B weight bytes over C byte shares
    int ctas, tiles;                   // C, and the token tiles per share (CTAs = C * tiles)
    int count;
    int stages;                    // D, units in flight per warp
    int off_stage, off_bar;        // shared-memory layout; activations below off_stage
    uint32_t* flags;
};
static_assert(sizeof(Params) <= 4096, "kernel parameters");

// What a CTA needs of its problem.
struct View {
    const uint8_t* w;
    int64_t wbytes;  // n_out * rowbytes
    int k, rowbytes, nseg;
};

// Byte offset of logical int8 index j of a token row in the swizzled layout: 16-byte chunk
// c = j / 16 of pair p = c / 4 is stored at chunk 4p + ((c % 4) ^ ((p >> 1) & 3)), so the
// lanes of a quarter warp (consecutive pairs) hit distinct bank groups.
__device__ __forceinline__ int q8_swizzle(int j)
{
    const int c = j >> 4, p = c >> 2;
    return (((p << 2) | ((c & 3) ^ ((p >> 1) & 3))) << 4) | (j & 15);
}

// Issues unit (row, seg) into a stage.  The copy starts at the 16-byte boundary at or below
// the unit's first byte (rows start 8 bytes past one when k % 256 == 128), so the unit's
// pairs begin at stage offset (start & 15).
__device__ __forceinline__ void issue_unit(const View& P, uint8_t* stage, uint64_t* bar, int64_t row, int seg)
{
    const int p0 = seg * kUnitPairs;
    const int np = (P.k >> 6) - p0 < kUnitPairs ? (P.k >> 6) - p0 : kUnitPairs;
    const int64_t start = row * P.rowbytes + 36LL * p0;
    const int64_t src = start & ~15LL;
    const uint32_t total = static_cast<uint32_t>(start - src) + 36u * np;
    uint32_t bulk = total & ~15u;
    if (bulk != total) {
        if (src + bulk + 16 <= P.wbytes) {
            bulk += 16;  // over-read up to 12 bytes that still lie inside the weights
        } else {
            // the end of the weights: the last 4-12 bytes by plain loads (4-byte aligned)
            for (uint32_t o = bulk; o < total; o += 4)
                *reinterpret_cast<uint32_t*>(stage + o) = __ldg(reinterpret_cast<const uint32_t*>(P.w + src + o));
        }
    }
    // order this thread's generic-proxy accesses to the stage before the async copy into it
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_arrive_expect_tx(bar, bulk);
    bulk_copy_g2s(stage, P.w + src, bulk, bar);
}

__device__ __forceinline__ double half_bits_to_double(unsigned short h)
{
    double d;
    asm("cvt.f64.f16 %0, %1;" : "=d"(d) : "h"(h));
    return d;
}

// One pair of blocks (nine words): block a (bytes 0..17) then block b (18..35).  qs holds
// the 16 code bytes of each block, 4-byte aligned (block a's are shifted into place); byte
// i of a block's codes has value i in its low nibble and value i + 16 in its high nibble.
struct PairW {
    uint32_t qs[8];
    uint32_t dh;  // the binary16 scales: block a's in the low half, block b's in the high half
};

__device__ __forceinline__ void load_pair(const uint32_t* w9, PairW& q)
{
    uint32_t w[9];
#pragma unroll
    for (int i = 0; i < 9; ++i) w[i] = w9[i];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        q.qs[m] = __funnelshift_r(w[m], w[m + 1], 16);
        q.qs[4 + m] = w[5 + m];
    }
    q.dh = __byte_perm(w[0], w[4], 0x7610);
}

__device__ __forceinline__ double scale_a(const PairW& q) { return half_bits_to_double(static_cast<unsigned short>(q.dh & 0xffffu)); }
__device__ __forceinline__ double scale_b(const PairW& q) { return half_bits_to_double(static_cast<unsigned short>(q.dh >> 16)); }

// acc += the two block terms of pair p for one token (d4a, d4b: the pair's scales).
__device__ __forceinline__ void pair_token(const PairW& q, double d4a, double d4b, const uint8_t* q8t,
                                           const int16_t* bst, const float* d8t, int p, int sw, double& acc)
{
    const uint8_t* qrow = q8t + (p << 6);
    uint4 v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = *reinterpret_cast<const uint4*>(qrow + ((j ^ sw) << 4));
    constexpr uint32_t L = 0x0F0F0F0Fu, H = 0xF0F0F0F0u;  // high nibbles kept in place: x16
    int la = 0, ha = 0, lb = 0, hb = 0;
    la = dp4a_us(q.qs[0] & L, v[0].x, la); la = dp4a_us(q.qs[1] & L, v[0].y, la);
    la = dp4a_us(q.qs[2] & L, v[0].z, la); la = dp4a_us(q.qs[3] & L, v[0].w, la);
    ha = dp4a_us(q.qs[0] & H, v[1].x, ha); ha = dp4a_us(q.qs[1] & H, v[1].y, ha);
    ha = dp4a_us(q.qs[2] & H, v[1].z, ha); ha = dp4a_us(q.qs[3] & H, v[1].w, ha);
    lb = dp4a_us(q.qs[4] & L, v[2].x, lb); lb = dp4a_us(q.qs[5] & L, v[2].y, lb);
    lb = dp4a_us(q.qs[6] & L, v[2].z, lb); lb = dp4a_us(q.qs[7] & L, v[2].w, lb);
    hb = dp4a_us(q.qs[4] & H, v[3].x, hb); hb = dp4a_us(q.qs[5] & H, v[3].y, hb);
    hb = dp4a_us(q.qs[6] & H, v[3].z, hb); hb = dp4a_us(q.qs[7] & H, v[3].w, hb);
    const uint32_t bsw = *reinterpret_cast<const uint32_t*>(bst + 2 * p);
    // the high-nibble products carry a factor 16, so the shift is exact
    const int ia = la + (ha >> 4) - 8 * static_cast<int>(static_cast<int16_t>(bsw & 0xffffu));
    const int ib = lb + (hb >> 4) - 8 * static_cast<int>(static_cast<int16_t>(bsw >> 16));
    const double d8 = static_cast<double>(d8t[p >> 1]);
    acc = fma(d8, d4a * static_cast<double>(ia), acc);
    acc = fma(d8, d4b * static_cast<double>(ib), acc);
}

// First row of a problem whose weights start at or after byte `off` of the problem (rows of
// `rowbytes` bytes; 0 before the problem, n_out past its end).  32-bit division when the
// offset allows it (the 64-bit one is a long call).
__device__ __forceinline__ int64_t row_at(int64_t off, int rowbytes, int64_t n_out)
{
    if (off <= 0) return 0;
    const int64_t r = off < (1LL << 31) ? static_cast<int64_t>((static_cast<uint32_t>(off) + (rowbytes - 1)) /
                                                               static_cast<uint32_t>(rowbytes))
                                        : (off + rowbytes - 1) / rowbytes;
    return r < n_out ? r : n_out;
}

// Start of share c of the launch's B weight bytes: floor(c * B / C) =
// c * (B / C) + floor(c * (B % C) / C), where c * (B % C) < C^2 < 2^32.
__device__ __forceinline__ int64_t share_start(const Params& P, uint32_t c)
{
    return static_cast<int64_t>(c) * P.share_q +
           static_cast<int64_t>(c * static_cast<uint32_t>(P.share_r) / static_cast<uint32_t>(P.ctas));
}

template <int TT, int W>
__global__ void __launch_bounds__(W * 32, TT == 1 && W == kWarps ? 2 : 1)
gemv_q4_0_q8_k128_kernel(const __grid_constant__ Params P)
{
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // CTA id = share * tiles + token tile: the token tiles of one share are neighbours in
    // launch order, so they run side by side and the share's weights come from DRAM about
    // once (the others read them from L2)
    const uint32_t share = blockIdx.x / static_cast<uint32_t>(P.tiles);
    const int64_t tok0 = static_cast<int64_t>(blockIdx.x - share * static_cast<uint32_t>(P.tiles)) * TT;
    uint8_t* stages = smem + P.off_stage + warp * P.stages * kUnitBytes;               // this warp's
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + P.off_bar) + warp * P.stages;  // this warp's
    const int D = P.stages;

    // Programmatic dependent launch: let the next kernel of the stream be scheduled as this
    // grid's CTAs retire.  (A no-op without the launch attribute.)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (lane == 0) {
        for (int i = 0; i < D; ++i) mbar_init(&bars[i], 1u);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }

    // the stage ring, shared by the issue and consume pointers (equal between problems)
    int s = 0;
    uint32_t ph = 0;
    bool aborted = false, staged = false;
    // units start on 64-pair boundaries, so a lane's pairs p0 + lane and p0 + lane + 32 share
    // the swizzle phase (p >> 1) & 3 = (lane >> 1) & 3
    const int sw = (lane >> 1) & 3;

    // This CTA's equal share [t0, t1) of the launch's weight bytes (the problems' weights
    // laid end to end): it takes the rows that start inside it, of one problem or several.
    // The first and last problems it touches and its first / end row in them are found once,
    // here, and parked in shared memory (the 64-bit divisions are calls that would otherwise
    // force the row loops' registers to the stack).
    __shared__ int64_t s_rng[W][4];
    static_assert(sizeof(s_rng) == static_smem(W), "static shared memory of the launch plan");
    {
        const int64_t t0 = share_start(P, share), t1 = share_start(P, share + 1);
        int pf = 0;
        while (pf + 1 < P.count && P.cum_bytes[pf + 1] <= t0) ++pf;
        int pl = pf;
        while (pl + 1 < P.count && P.cum_bytes[pl + 1] < t1) ++pl;
        if (lane == 0) {
            s_rng[warp][0] = pf;
            s_rng[warp][1] = row_at(t0 - P.cum_bytes[pf], (P.prob[pf].k >> 5) * 18, P.prob[pf].n_out);
            s_rng[warp][2] = pl;
            s_rng[warp][3] = row_at(t1 - P.cum_bytes[pl], (P.prob[pl].k >> 5) * 18, P.prob[pl].n_out);
        }
        __syncwarp();
    }

    // Everything above reads only the parameters and shared memory.  Wait for the previous
    // kernel of the stream (completion and memory flush) before the first access to global
    // memory.  (A no-op without the launch attribute.)
    asm volatile("griddepcontrol.wait;" ::: "memory");

    for (int pi = static_cast<int>(s_rng[warp][0]); pi <= static_cast<int>(s_rng[warp][2]); ++pi) {
        const Problem& pr = P.prob[pi];
        const int k = pr.k, nb8 = k >> 7, nb4 = k >> 5, npairs = k >> 6;
        View V;
        V.w = pr.w;
        V.k = k;
        V.rowbytes = nb4 * 18;
        V.wbytes = pr.n_out * V.rowbytes;
        V.nseg = (npairs + kUnitPairs - 1) / kUnitPairs;
        const int64_t r_begin = pi == static_cast<int>(s_rng[warp][0]) ? s_rng[warp][1] : 0;
        const int64_t r_end = pi == static_cast<int>(s_rng[warp][2]) ? s_rng[warp][3] : pr.n_out;
        // rows of this CTA, counted from r_begin (a share of one wave: far below 2^31)
        const int nrows = static_cast<int>(r_end - r_begin);
        if (nrows <= 0 || tok0 >= pr.n_tok) continue;  // the same for the whole CTA
        const int nt = static_cast<int>(pr.n_tok - tok0 < TT ? pr.n_tok - tok0 : TT);
        const int act_q8_bytes = (k + 15) & ~15;
        uint8_t* q8s = smem;                                                                  // [TT][k]
        float* d8s = reinterpret_cast<float*>(smem + TT * act_q8_bytes);                      // [TT][k/128]
        int16_t* bss = reinterpret_cast<int16_t*>(smem + ((TT * act_q8_bytes + TT * nb8 * 4 + 15) & ~15));
        const int nseg = V.nseg;

        // issue pointer: the next unit (irow, iseg) to copy; the first D go out now
        int irow = warp;
        int iseg = 0;
        int is = s;
        if (!aborted) {
            for (int u = 0; u < D && irow < nrows; ++u) {
                if (lane == 0) issue_unit(V, stages + is * kUnitBytes, &bars[is], r_begin + irow, iseg);
                if (++iseg == nseg) {
                    iseg = 0;
                    irow += W;
                }
                if (++is == D) is = 0;
            }
        }

        // Stage the token tile's activations while the first units are in flight: one warp
        // per 140-byte block, lane i copying code word i, several blocks of a warp in
        // flight at once (the tile's blocks are contiguous in global memory: its tokens'
        // rows follow one another).  The barrier before it keeps the previous problem's
        // activations until every warp has finished with them.
        if (staged) __syncthreads();
        staged = true;
        {
            // (4 with one token: 8 would push the row loop's registers to the stack)
            constexpr int kStageBlocks = TT == 1 ? 4 : 8;
            const int nblk = nt * nb8;
            const uint8_t* abase = pr.a + tok0 * nb8 * 140;
            for (int b0 = warp; b0 < nblk; b0 += kStageBlocks * W) {
                uint32_t v[kStageBlocks], e[kStageBlocks];
#pragma unroll
                for (int u = 0; u < kStageBlocks; ++u) {
                    const int b = b0 + u * W;
                    v[u] = 0u;
                    e[u] = 0u;
                    if (b < nblk) {
                        const uint32_t* src = reinterpret_cast<const uint32_t*>(abase + static_cast<int64_t>(b) * 140);
                        v[u] = __ldg(src + 1 + lane);
                        if (lane < 3) e[u] = __ldg(src + (lane == 0 ? 0 : 32 + lane));
                    }
                }
#pragma unroll
                for (int u = 0; u < kStageBlocks; ++u) {
                    const int b = b0 + u * W;
                    if (b < nblk) {
                        const int t = b / nb8, g = b - t * nb8;
                        *reinterpret_cast<uint32_t*>(q8s + t * act_q8_bytes + q8_swizzle(128 * g + 4 * lane)) = v[u];
                        if (lane == 0) d8s[t * nb8 + g] = __uint_as_float(e[u]);
                        else if (lane < 3)
                            *reinterpret_cast<uint32_t*>(bss + t * nb4 + 4 * g + 2 * (lane - 1)) = e[u];
                    }
                }
            }
        }
        __syncthreads();
        if (aborted) continue;  // a warp that gave up still meets every barrier

        double acc[TT];
#pragma unroll
        for (int t = 0; t < TT; ++t) acc[t] = 0.0;
        // consume pointer: unit (row, seg) in stage s, phase parity ph
        int row = warp;
        int seg = 0;
        while (row < nrows) {
            const bool timed_out = !mbar_wait(&bars[s], ph);
            if (__any_sync(0xffffffffu, timed_out)) {
                aborted = true;
                break;
            }
            const int p0 = seg * kUnitPairs;
            const int np = npairs - p0 < kUnitPairs ? npairs - p0 : kUnitPairs;
            const int64_t start = (r_begin + row) * V.rowbytes + 36LL * p0;
            const uint32_t* w9 = reinterpret_cast<const uint32_t*>(stages + s * kUnitBytes + (start & 15));

            PairW q0, q1;
            const bool has0 = lane < np, has1 = lane + 32 < np;
            if (has0) load_pair(w9 + 9 * lane, q0);
            if (has1) load_pair(w9 + 9 * (lane + 32), q1);
            __syncwarp();
            // every lane holds its words: refill the stage with the next unit to copy
            if (irow < nrows) {
                if (lane == 0) issue_unit(V, stages + s * kUnitBytes, &bars[s], r_begin + irow, iseg);
                if (++iseg == nseg) {
                    iseg = 0;
                    irow += W;
                }
            }
            if (TT == 1) {
                // one token: each scale is used once, converted where it is used (fewer
                // registers live across the unit)
                if (has0) pair_token(q0, scale_a(q0), scale_b(q0), q8s, bss, d8s, p0 + lane, sw, acc[0]);
                if (has1) pair_token(q1, scale_a(q1), scale_b(q1), q8s, bss, d8s, p0 + lane + 32, sw, acc[0]);
            } else {
                const double a0 = scale_a(q0), b0s = scale_b(q0), a1 = scale_a(q1), b1s = scale_b(q1);
#pragma unroll
                for (int t = 0; t < TT; ++t) {
                    if (t < nt) {
                        const uint8_t* q8t = q8s + t * act_q8_bytes;
                        const int16_t* bst = bss + t * nb4;
                        const float* d8t = d8s + t * nb8;
                        if (has0) pair_token(q0, a0, b0s, q8t, bst, d8t, p0 + lane, sw, acc[t]);
                        if (has1) pair_token(q1, a1, b1s, q8t, bst, d8t, p0 + lane + 32, sw, acc[t]);
                    }
                }
            }
            if (++seg == nseg) {  // the row is complete
#pragma unroll
                for (int t = 0; t < TT; ++t) {
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
                }
                if (lane == 0) {
#pragma unroll
                    for (int t = 0; t < TT; ++t)
                        if (t < nt) pr.y[(tok0 + t) * pr.n_out + r_begin + row] = static_cast<float>(acc[t]);
                }
#pragma unroll
                for (int t = 0; t < TT; ++t) acc[t] = 0.0;
                seg = 0;
                row += W;
            }
            if (++s == D) {
                s = 0;
                ph ^= 1u;
            }
        }

        if (aborted && lane == 0) {
            // a wait ran out: report, then wait (bounded) for this warp's copies in flight,
            // which are the units from (row, seg) up to the issue pointer
            iqq::raise_flags(P.flags, IQQ_FLAG_WAIT_TIMEOUT);
            for (int j = 0; j < D && (row < irow || (row == irow && seg < iseg)); ++j) {
                (void)mbar_wait(&bars[s], ph);
                if (++seg == nseg) {
                    seg = 0;
                    row += W;
                }
                if (++s == D) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
    }
}

// Per-device launch facts, queried once per process and device (a call otherwise spends more
// time in these queries than a small matrix takes on the GPU).
struct DeviceCache {
    std::atomic<int> sms{0};
    std::atomic<int> smem_set[8] = {};  // dynamic smem opted in, per (TT, W)
    std::atomic<int> regs[8] = {};      // registers per thread, per (TT, W)
};
constexpr int kMaxDevices = 64;
DeviceCache g_cache[kMaxDevices];

int current_device()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) dev = 0;
    return dev;
}

int sm_count_gemv(int dev)
{
    int sms = g_cache[dev].sms.load(std::memory_order_relaxed);
    if (sms == 0) {
        sms = 148;
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        g_cache[dev].sms.store(sms, std::memory_order_relaxed);
    }
    return sms;
}

constexpr int tt_slot(int tt, int w)
{
    return 2 * (tt == 1 ? 0 : (tt == 2 ? 1 : (tt == 4 ? 2 : 3))) + (w == kWarps ? 0 : 1);
}

int align16(int v) { return (v + 15) & ~15; }

// Shared-memory layout of a launch: activations of tt tokens for the largest k, then d
// units per warp, then the warps' mbarriers.
int act_bytes(int tt, int k) { return align16(align16(tt * align16(k) + tt * (k / 128) * 4) + tt * (k / 32) * 2); }

void make_plan(Params& P, int tt, int kmax, int d, int w)
{
    P.stages = d;
    P.off_stage = act_bytes(tt, kmax);
    P.off_bar = P.off_stage + w * d * kUnitBytes;
}

int smem_bytes(const Params& P, int w) { return P.off_bar + w * P.stages * 8; }

// Resident CTAs per SM: 228 KB of shared memory (1 KB reserved per CTA) and 64 K registers
// (allocated per warp in units of 256).
int ctas_per_sm(int smem, int regs, int w)
{
    int occ = kSmemPerSm / (smem + static_smem(w) + 1024);
    const int regs_cta = ((regs * 32 + 255) / 256) * 256 * w;
    if (65536 / regs_cta < occ) occ = 65536 / regs_cta;
    return occ;
}

template <int TT, int W>
int kernel_regs(int dev)
{
    std::atomic<int>& cached = g_cache[dev].regs[tt_slot(TT, W)];
    int regs = cached.load(std::memory_order_relaxed);
    if (regs == 0) {
        cudaFuncAttributes fa{};
        regs = 64;
        if (cudaFuncGetAttributes(&fa, gemv_q4_0_q8_k128_kernel<TT, W>) == cudaSuccess && fa.numRegs > 0)
            regs = fa.numRegs;
        cached.store(regs, std::memory_order_relaxed);
    }
    return regs;
}

// Chooses D in 2..4 for CTAs of w warps: the most units in flight per SM among the layouts
// that fit, and at equal flight the layout with more resident warps (measured on B200: 32
// warps x 2 units beat 16 warps x 4 units, the per-unit arithmetic needing the extra warps to
// hide its latency).  Returns the flight (0: nothing fits).
int plan_w(Params& P, int tt, int kmax, int regs, int w, int& ctas)
{
    int best_d = 0, best_flight = 0, best_ctas = 0;
    for (int d = 2; d <= 4; ++d) {
        make_plan(P, tt, kmax, d, w);
        const int smem = smem_bytes(P, w);
        if (smem > kSmemCta - static_smem(w)) break;
        const int c = ctas_per_sm(smem, regs, w);
        if (c < 1) break;
        if (c * d > best_flight) {
            best_flight = c * d;
            best_d = d;
            best_ctas = c;
        }
    }
    if (best_d == 0) return 0;
    make_plan(P, tt, kmax, best_d, w);
    ctas = best_ctas;
    return best_flight * w;
}

// The launch plan of a token tile: CTAs of 16 warps; at one token, when the activations
// leave room for only one such CTA per SM (very wide rows), CTAs of 32 warps sharing one
// activation copy if they keep as many units in flight (twice the warps to hide the
// per-unit arithmetic).
template <int TT>
bool plan_tt(Params& P, int kmax, int dev, int& ctas, int& warps)
{
    int c16 = 0;
    const int f16 = plan_w(P, TT, kmax, kernel_regs<TT, kWarps>(dev), kWarps, c16);
    if constexpr (TT == 1) {
        if (IQQ_GEMV_WIDE && (f16 == 0 || c16 == 1)) {
            Params Q = P;
            int c32 = 0;
            const int f32 = plan_w(Q, TT, kmax, kernel_regs<TT, kWarpsWide>(dev), kWarpsWide, c32);
            if (f32 > 0 && f32 >= f16) {
                P = Q;
                ctas = c32;
                warps = kWarpsWide;
                return true;
            }
        }
    }
    if (f16 == 0) return false;
    ctas = c16;
    warps = kWarps;
    return true;
}

// Launches P.count (<= kMaxBatch) problems: c0 byte shares, one wave of CTAs (fewer when the
// problems have fewer than 16 rows per CTA) splitting the problems' weight bytes evenly, each
// share times the token tiles, on a one-dimensional grid.
template <int TT, int W>
iqq_status opt_in_smem(int dev, int smem)
{
    std::atomic<int>& opted = g_cache[dev].smem_set[tt_slot(TT, W)];
    if (opted.load(std::memory_order_relaxed) < smem) {
        const int cap = kSmemCta - static_smem(W);
        if (cudaFuncSetAttribute(gemv_q4_0_q8_k128_kernel<TT, W>, cudaFuncAttributeMaxDynamicSharedMemorySize, cap) !=
            cudaSuccess)
            return iqq::launch_status();
        opted.store(cap, std::memory_order_relaxed);
    }
    return IQQ_OK;
}

template <int TT>
iqq_status launch_tt(Params& P, int kmax, int64_t max_tok, cudaStream_t st, bool& fits)
{
    const int dev = current_device();
    int ctas = 0, warps = kWarps;
    fits = plan_tt<TT>(P, kmax, dev, ctas, warps);
    if (!fits) return IQQ_OK;
    const int smem = smem_bytes(P, warps);
    void (*kern)(Params) = gemv_q4_0_q8_k128_kernel<TT, kWarps>;
    if constexpr (TT == 1) {
        if (warps == kWarpsWide) kern = gemv_q4_0_q8_k128_kernel<TT, kWarpsWide>;
    }
    {
        iqq_status o = IQQ_OK;
        if constexpr (TT == 1) {
            o = warps == kWarpsWide ? opt_in_smem<TT, kWarpsWide>(dev, smem) : opt_in_smem<TT, kWarps>(dev, smem);
        } else {
            o = opt_in_smem<TT, kWarps>(dev, smem);
        }
        if (o != IQQ_OK) return o;
    }
    int64_t rows = 0;
    P.cum_bytes[0] = 0;
    for (int i = 0; i < P.count; ++i) {
        P.cum_bytes[i + 1] = P.cum_bytes[i] + P.prob[i].n_out * ((P.prob[i].k / 32) * 18);
        rows += P.prob[i].n_out;
    }
    int64_t c0 = static_cast<int64_t>(sm_count_gemv(dev)) * ctas;
    if (c0 > (rows + warps - 1) / warps) c0 = (rows + warps - 1) / warps;
    if (c0 < 1) c0 = 1;
    if (c0 > 65535) c0 = 65535;  // keeps c * (B % C) below 2^32
    P.share_q = P.cum_bytes[P.count] / c0;
    P.share_r = P.cum_bytes[P.count] % c0;
    const int64_t gy = (max_tok + TT - 1) / TT;
    if (gy > 65535 || c0 * gy > 0x7fffffffLL) return IQQ_ERR_SHAPE;
    P.ctas = static_cast<int>(c0);
    P.tiles = static_cast<int>(gy);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(c0 * gy));
    cfg.blockDim = dim3(static_cast<unsigned>(warps * 32));
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = IQQ_GEMV_PDL;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, P) != cudaSuccess) return iqq::launch_status();
    return iqq::launch_status();
}

// Host checks of one problem, before anything is enqueued.
iqq_status check_problem(const iqq_gemv_problem& q)
{
    if (q.n_out < 0 || q.k < 0 || q.n_tok < 0 || q.k % 128 != 0 || q.k > IQQ_GEMV_MAX_K) return IQQ_ERR_SHAPE;
    if (!iqq::size_ok(q.n_out, q.k, 1) || !iqq::size_ok(q.n_tok, q.k, 2) || !iqq::size_ok(q.n_tok, q.n_out, 4))
        return IQQ_ERR_SHAPE;
    if (q.n_out == 0 || q.n_tok == 0) return IQQ_OK;
    if (q.y == nullptr) return IQQ_ERR_NULL;
    if (!iqq::aligned(q.y, 4)) return IQQ_ERR_ALIGN;
    if (q.k == 0) return IQQ_OK;
    if (q.w_blocks == nullptr || q.a_blocks == nullptr) return IQQ_ERR_NULL;
    if (!iqq::aligned(q.w_blocks, 16) || !iqq::aligned(q.a_blocks, 4)) return IQQ_ERR_ALIGN;
    return IQQ_OK;
}

iqq_status gemv_batch(const iqq_gemv_problem* probs, int64_t count, uint32_t* d_flags, cudaStream_t st)
{
    if (count < 0) return IQQ_ERR_SHAPE;
    if (count > 0 && probs == nullptr) return IQQ_ERR_NULL;
    if (!iqq::aligned(d_flags, 4)) return IQQ_ERR_ALIGN;
    for (int64_t i = 0; i < count; ++i) {
        const iqq_status c = check_problem(probs[i]);
        if (c != IQQ_OK) return c;
    }
    Params P{};
    P.flags = d_flags;
    int kmax = 0;
    int64_t max_tok = 0;
    auto flush = [&]() -> iqq_status {
        if (P.count == 0) return IQQ_OK;
        // token tile: the smallest of 1, 2, 4, 8 covering the largest n_tok (8 beyond),
        // halved while the activations do not fit beside the weight stages
        int tt = max_tok >= 5 ? 8 : (max_tok >= 3 ? 4 : static_cast<int>(max_tok));
        iqq_status s = IQQ_OK;
        for (;;) {
            bool fits = false;
            switch (tt) {
            case 1: s = launch_tt<1>(P, kmax, max_tok, st, fits); break;
            case 2: s = launch_tt<2>(P, kmax, max_tok, st, fits); break;
            case 4: s = launch_tt<4>(P, kmax, max_tok, st, fits); break;
            default: s = launch_tt<8>(P, kmax, max_tok, st, fits); break;
            }
            if (fits || s != IQQ_OK) break;
            if (tt == 1) return IQQ_ERR_SHAPE;
            tt >>= 1;
        }
        P.count = 0;
        kmax = 0;
        max_tok = 0;
        return s;
    };
    for (int64_t i = 0; i < count; ++i) {
        const iqq_gemv_problem& q = probs[i];
        if (q.n_out == 0 || q.n_tok == 0) continue;
        if (q.k == 0) {
            // the dot product of empty vectors
            if (cudaMemsetAsync(q.y, 0, static_cast<size_t>(q.n_tok * q.n_out) * sizeof(float), st) != cudaSuccess)
                return iqq::launch_status();
            continue;
        }
        Problem& pr = P.prob[P.count++];
        pr.w = static_cast<const uint8_t*>(q.w_blocks);
        pr.a = static_cast<const uint8_t*>(q.a_blocks);
        pr.y = q.y;
        pr.n_out = q.n_out;
        pr.k = static_cast<int32_t>(q.k);
        pr.n_tok = static_cast<int32_t>(q.n_tok);
        if (pr.k > kmax) kmax = pr.k;
        if (q.n_tok > max_tok) max_tok = q.n_tok;
        if (P.count == kMaxBatch) {
            const iqq_status s = flush();
            if (s != IQQ_OK) return s;
        }
    }
    return flush();
}

}  // namespace

extern "C" iqq_status iqq_gemv_q4_0_q8_k128(const void* w_blocks, const void* a_blocks, float* y,
                                            int64_t n_out, int64_t k, int64_t n_tok, uint32_t* d_flags,
                                            void* stream)
{
    iqq_gemv_problem q;
    q.w_blocks = w_blocks;
    q.a_blocks = a_blocks;
    q.y = y;
    q.n_out = n_out;
    q.k = k;
    q.n_tok = n_tok;
    return gemv_batch(&q, 1, d_flags, static_cast<cudaStream_t>(stream));
}

extern "C" iqq_status iqq_gemv_q4_0_q8_k128_batch(const iqq_gemv_problem* problems, int64_t count,
                                                  uint32_t* d_flags, void* stream)
{
    return gemv_batch(problems, count, d_flags, static_cast<cudaStream_t>(stream));
}
