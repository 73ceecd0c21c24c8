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
// The sums run in a fixed order for a given (n_out, k): per lane over its pairs of blocks, a
// warp butterfly, then the row's segment partials in order -- so results are reproducible
// and within (K/32 + 16) * 2^-53 * sum|terms| of the exact dot before the final rounding.
//
// Mapping (HBM-bound on the weight stream at small token counts):
//  * The weights stream through shared memory in chunks of R whole rows (rows are
//    contiguous, so a chunk is one contiguous byte range) with cp.async.bulk, completing on
//    an mbarrier per stage; 2-4 stages are in flight per CTA.  The CTA is persistent over
//    chunks c = blockIdx.x + i * gridDim.x.
//  * The activations of the CTA's token tile (TT tokens) are staged once: int8 codes with a
//    16-byte-chunk swizzle that makes the per-lane 128-bit loads conflict-free, the binary32
//    scales and the int16 block sums.
//  * A warp owns one (row, segment) task per chunk; a lane takes a pair of blocks (64 values,
//    36 bytes read as nine 32-bit words -- conflict-free because 9 is odd).
//  * Every wait on an mbarrier is bounded by a clock limit; on expiry the CTA raises
//    IQQ_FLAG_WAIT_TIMEOUT, drains its copies in flight (again bounded) and returns.
#include <cuda_fp16.h>

#include <atomic>

#include "common.cuh"

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxStages = 4;
constexpr int kChunkTarget = 32 * 1024;
constexpr int kSmemMax = 227 * 1024;
constexpr int kSmemPerSm = 228 * 1024;
constexpr long long kWaitCycles = 4000000000LL;  // about 2 s at the maximum SM clock

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
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
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

struct Params {
    const uint8_t* w;
    const uint8_t* a;
    float* y;
    uint32_t* flags;
    int64_t n_out;
    int64_t n_tok;
    int k;
    int rowbytes;     // (k / 32) * 18
    int rows;         // R, rows per chunk
    int seg;          // segments per row (R * seg == kWarps)
    int pps;          // pairs of blocks per segment
    int stages;
    int64_t nchunks;
    int act_q8_bytes;  // per token, k
    int chunk_bytes;   // R * rowbytes rounded up to 16
    int off_d8, off_bs, off_stage, off_part, off_bar;  // shared-memory layout
};

// Byte offset of logical int8 index j of a token row in the swizzled layout: 16-byte chunk
// c = j / 16 of pair p = c / 4 is stored at chunk 4p + ((c % 4) ^ ((p >> 1) & 3)).
__host__ __device__ __forceinline__ int q8_swizzle(int j)
{
    const int c = j >> 4, p = c >> 2;
    return (((p << 2) | ((c & 3) ^ ((p >> 1) & 3))) << 4) | (j & 15);
}

__device__ __forceinline__ void issue_chunk(const Params& P, uint8_t* stage, uint64_t* bar, int64_t c)
{
    const int64_t row0 = c * P.rows;
    const int64_t nr = P.n_out - row0 < P.rows ? P.n_out - row0 : P.rows;
    const uint32_t bytes = static_cast<uint32_t>(nr * P.rowbytes);
    const uint32_t body = bytes & ~15u;
    const uint8_t* src = P.w + row0 * P.rowbytes;
    if (bytes != body) {
        // last chunk of a matrix whose byte size is 8 mod 16: the final 8 bytes by a plain
        // load (8-byte aligned: body is a multiple of 16 from a 16-byte aligned start)
        *reinterpret_cast<uint2*>(stage + body) = __ldg(reinterpret_cast<const uint2*>(src + body));
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    mbar_arrive_expect_tx(bar, body);
    bulk_copy_g2s(stage, src, body, bar);
}

template <int TT>
__global__ void __launch_bounds__(kThreads)
gemv_q4_0_q8_k128_kernel(const Params P)
{
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t* q8s = smem;                                              // [TT][k] swizzled
    float* d8s = reinterpret_cast<float*>(smem + P.off_d8);           // [TT][k/128]
    int16_t* bss = reinterpret_cast<int16_t*>(smem + P.off_bs);       // [TT][k/32]
    uint8_t* stages = smem + P.off_stage;                             // [stages][chunk_bytes]
    double* part = reinterpret_cast<double*>(smem + P.off_part);      // [2][kWarps][TT]
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + P.off_bar);   // [stages]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t tok0 = static_cast<int64_t>(blockIdx.y) * TT;
    const int nt = static_cast<int>(P.n_tok - tok0 < TT ? P.n_tok - tok0 : TT);
    const int k = P.k, nb8 = k >> 7, nb4 = k >> 5;

    if (tid == 0) {
        for (int s = 0; s < P.stages; ++s) mbar_init(&bars[s], 1u);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    __syncthreads();
    if (tid == 0) {
        for (int s = 0; s < P.stages; ++s) {
            const int64_t c = blockIdx.x + static_cast<int64_t>(s) * gridDim.x;
            if (c < P.nchunks) issue_chunk(P, stages + s * P.chunk_bytes, &bars[s], c);
        }
    }

    // Stage the token tile's activations (35 words per 140-byte block) while the first
    // weight chunks are in flight.
    {
        const int words = nt * nb8 * 35;
        for (int i = tid; i < words; i += kThreads) {
            const int t = i / (nb8 * 35), rem = i - t * (nb8 * 35);
            const int g = rem / 35, wi = rem - g * 35;
            const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(
                P.a + ((tok0 + t) * nb8 + g) * 140 + 4 * wi));
            if (wi == 0) {
                d8s[t * nb8 + g] = __uint_as_float(v);
            } else if (wi <= 32) {
                *reinterpret_cast<uint32_t*>(q8s + t * P.act_q8_bytes + q8_swizzle(128 * g + 4 * (wi - 1))) = v;
            } else {
                *reinterpret_cast<uint32_t*>(bss + t * nb4 + 4 * g + 2 * (wi - 33)) = v;
            }
        }
    }
    __syncthreads();

    const int P2 = k >> 6;  // pairs of blocks per row
    int64_t it = 0;
    bool aborted = false;
    for (int64_t c = blockIdx.x; c < P.nchunks; c += gridDim.x, ++it) {
        const int s = static_cast<int>(it % P.stages);
        const uint32_t parity = static_cast<uint32_t>((it / P.stages) & 1);
        const bool timed_out = !mbar_wait(&bars[s], parity);
        const uint8_t* stage = stages + s * P.chunk_bytes;
        const int64_t row0 = c * P.rows;
        double* pw = part + (it & 1) * (kWarps * TT);

        // one (row, segment) task per warp
        const int rho = warp / P.seg, sigma = warp - rho * P.seg;
        double acc[TT];
#pragma unroll
        for (int t = 0; t < TT; ++t) acc[t] = 0.0;
        if (row0 + rho < P.n_out) {
            const int pb = sigma * P.pps;
            const int pe = pb + P.pps < P2 ? pb + P.pps : P2;
            const uint32_t* rw = reinterpret_cast<const uint32_t*>(stage + rho * P.rowbytes);
            for (int p = pb + lane; p < pe; p += 32) {
                uint32_t w[9];
#pragma unroll
                for (int i = 0; i < 9; ++i) w[i] = rw[9 * p + i];
                const float d4a = __half2float(__ushort_as_half(static_cast<unsigned short>(w[0] & 0xffffu)));
                const float d4b = __half2float(__ushort_as_half(static_cast<unsigned short>(w[4] >> 16)));
                uint32_t lo[8], hi[8];  // nibbles of block a (0..3) and block b (4..7)
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const uint32_t qa = __funnelshift_r(w[m], w[m + 1], 16);
                    lo[m] = qa & 0x0F0F0F0Fu;
                    hi[m] = (qa >> 4) & 0x0F0F0F0Fu;
                    lo[4 + m] = w[5 + m] & 0x0F0F0F0Fu;
                    hi[4 + m] = (w[5 + m] >> 4) & 0x0F0F0F0Fu;
                }
                const int sw = (p >> 1) & 3;
#pragma unroll
                for (int t = 0; t < TT; ++t) {
                    if (t < nt) {
                        const uint8_t* qrow = q8s + t * P.act_q8_bytes + (p << 6);
                        uint4 q[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) q[j] = *reinterpret_cast<const uint4*>(qrow + ((j ^ sw) << 4));
                        // block a: values 0..15 <- q[0], q[1]; values 16..31 <- q[2], q[3]
                        int sa = 0, sb = 0;
                        sa = dp4a_us(lo[0], q[0].x, sa); sa = dp4a_us(lo[1], q[0].y, sa);
                        sa = dp4a_us(lo[2], q[0].z, sa); sa = dp4a_us(lo[3], q[0].w, sa);
                        sa = dp4a_us(hi[0], q[1].x, sa); sa = dp4a_us(hi[1], q[1].y, sa);
                        sa = dp4a_us(hi[2], q[1].z, sa); sa = dp4a_us(hi[3], q[1].w, sa);
                        sb = dp4a_us(lo[4], q[2].x, sb); sb = dp4a_us(lo[5], q[2].y, sb);
                        sb = dp4a_us(lo[6], q[2].z, sb); sb = dp4a_us(lo[7], q[2].w, sb);
                        sb = dp4a_us(hi[4], q[3].x, sb); sb = dp4a_us(hi[5], q[3].y, sb);
                        sb = dp4a_us(hi[6], q[3].z, sb); sb = dp4a_us(hi[7], q[3].w, sb);
                        const uint32_t bsw = *reinterpret_cast<const uint32_t*>(bss + t * nb4 + 2 * p);
                        const int ia = sa - 8 * static_cast<int>(static_cast<int16_t>(bsw & 0xffffu));
                        const int ib = sb - 8 * static_cast<int>(static_cast<int16_t>(bsw >> 16));
                        const double d8 = static_cast<double>(d8s[t * nb8 + (p >> 1)]);
                        acc[t] += d8 * (static_cast<double>(d4a) * static_cast<double>(ia));
                        acc[t] += d8 * (static_cast<double>(d4b) * static_cast<double>(ib));
                    }
                }
            }
        }
#pragma unroll
        for (int t = 0; t < TT; ++t) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
        }
        if (lane == 0) {
#pragma unroll
            for (int t = 0; t < TT; ++t) pw[warp * TT + t] = acc[t];
        }
        if (__syncthreads_or(timed_out)) {  // uniform across the CTA
            aborted = true;
            break;
        }
        // refill the stage just consumed (every thread has passed its reads)
        if (tid == 0) {
            const int64_t cn = c + static_cast<int64_t>(P.stages) * gridDim.x;
            if (cn < P.nchunks) issue_chunk(P, stages + s * P.chunk_bytes, &bars[s], cn);
        }
        // finalize: row partials summed over segments in order
        if (tid < P.rows * nt) {
            const int r = tid / nt, t = tid - r * nt;
            if (row0 + r < P.n_out) {
                double v = 0.0;
                for (int sg = 0; sg < P.seg; ++sg) v += pw[(r * P.seg + sg) * TT + t];
                P.y[(tok0 + t) * P.n_out + row0 + r] = static_cast<float>(v);
            }
        }
    }

    if (aborted && tid == 0) {
        iqq::raise_flags(P.flags, IQQ_FLAG_WAIT_TIMEOUT);
        // drain: wait (bounded) for every copy this CTA issued and did not consume
        int64_t j = it;
        for (int64_t c = blockIdx.x + it * static_cast<int64_t>(gridDim.x); c < P.nchunks && j < it + P.stages;
             c += gridDim.x, ++j) {
            const int s = static_cast<int>(j % P.stages);
            (void)mbar_wait(&bars[s], static_cast<uint32_t>((j / P.stages) & 1));
        }
    }
}

// Per-device launch facts, queried once per process and device (a call otherwise spends more
// time in these queries than a small matrix takes on the GPU).
struct DeviceCache {
    std::atomic<int> sms{0};
    std::atomic<int> smem_set[4] = {{0}, {0}, {0}, {0}};  // largest dynamic smem opted in, per TT
    std::atomic<int> regs[4] = {{0}, {0}, {0}, {0}};      // registers per thread, per TT
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

int align16(int v) { return (v + 15) & ~15; }

// Shared-memory plan for a token tile of tt tokens; false if it does not fit.
bool make_plan(Params& P, int tt)
{
    const int k = P.k;
    P.rowbytes = (k / 32) * 18;
    const bool row16 = (P.rowbytes % 16) == 0;
    int R = 8;
    while (R > 1 && R * P.rowbytes > kChunkTarget) R >>= 1;
    if (!row16 && R < 2) R = 2;  // chunks must start on 16-byte boundaries
    P.rows = R;
    P.seg = kWarps / R;
    const int pairs = k / 64;
    P.pps = (pairs + P.seg - 1) / P.seg;
    P.nchunks = (P.n_out + R - 1) / R;
    P.act_q8_bytes = align16(k);
    P.off_d8 = tt * P.act_q8_bytes;
    P.off_bs = align16(P.off_d8 + tt * (k / 128) * 4);
    P.off_part = align16(P.off_bs + tt * (k / 32) * 2);
    P.off_bar = P.off_part + 2 * kWarps * tt * 8;
    P.off_stage = align16(P.off_bar + kMaxStages * 8);
    P.chunk_bytes = align16(R * P.rowbytes);
    const int room = kSmemMax - P.off_stage;
    int st = room / P.chunk_bytes;
    if (st > kMaxStages) st = kMaxStages;
    if (st < 2) return false;
    P.stages = st;
    return true;
}

template <int TT>
iqq_status launch_tt(Params& P, cudaStream_t st)
{
    constexpr int slot = TT == 1 ? 0 : (TT == 2 ? 1 : (TT == 4 ? 2 : 3));
    const int smem = P.off_stage + P.stages * P.chunk_bytes;
    auto kern = gemv_q4_0_q8_k128_kernel<TT>;
    const int dev = current_device();
    std::atomic<int>& opted = g_cache[dev].smem_set[slot];
    if (opted.load(std::memory_order_relaxed) < smem) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax) != cudaSuccess)
            return iqq::launch_status();
        opted.store(kSmemMax, std::memory_order_relaxed);
    }
    int regs = g_cache[dev].regs[slot].load(std::memory_order_relaxed);
    if (regs == 0) {
        cudaFuncAttributes fa{};
        if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return iqq::launch_status();
        regs = fa.numRegs > 0 ? fa.numRegs : 255;
        g_cache[dev].regs[slot].store(regs, std::memory_order_relaxed);
    }
    // resident CTAs per SM: 228 KB of shared memory (1 KB reserved per CTA) and 64 K
    // registers (allocated per warp in units of 256)
    int occ = kSmemPerSm / (smem + 1024);
    const int regs_cta = ((regs * 32 + 255) / 256) * 256 * kWarps;
    if (65536 / regs_cta < occ) occ = 65536 / regs_cta;
    if (occ < 1) occ = 1;
    if (occ > 4) occ = 4;
    const int64_t cap = static_cast<int64_t>(sm_count_gemv(dev)) * occ;
    const int gx = static_cast<int>(P.nchunks < cap ? P.nchunks : cap);
    const int64_t gy = (P.n_tok + TT - 1) / TT;
    if (gy > 65535) return IQQ_ERR_SHAPE;
    kern<<<dim3(gx, static_cast<unsigned>(gy)), kThreads, smem, st>>>(P);
    return iqq::launch_status();
}

}  // namespace

extern "C" iqq_status iqq_gemv_q4_0_q8_k128(const void* w_blocks, const void* a_blocks, float* y,
                                            int64_t n_out, int64_t k, int64_t n_tok, uint32_t* d_flags,
                                            void* stream)
{
    if (n_out < 0 || k < 0 || n_tok < 0 || k % 128 != 0 || k > IQQ_GEMV_MAX_K) return IQQ_ERR_SHAPE;
    if (!iqq::size_ok(n_out, k, 1) || !iqq::size_ok(n_tok, k, 2) || !iqq::size_ok(n_tok, n_out, 4))
        return IQQ_ERR_SHAPE;
    if (n_out == 0 || n_tok == 0) return IQQ_OK;
    if (y == nullptr) return IQQ_ERR_NULL;
    if (!iqq::aligned(y, 4) || !iqq::aligned(d_flags, 4)) return IQQ_ERR_ALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (k == 0) {
        // the dot product of empty vectors
        if (cudaMemsetAsync(y, 0, static_cast<size_t>(n_tok * n_out) * sizeof(float), st) != cudaSuccess)
            return iqq::launch_status();
        return IQQ_OK;
    }
    if (w_blocks == nullptr || a_blocks == nullptr) return IQQ_ERR_NULL;
    if (!iqq::aligned(w_blocks, 16) || !iqq::aligned(a_blocks, 4)) return IQQ_ERR_ALIGN;

    Params P{};
    P.w = static_cast<const uint8_t*>(w_blocks);
    P.a = static_cast<const uint8_t*>(a_blocks);
    P.y = y;
    P.flags = d_flags;
    P.n_out = n_out;
    P.n_tok = n_tok;
    P.k = static_cast<int>(k);
    int tt = n_tok >= 8 ? 8 : (n_tok >= 4 ? (n_tok == 4 ? 4 : 8) : (n_tok == 3 ? 4 : static_cast<int>(n_tok)));
    while (!make_plan(P, tt)) {
        if (tt == 1) return IQQ_ERR_SHAPE;
        tt >>= 1;
    }
    switch (tt) {
    case 1: return launch_tt<1>(P, st);
    case 2: return launch_tt<2>(P, st);
    case 4: return launch_tt<4>(P, st);
    default: return launch_tt<8>(P, st);
    }
}
