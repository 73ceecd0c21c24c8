// dequant_rmse.cu -- dequantization and the round-trip weighted RMSE of the 32-value
// block formats on sm_100a.
//
// Q4_0 blocks (written by qx_0_w.cu): bytes 0-1 binary16 d (LE), byte 2+i holds code
// i + 8 in its low nibble and code i+16 + 8 in its high nibble.  A value decodes to
// fp16(d) * (nibble - 8), exact in binary32.  Q5_0 / Q6_0 / Q8_0 layouts are in iqq.h.
//
// The weighted RMSE follows the quantize-stats statistics named on page
// "量化方法论实证：为什么 LQER/L²QER 难以改进 ik_llama.cpp 的 k-quants 与
// i-quants" (www.0539edu.com/news/4792009) §3.2 (rmse and maxerr), weighted by
// the imatrix entries qw: with e = x - y rounded to binary32 it adds
// {sum qw e^2, sum qw, sum e^2} in binary64 and takes max|e|.  The decoded y goes
// to memory only when asked for (the one-pass dequantization + round trip).
//
// All kernels are HBM bound.  Dequantization: one thread per 4 consecutive values (a
// "quad"); 8 quads make a block, so the 8 threads of a block share its bytes through L1
// and every warp writes 512 contiguous bytes per store.  Round trip: one thread per
// column quad over a run of rows (4 in flight), per-column binary64 sums.
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

#ifndef IQQ_DQ_UNROLL
#define IQQ_DQ_UNROLL 1  // independent quads in flight per thread (dequant)
#endif
#ifndef IQQ_DQ_CTAS
#define IQQ_DQ_CTAS 16   // CTAs per SM in the grid (dequant)
#endif
#ifndef IQQ_RMSE_UNROLL
#define IQQ_RMSE_UNROLL 4  // independent rows in flight per thread (weighted RMSE)
#endif
#ifndef IQQ_RMSE_CTAS
#define IQQ_RMSE_CTAS 4    // CTAs per SM in the grid (weighted RMSE; measured best of 4-32 with 1-8 rows in flight)
#endif
#ifndef IQQ_RMSE_PDL
#define IQQ_RMSE_PDL 1     // programmatic dependent launch between consecutive launches
#endif
#ifndef IQQ_RMSE_MIN_ROWS
#define IQQ_RMSE_MIN_ROWS 8  // rows per CTA at least (weighted RMSE)
#endif
constexpr int kUnroll = IQQ_DQ_UNROLL;
constexpr int kRowUnroll = IQQ_RMSE_UNROLL;

__global__ void __launch_bounds__(kThreads)
dequant_q4_0_kernel(const uint8_t* __restrict__ blocks, float4* __restrict__ y, int64_t nquads)
{
    // each iteration handles kUnroll quads spaced kThreads apart, so every warp-level
    // store stays contiguous; all loads of an iteration are issued before any store
    const int64_t step = static_cast<int64_t>(gridDim.x) * kThreads * kUnroll;
    for (int64_t t0 = static_cast<int64_t>(blockIdx.x) * kThreads * kUnroll + threadIdx.x; t0 < nquads;
         t0 += step) {
        Quad q[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t t = t0 + u * kThreads;
            if (t < nquads) q[u] = load_quad(blocks + (t >> 3) * IQQ_Q4_0_BLOCK_BYTES, static_cast<int>(t & 7));
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t t = t0 + u * kThreads;
            if (t < nquads) {
                float4 o;
                o.x = __fmul_rn(q[u].d, code_value(q[u].nib4, 0));
                o.y = __fmul_rn(q[u].d, code_value(q[u].nib4, 1));
                o.z = __fmul_rn(q[u].d, code_value(q[u].nib4, 2));
                o.w = __fmul_rn(q[u].d, code_value(q[u].nib4, 3));
                __stcs(y + t, o);  // streaming store: the output is not re-read here
            }
        }
    }
}

// Adds the squared errors of one row's quad to the per-column accumulators.
// Q5_0 / Q6_0 / Q8_0 (layouts in iqq.h): the four codes of quad qd (values 4qd..4qd+3).
template <int BITS>
__device__ __forceinline__ void load_quad_qx(const uint8_t* blk, int qd, float& d, int (&c)[4])
{
    const uint16_t* h = reinterpret_cast<const uint16_t*>(blk);
    d = __half2float(__ushort_as_half(__ldg(h)));
    if (BITS == 8) {
        const uint32_t b = static_cast<uint32_t>(__ldg(h + 1 + 2 * qd)) |
                           (static_cast<uint32_t>(__ldg(h + 2 + 2 * qd)) << 16);
#pragma unroll
        for (int k = 0; k < 4; ++k) c[k] = static_cast<int>(static_cast<int8_t>((b >> (8 * k)) & 0xffu));
        return;
    }
    constexpr int nmax = BITS == 5 ? 16 : 32;
    constexpr int hw = BITS == 5 ? 2 : 4;  // 16-bit words of high bits
    const int m = qd & 3;
    const uint32_t lo4 = static_cast<uint32_t>(__ldg(h + 1 + hw + 2 * m)) |
                         (static_cast<uint32_t>(__ldg(h + 2 + hw + 2 * m)) << 16);
    const uint32_t sel = qd < 4 ? lo4 : (lo4 >> 4);
    uint32_t hi;
    if (BITS == 5) {
        const uint32_t qh = static_cast<uint32_t>(__ldg(h + 1)) | (static_cast<uint32_t>(__ldg(h + 2)) << 16);
        hi = qh >> (4 * qd);  // bit k = high bit of value 4qd + k
    } else {
        hi = static_cast<uint32_t>(__ldg(h + 1 + (qd >> 1))) >> (8 * (qd & 1));  // 2 bits per value
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t low = (sel >> (8 * k)) & 0xfu;
        const uint32_t high = BITS == 5 ? ((hi >> k) & 1u) : ((hi >> (2 * k)) & 3u);
        c[k] = static_cast<int>(low | (high << 4)) - nmax;
    }
}

template <int BITS>
__global__ void __launch_bounds__(kThreads)
dequant_qx_kernel(const uint8_t* __restrict__ blocks, float4* __restrict__ y, int64_t nquads)
{
    constexpr int kBytes = BITS == 5 ? 22 : (BITS == 6 ? 26 : 34);
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; t < nquads; t += stride) {
        float d;
        int c[4];
        load_quad_qx<BITS>(blocks + (t >> 3) * kBytes, static_cast<int>(t & 7), d, c);
        float4 o;
        o.x = __fmul_rn(d, static_cast<float>(c[0]));
        o.y = __fmul_rn(d, static_cast<float>(c[1]));
        o.z = __fmul_rn(d, static_cast<float>(c[2]));
        o.w = __fmul_rn(d, static_cast<float>(c[3]));
        __stcs(y + t, o);
    }
}

// The scale and the four signed codes of quad qd of a block of any 32-value format.
struct QuadC {
    float d;
    int c[4];
};

template <int BITS>
__device__ __forceinline__ QuadC load_codes(const uint8_t* blk, int qd)
{
    QuadC q;
    if (BITS == 4) {
        const Quad n = load_quad(blk, qd);
        q.d = n.d;
#pragma unroll
        for (int k = 0; k < 4; ++k) q.c[k] = static_cast<int>((n.nib4 >> (4 * k)) & 0xfu) - 8;
    } else {
        load_quad_qx<BITS>(blk, qd, q.d, q.c);
    }
    return q;
}

template <int BITS>
__host__ __device__ constexpr int block_bytes() { return BITS == 4 ? 18 : (BITS == 5 ? 22 : (BITS == 6 ? 26 : 34)); }

// Adds the quad's round trip to the column sums; y (optional) receives its dequantized
// values y = fp16(d) * l.
__device__ __forceinline__ void rmse_quad(const float4 xv, const QuadC q, double (&col)[4], float& emax,
                                          float4* y)
{
    float yk[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) yk[k] = __fmul_rn(q.d, static_cast<float>(q.c[k]));
    if (y != nullptr) __stcs(y, make_float4(yk[0], yk[1], yk[2], yk[3]));
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float xk = k == 0 ? xv.x : k == 1 ? xv.y : k == 2 ? xv.z : xv.w;
        const float e = __fsub_rn(xk, yk[k]);
        emax = fmaxf(emax, fabsf(e));
        const double ed = static_cast<double>(e);
        col[k] = fma(ed, ed, col[k]);
    }
}

// One CTA's work: rows [by*rows_per_cta, ...) x column quad bx*kThreads + threadIdx.x.
// Per column the thread keeps sum_r e^2 (binary64) and multiplies by qw once per
// imatrix row, so qw is read and converted once per row segment, not per value.
template <int BITS, typename XT>
__device__ __forceinline__ void rmse_unit(const XT* __restrict__ x, const uint8_t* __restrict__ blocks,
                                          const float* __restrict__ qw, int64_t nrows, int64_t n_per_row,
                                          int64_t rows_per_qw, int rows_per_cta, int64_t bx, int64_t by,
                                          double* __restrict__ acc, float* __restrict__ y)
{
    const int64_t nq = n_per_row / 4;
    const int64_t nb = n_per_row / IQQ_Q4_0_BLOCK_VALUES;
    const int64_t cq = bx * kThreads + threadIdx.x;
    const int64_t r0 = by * rows_per_cta;
    const int64_t r1 = min(nrows, r0 + rows_per_cta);

    double sw = 0.0, sq = 0.0, se = 0.0;
    float emax = 0.0f;
    if (cq < nq) {
        const int64_t b = cq >> 3;
        const int qd = static_cast<int>(cq & 7);
        for (int64_t s0 = r0; s0 < r1;) {
            // a segment of rows sharing one imatrix row
            const int64_t qrow = rows_per_qw > 0 ? s0 / rows_per_qw : 0;
            const int64_t s1 = rows_per_qw > 0 ? min(r1, (qrow + 1) * rows_per_qw) : r1;
            double col[4] = {0.0, 0.0, 0.0, 0.0};
            int64_t r = s0;
            for (; r + kRowUnroll <= s1; r += kRowUnroll) {
                float4 xv[kRowUnroll];
                QuadC q[kRowUnroll];
#pragma unroll
                for (int u = 0; u < kRowUnroll; ++u) {
                    xv[u] = iqq::ld4_stream(x + (r + u) * n_per_row + 4 * cq);
                    q[u] = load_codes<BITS>(blocks + ((r + u) * nb + b) * block_bytes<BITS>(), qd);
                }
#pragma unroll
                for (int u = 0; u < kRowUnroll; ++u)
                    rmse_quad(xv[u], q[u], col, emax,
                              y != nullptr ? reinterpret_cast<float4*>(y + (r + u) * n_per_row) + cq : nullptr);
            }
            for (; r < s1; ++r) {
                const float4 xv = iqq::ld4_stream(x + r * n_per_row + 4 * cq);
                rmse_quad(xv, load_codes<BITS>(blocks + (r * nb + b) * block_bytes<BITS>(), qd), col, emax,
                          y != nullptr ? reinterpret_cast<float4*>(y + r * n_per_row) + cq : nullptr);
            }
            float4 w = make_float4(1.0f, 1.0f, 1.0f, 1.0f);
            if (qw != nullptr) w = __ldg(reinterpret_cast<const float4*>(qw + qrow * n_per_row) + cq);
            const double nr = static_cast<double>(s1 - s0);
            sw = fma(static_cast<double>(w.x), col[0], sw);
            sw = fma(static_cast<double>(w.y), col[1], sw);
            sw = fma(static_cast<double>(w.z), col[2], sw);
            sw = fma(static_cast<double>(w.w), col[3], sw);
            se += (col[0] + col[1]) + (col[2] + col[3]);
            sq = fma(static_cast<double>(w.x) + static_cast<double>(w.y) + static_cast<double>(w.z) +
                         static_cast<double>(w.w), nr, sq);
            s0 = s1;
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

// Programmatic dependent launch: the next kernel of the stream may be scheduled as this
// grid's CTAs retire; the grid waits for its predecessor (the blocks' writer, typically)
// before its first global access.  (No-ops without the launch attribute.)
__device__ __forceinline__ void pdl_prologue()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

template <int BITS, typename XT>
__global__ void __launch_bounds__(kThreads)
weighted_rmse_kernel(const XT* __restrict__ x, const uint8_t* __restrict__ blocks,
                     const float* __restrict__ qw, int64_t nrows, int64_t n_per_row,
                     int64_t rows_per_qw, int rows_per_cta, double* __restrict__ acc, float* __restrict__ y)
{
    pdl_prologue();
    rmse_unit<BITS, XT>(x, blocks, qw, nrows, n_per_row, rows_per_qw, rows_per_cta, blockIdx.x, blockIdx.y, acc,
                        y);
}

// Several Q4_0 tensors in one launch: their CTAs (column tiles x row groups, each tensor's
// as its single launch has them) laid end to end on a one-dimensional grid.
struct RmseProb {
    const float* x;
    const uint8_t* blocks;
    const float* qw;
    float* y;
    int64_t nrows, n_per_row, rows_per_qw;
    int rows_per_cta, gx;
};
constexpr int kRmseBatch = 48;
struct RmseBatch {
    RmseProb p[kRmseBatch];
    int64_t cum[kRmseBatch + 1];  // CTAs before tensor i
    int count;
};
static_assert(sizeof(RmseBatch) + 16 <= 4096, "kernel parameters");
static_assert(kRmseBatch <= 64, "the tensor lookup searches 64 entries");

__global__ void __launch_bounds__(kThreads)
weighted_rmse_batch_kernel(const __grid_constant__ RmseBatch B, double* __restrict__ acc)
{
    pdl_prologue();
    const int64_t b = blockIdx.x;
    // the tensor whose CTAs hold b: a fixed six-step binary search over cum (a linear scan
    // cost about 8% of the layer set's time, each CTA being only a few microseconds of work)
    int pi = 0;
#pragma unroll
    for (int s = 32; s > 0; s >>= 1)
        if (pi + s < B.count && B.cum[pi + s] <= b) pi += s;
    const RmseProb& P = B.p[pi];
    const int64_t u = b - B.cum[pi];
    rmse_unit<4, float>(P.x, P.blocks, P.qw, P.nrows, P.n_per_row, P.rows_per_qw, P.rows_per_cta, u % P.gx,
                        u / P.gx, acc, P.y);
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
    const int64_t need = (nquads + kThreads * kUnroll - 1) / (kThreads * kUnroll);
    const int64_t cap = static_cast<int64_t>(sm_count()) * IQQ_DQ_CTAS;
    const int grid = static_cast<int>(need < cap ? need : cap);
    dequant_q4_0_kernel<<<grid, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint8_t*>(blocks), reinterpret_cast<float4*>(y), nquads);
    return iqq::launch_status();
}

extern "C" iqq_status iqq_dequant_qx_0(int bits, const void* blocks, float* y, int64_t nrows,
                                       int64_t n_per_row, void* stream)
{
    if (bits != 4 && bits != 5 && bits != 6 && bits != 8) return IQQ_ERR_ARG;
    if (bits == 4) return iqq_dequant_q4_0(blocks, y, nrows, n_per_row, stream);
    if (!iqq::size_ok(nrows, n_per_row, 4)) return IQQ_ERR_SHAPE;
    if (n_per_row % IQQ_Q4_0_BLOCK_VALUES != 0) return IQQ_ERR_SHAPE;
    if (nrows == 0 || n_per_row == 0) return IQQ_OK;
    if (blocks == nullptr || y == nullptr) return IQQ_ERR_NULL;
    if (!iqq::aligned(blocks, 2) || !iqq::aligned(y, 16)) return IQQ_ERR_ALIGN;
    const int64_t nquads = nrows * n_per_row / 4;
    const int64_t need = (nquads + kThreads - 1) / kThreads;
    const int64_t cap = static_cast<int64_t>(sm_count()) * IQQ_DQ_CTAS;
    const int grid = static_cast<int>(need < cap ? need : cap);
    const uint8_t* bl = static_cast<const uint8_t*>(blocks);
    float4* yy = reinterpret_cast<float4*>(y);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (bits == 5) dequant_qx_kernel<5><<<grid, kThreads, 0, st>>>(bl, yy, nquads);
    else if (bits == 6) dequant_qx_kernel<6><<<grid, kThreads, 0, st>>>(bl, yy, nquads);
    else dequant_qx_kernel<8><<<grid, kThreads, 0, st>>>(bl, yy, nquads);
    return iqq::launch_status();
}

namespace {

// The weighted-RMSE grid of a tensor: gx column tiles of kThreads quads, gy row groups of rpc
// rows (IQQ_RMSE_CTAS CTAs per SM, at least IQQ_RMSE_MIN_ROWS rows per CTA).
void rmse_grid(int64_t nrows, int64_t n_per_row, int64_t& gx, int64_t& gy, int64_t& rpc)
{
    const int64_t nq = n_per_row / 4;
    gx = (nq + kThreads - 1) / kThreads;
    const int64_t target = static_cast<int64_t>(sm_count()) * IQQ_RMSE_CTAS;
    gy = target / gx;
    if (gy < 1) gy = 1;
    rpc = (nrows + gy - 1) / gy;
    if (rpc < IQQ_RMSE_MIN_ROWS) rpc = IQQ_RMSE_MIN_ROWS;
    gy = (nrows + rpc - 1) / rpc;
}

template <int BITS, typename XT = float>
iqq_status rmse_launch(const XT* x, const void* blocks, const float* qw, int64_t nrows, int64_t n_per_row,
                       int64_t rows_per_qw, double* d_acc, void* stream, float* y = nullptr)
{
    if (!iqq::size_ok(nrows, n_per_row, 4) || rows_per_qw < 0) return IQQ_ERR_SHAPE;
    if (n_per_row % IQQ_Q4_0_BLOCK_VALUES != 0) return IQQ_ERR_SHAPE;
    if (nrows == 0 || n_per_row == 0) return IQQ_OK;
    if (x == nullptr || blocks == nullptr || d_acc == nullptr) return IQQ_ERR_NULL;
    if (!iqq::aligned(x, 16) || !iqq::aligned(blocks, 2) || (qw && !iqq::aligned(qw, 16)) ||
        !iqq::aligned(d_acc, 8) || !iqq::aligned(y, 16))
        return IQQ_ERR_ALIGN;
    int64_t gx = 0, gy = 0, rpc = 0;
    rmse_grid(nrows, n_per_row, gx, gy, rpc);
    if (gx > 0x7fffffff || gy > 65535) return IQQ_ERR_SHAPE;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
    cfg.blockDim = dim3(kThreads);
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = IQQ_RMSE_PDL;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, weighted_rmse_kernel<BITS, XT>, x, static_cast<const uint8_t*>(blocks), qw, nrows,
                           n_per_row, rows_per_qw, static_cast<int>(rpc), d_acc, y) != cudaSuccess)
        return iqq::launch_status();
    return iqq::launch_status();
}

}  // namespace

extern "C" iqq_status iqq_weighted_rmse(const float* x, const void* blocks, const float* qw,
                                        int64_t nrows, int64_t n_per_row, int64_t rows_per_qw,
                                        double* d_acc, void* stream)
{
    return rmse_launch<4>(x, blocks, qw, nrows, n_per_row, rows_per_qw, d_acc, stream);
}

extern "C" iqq_status iqq_dequant_rmse_qx(int bits, const float* x, const void* blocks, const float* qw,
                                          int64_t nrows, int64_t n_per_row, int64_t rows_per_qw, float* y,
                                          double* d_acc, void* stream)
{
    if (y == nullptr && nrows > 0 && n_per_row > 0) return IQQ_ERR_NULL;
    switch (bits) {
    case 4: return rmse_launch<4>(x, blocks, qw, nrows, n_per_row, rows_per_qw, d_acc, stream, y);
    case 5: return rmse_launch<5>(x, blocks, qw, nrows, n_per_row, rows_per_qw, d_acc, stream, y);
    case 6: return rmse_launch<6>(x, blocks, qw, nrows, n_per_row, rows_per_qw, d_acc, stream, y);
    case 8: return rmse_launch<8>(x, blocks, qw, nrows, n_per_row, rows_per_qw, d_acc, stream, y);
    default: return IQQ_ERR_ARG;
    }
}

extern "C" iqq_status iqq_weighted_rmse_qx(int bits, const float* x, const void* blocks, const float* qw,
                                           int64_t nrows, int64_t n_per_row, int64_t rows_per_qw,
                                           double* d_acc, void* stream)
{
    switch (bits) {
    case 4: return rmse_launch<4>(x, blocks, qw, nrows, n_per_row, rows_per_qw, d_acc, stream);
    case 5: return rmse_launch<5>(x, blocks, qw, nrows, n_per_row, rows_per_qw, d_acc, stream);
    case 6: return rmse_launch<6>(x, blocks, qw, nrows, n_per_row, rows_per_qw, d_acc, stream);
    case 8: return rmse_launch<8>(x, blocks, qw, nrows, n_per_row, rows_per_qw, d_acc, stream);
    default: return IQQ_ERR_ARG;
    }
}

extern "C" iqq_status iqq_dequant_rmse_qx_bf16(int bits, const void* x, const void* blocks, const float* qw,
                                               int64_t nrows, int64_t n_per_row, int64_t rows_per_qw, float* y,
                                               double* d_acc, void* stream)
{
    if (y == nullptr && nrows > 0 && n_per_row > 0) return IQQ_ERR_NULL;
    const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
    switch (bits) {
    case 4: return rmse_launch<4>(xb, blocks, qw, nrows, n_per_row, rows_per_qw, d_acc, stream, y);
    case 5: return rmse_launch<5>(xb, blocks, qw, nrows, n_per_row, rows_per_qw, d_acc, stream, y);
    case 6: return rmse_launch<6>(xb, blocks, qw, nrows, n_per_row, rows_per_qw, d_acc, stream, y);
    case 8: return rmse_launch<8>(xb, blocks, qw, nrows, n_per_row, rows_per_qw, d_acc, stream, y);
    default: return IQQ_ERR_ARG;
    }
}

namespace {

iqq_status rmse_batch_launch(const RmseBatch& B, double* d_acc, void* stream)
{
    const int64_t ctas = B.cum[B.count];
    if (ctas == 0) return IQQ_OK;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(ctas));
    cfg.blockDim = dim3(kThreads);
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = IQQ_RMSE_PDL;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, weighted_rmse_batch_kernel, B, d_acc) != cudaSuccess) return iqq::launch_status();
    return iqq::launch_status();
}

}  // namespace

extern "C" iqq_status iqq_dequant_rmse_q4_0_batch(const iqq_dequant_rmse_problem* problems, int64_t count,
                                                  double* d_acc, void* stream)
{
    if (count < 0) return IQQ_ERR_SHAPE;
    if (count > 0 && problems == nullptr) return IQQ_ERR_NULL;
    if (!iqq::aligned(d_acc, 8)) return IQQ_ERR_ALIGN;
    for (int64_t i = 0; i < count; ++i) {
        const iqq_dequant_rmse_problem& q = problems[i];
        if (!iqq::size_ok(q.nrows, q.n_per_row, 4) || q.rows_per_qw < 0) return IQQ_ERR_SHAPE;
        if (q.n_per_row % IQQ_Q4_0_BLOCK_VALUES != 0) return IQQ_ERR_SHAPE;
        if (q.nrows == 0 || q.n_per_row == 0) continue;
        if (q.x == nullptr || q.blocks == nullptr || d_acc == nullptr) return IQQ_ERR_NULL;
        if (!iqq::aligned(q.x, 16) || !iqq::aligned(q.blocks, 2) || (q.qw && !iqq::aligned(q.qw, 16)) ||
            !iqq::aligned(q.y, 16))
            return IQQ_ERR_ALIGN;
        int64_t gx = 0, gy = 0, rpc = 0;
        rmse_grid(q.nrows, q.n_per_row, gx, gy, rpc);
        if (gx * gy > 0x7fffffff / kRmseBatch || rpc > 0x7fffffff) return IQQ_ERR_SHAPE;
    }
    RmseBatch B;
    B.count = 0;
    B.cum[0] = 0;
    for (int64_t i = 0; i < count; ++i) {
        const iqq_dequant_rmse_problem& q = problems[i];
        if (q.nrows == 0 || q.n_per_row == 0) continue;
        int64_t gx = 0, gy = 0, rpc = 0;
        rmse_grid(q.nrows, q.n_per_row, gx, gy, rpc);
        B.p[B.count] = RmseProb{q.x, static_cast<const uint8_t*>(q.blocks), q.qw, q.y, q.nrows, q.n_per_row,
                                q.rows_per_qw, static_cast<int>(rpc), static_cast<int>(gx)};
        B.cum[B.count + 1] = B.cum[B.count] + gx * gy;
        if (++B.count == kRmseBatch) {
            const iqq_status st = rmse_batch_launch(B, d_acc, stream);
            if (st != IQQ_OK) return st;
            B.count = 0;
        }
    }
    if (B.count == 0) return IQQ_OK;
    return rmse_batch_launch(B, d_acc, stream);
}
