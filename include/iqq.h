/*
 * iqq.h -- C ABI of the B200 (sm_100a) library for importance-matrix-weighted
 * Q4_0 weight quantization, Q8_K_128 activation quantization, Q4_0
 * dequantization and the round-trip weighted RMSE.
 *
 * Sources (page title, address, section):
 *  [W]   "ik_llama.cpp 量化权重之谜：weight[j] = qw[j] * sqrtf(sigma2 +
 *        xb[j]*xb[j])的由来与原理" (www.dpshk.com/news/4810665)
 *  [Q8]  "ik_llama.cpp 量化精度修复实录：用 Q8_K_128 替代 Q8_1 根治
 *        IQ1_S_R4 / IQ1_M_R4 的 fp16 溢出" (www.hnwysp.cn/news/39281)
 *  [SVD] "量化方法论实证：为什么 LQER/L²QER 难以改进 ik_llama.cpp 的
 *        k-quants 与 i-quants" (www.0539edu.com/news/4792009)
 *
 * Conventions shared by every entry point:
 *  - Memory: every data pointer is DEVICE memory owned by the caller (for
 *    example a torch CUDA tensor's data_ptr()).  The library never allocates,
 *    frees or keeps a pointer after the call returns.
 *  - Streams: `stream` is a cudaStream_t passed as void* (NULL = the legacy
 *    default stream).  Work is enqueued asynchronously on it; the call never
 *    synchronizes.  Results and flags are valid after the caller synchronizes
 *    the stream.
 *  - Errors: the return value reports host-side validation and launch
 *    failures only.  Validation happens before any CUDA call, so a rejected
 *    call enqueues nothing.  IQQ_ERR_CUDA means the launch itself failed;
 *    iqq_last_cuda_error() returns the cudaError_t value.
 *  - Data problems found on the device (NaN/Inf input, negative importance,
 *    a scale beyond binary16) are ORed as IQQ_FLAG_* bits into the optional
 *    caller-owned device word *d_flags (may be NULL).  Nothing on the device
 *    traps or asserts.  The only waits on the device are the GEMV kernel's
 *    waits for its own bulk copies: each is bounded (about 2 s), and on expiry
 *    the kernel sets IQQ_FLAG_WAIT_TIMEOUT, drains its copies and returns.
 *  - Empty input (nrows == 0 or n_per_row == 0) is valid and enqueues
 *    nothing; pointers may then be NULL.
 *  - Layouts are row-major: element (r, j) of an [nrows, n_per_row] float
 *    matrix is at index r*n_per_row + j, and block b of row r is the
 *    (r*nb + b)-th block of the output, nb = n_per_row / block values.
 */
#ifndef IQQ_H
#define IQQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    IQQ_OK = 0,
    IQQ_ERR_NULL = 1,  /* a required pointer is NULL                              */
    IQQ_ERR_SHAPE = 2, /* negative size, n_per_row not a multiple of the block,   */
                       /* or a size whose byte count overflows int64              */
    IQQ_ERR_ALIGN = 3, /* a pointer lacks the alignment its argument states       */
    IQQ_ERR_CUDA = 4,  /* the kernel launch failed (see iqq_last_cuda_error)      */
    IQQ_ERR_ARG = 5    /* an enumerated argument is out of range (weight_mode 0..5) */
} iqq_status;

/* Device-side flag bits, ORed into *d_flags. */
#define IQQ_FLAG_NONFINITE_INPUT 1u /* NaN or Inf in x (or in qw)                    */
#define IQQ_FLAG_NEG_QW 2u          /* an importance qw < 0                          */
#define IQQ_FLAG_SCALE_OVERFLOW 4u  /* a finite Q4_0 scale rounded to +-Inf in fp16 */
#define IQQ_FLAG_WAIT_TIMEOUT 8u    /* a staged copy did not arrive within the bounded
                                       wait (about 2 s); the results are unspecified  */

/* Block formats. */
#define IQQ_Q4_0_BLOCK_VALUES 32
#define IQQ_Q4_0_BLOCK_BYTES 18
#define IQQ_Q8_K128_BLOCK_VALUES 128
#define IQQ_Q8_K128_BLOCK_BYTES 140

/*
 * iqq_quantize_q4_0_w -- imatrix-weighted Q4_0 quantization, [W] §一
 * (quantize_row_q4_0_impl with make_qx_quants(QK4_0, 8, ...)).
 *
 * Per row r: sigma2 = sum_j x[r,j]^2 / n_per_row (binary64 sum, rounded to
 * binary32).  Per 32-value block: weight[j] = qw[j]*sqrtf(sigma2 + x[j]^2)
 * (weight_mode 0) or qw[j] (weight_mode 1); a weighted least-squares scale
 * search over iscale = -(8 + 0.1k)/xmax, k = -9..9, codes clamp(rint(iscale*x),
 * -8, 7), best sumlx^2/suml2 (ties to the lowest k); at most 5 greedy passes
 * that move one code by +-1 in the direction of g = d*w*(x - d*l) when the
 * weighted error drops; d = sumlx/suml2 rounded to binary16.
 *
 *  x          [nrows, n_per_row] float32, 16-byte aligned.
 *  qw         imatrix rows, float32, 16-byte aligned, or NULL (qw = 1).  Row r
 *             uses qw + (rows_per_qw > 0 ? r / rows_per_qw : 0) * n_per_row, so qw
 *             must hold (rows_per_qw > 0 ? ceil(nrows / rows_per_qw) : 1) * n_per_row
 *             values on the device of x (the library cannot check this; the Python
 *             binding does).
 *  out        nrows * n_per_row / 32 blocks of 18 bytes, 2-byte aligned:
 *             bytes 0-1 binary16 d (little endian), byte 2+i holds
 *             (l[i]+8) | (l[i+16]+8) << 4 for i = 0..15.
 *  nrows, n_per_row   n_per_row % 32 == 0, both >= 0.
 *  rows_per_qw        >= 0; 0 = one imatrix row shared by all rows.
 *  weight_mode        0 = qw*sqrt(sigma2 + x^2), 1 = qw, and the magnitude forms
 *                     [W] §二 lists as tried before imatrix existed, times qw:
 *                     2 = qw*x^2, 3 = qw*|x|, 4 = qw*(sigma2 + x^2),
 *                     5 = qw*(sqrt(sigma2) + |x|)  (qw = NULL: the pure forms).
 *  d_flags    optional device uint32 (4-byte aligned) receiving IQQ_FLAG_*.
 *  stream     cudaStream_t.
 *
 * Invalid input is flagged, not trapped: a row whose x holds NaN/Inf, or a block
 * whose qw holds NaN/Inf or a negative value, gets unspecified bytes; all other
 * rows and blocks are exact.
 */
iqq_status iqq_quantize_q4_0_w(const float* x, const float* qw, void* out, int64_t nrows,
                               int64_t n_per_row, int64_t rows_per_qw, int weight_mode,
                               uint32_t* d_flags, void* stream);

/*
 * iqq_quantize_q4_0_w_direct -- iqq_quantize_q4_0_w computed by the direct sweep: every
 * block evaluates all 19 candidates' sequential sums (the definition above, step by step).
 * iqq_quantize_q4_0_w reaches the same winner by placing each code step between candidates
 * and computing exact sums only for the candidates an error bound cannot exclude; the two
 * write identical bytes and flags.  Kept to cross-check that path on large inputs and as
 * the reference point of its speed.  Arguments and errors as for iqq_quantize_q4_0_w.
 */
iqq_status iqq_quantize_q4_0_w_direct(const float* x, const float* qw, void* out, int64_t nrows,
                                      int64_t n_per_row, int64_t rows_per_qw, int weight_mode,
                                      uint32_t* d_flags, void* stream);

/*
 * iqq_quantize_q4_0_w_batch -- iqq_quantize_q4_0_w ([W] §一) for several tensors in few
 * launches.  The pages have no counterpart: this is a launch form, not an operation.  A
 * launch lays the 32-block tiles of up to 64 tensors end to end and spreads them evenly over
 * one wave of CTAs, so the start and drain of a launch (about 13 us on B200, against about
 * 230 us of work for a 4096x4096 tensor) are paid once per 64 tensors, not once per tensor.
 * Every tensor's blocks and flags are those of iqq_quantize_q4_0_w on it, byte for byte.
 *  problems   host array of `count` descriptions (read before the call returns): x, qw, out,
 *             nrows, n_per_row and rows_per_qw of each tensor, as for iqq_quantize_q4_0_w
 *             (device pointers; tensors may share qw; outputs must not overlap).
 *  weight_mode, fudge  as for iqq_quantize_qx_0_w_ex, shared by all the tensors.
 *  d_flags    one optional flag word for all the tensors.
 * Errors: those of iqq_quantize_q4_0_w for any tensor, and a row of 2^22 blocks or more
 * (IQQ_ERR_SHAPE; iqq_quantize_q4_0_w serves those), all checked before anything is
 * enqueued; count < 0: IQQ_ERR_SHAPE; problems NULL with count > 0: IQQ_ERR_NULL.
 */
typedef struct iqq_q4_0_problem {
    const float* x;
    const float* qw;
    void* out;
    int64_t nrows;
    int64_t n_per_row;
    int64_t rows_per_qw;
} iqq_q4_0_problem;
iqq_status iqq_quantize_q4_0_w_batch(const iqq_q4_0_problem* problems, int64_t count, int weight_mode,
                                     float fudge, uint32_t* d_flags, void* stream);

/*
 * iqq_quantize_qx_0_w -- the same weighted search for the other 32-value formats
 * of the family ([W] §一: the weighting appears in quantize_row_q5_0_impl,
 * quantize_row_q6_0_impl, ...): bits = 4 (Q4_0, exactly iqq_quantize_q4_0_w),
 * 5 (Q5_0), 6 (Q6_0) or 8 (Q8_0); nmax = 8, 16, 32, 128, codes in
 * [-nmax, nmax-1], candidates iscale = -c_k/xmax with c_k = (float)(nmax*(80+k))/80.
 * Other arguments as for iqq_quantize_q4_0_w; out holds 18/22/26/34-byte blocks
 * (2-byte aligned).  With n = l + nmax the biased code:
 *   Q5_0 (22 B): d16 | qh u32 LE, bit j = (n_j >> 4) & 1 | qs[16], qs[i] = (n_i & 15) | (n_{i+16} & 15) << 4
 *   Q6_0 (26 B): d16 | qh u64 LE, bits 2j..2j+1 = n_j >> 4 | qs[16] as for Q5_0
 *   Q8_0 (34 B): d16 | int8 l[32]
 * bits outside {4, 5, 6, 8} return IQQ_ERR_ARG.
 */
#define IQQ_Q5_0_BLOCK_BYTES 22
#define IQQ_Q6_0_BLOCK_BYTES 26
#define IQQ_Q8_0_BLOCK_BYTES 34
iqq_status iqq_quantize_qx_0_w(int bits, const float* x, const float* qw, void* out, int64_t nrows,
                               int64_t n_per_row, int64_t rows_per_qw, int weight_mode,
                               uint32_t* d_flags, void* stream);

/*
 * iqq_quantize_qx_0_w_ws -- iqq_quantize_qx_0_w with a caller-owned device workspace for
 * wide rows.  A row spanning at least 4 CTAs of the quantizer (n_per_row > 12288) has its
 * sigma2 computed once by a separate per-row pass into the workspace (nrows floats),
 * instead of once per CTA of the row; the binary64 sum of exact squares and its rounding are
 * those of iqq_quantize_qx_0_w (only the summation order can differ, as there), and the
 * pass reports IQQ_FLAG_NONFINITE_INPUT.  Narrower rows need no workspace and take the
 * fused path.
 *  workspace        device memory of at least iqq_quantize_qx_0_w_workspace_bytes(nrows,
 *                   n_per_row) bytes, 16-byte aligned; may be NULL when that size is 0.
 *                   Overwritten; free for reuse once the stream has passed the call.
 *  workspace_bytes  its size.  Too small: IQQ_ERR_SHAPE; NULL when needed: IQQ_ERR_NULL.
 * Other arguments and errors as for iqq_quantize_qx_0_w.
 */
size_t iqq_quantize_qx_0_w_workspace_bytes(int64_t nrows, int64_t n_per_row);
iqq_status iqq_quantize_qx_0_w_ws(int bits, const float* x, const float* qw, void* out, int64_t nrows,
                                  int64_t n_per_row, int64_t rows_per_qw, int weight_mode, void* workspace,
                                  size_t workspace_bytes, uint32_t* d_flags, void* stream);

/*
 * iqq_quantize_qx_0_w_ex -- the general form of the weighted quantizers: any 32-value
 * format, an optional workspace, an optional dequantized output and an optional
 * round-trip error accumulator (quantization, dequantization and the weighted RMSE of a
 * tensor in one pass over it).
 *  fudge            the importance's correction factor ([W] §四 names a fudge factor that
 *                   corrects the approximate Hessian, without its values): it scales the
 *                   sigma2 term of weight modes 0, 4 and 5, sigma2 -> fl(fudge * sigma2);
 *                   1 changes nothing.  Finite and >= 0, else IQQ_ERR_ARG.
 *  workspace, workspace_bytes  as for iqq_quantize_qx_0_w_ws, but optional: with NULL the
 *                   per-CTA row reduction is used for every width.
 *  y_out            optional device float32 [nrows, n_per_row] (16-byte aligned): the
 *                   kernel that writes the blocks also writes their dequantized values,
 *                   bit for bit those of iqq_dequant_qx_0.
 *  d_acc            optional device double[4] (8-byte aligned), caller-owned and zeroed by
 *                   the caller.  When given, the kernel that writes the blocks also adds
 *                   the round trip of every block written, exactly as iqq_weighted_rmse
 *                   does over them (e = x - fp16(d) * l in binary32; {sum qw e^2, sum qw,
 *                   sum e^2} in binary64, max |e|), so the tensor is read once for both
 *                   ([SVD] §3.2 rmse / maxerr, weighted by the imatrix).
 * Other arguments and errors as for iqq_quantize_qx_0_w.
 */
iqq_status iqq_quantize_qx_0_w_ex(int bits, const float* x, const float* qw, void* out, int64_t nrows,
                                  int64_t n_per_row, int64_t rows_per_qw, int weight_mode, float fudge,
                                  void* workspace, size_t workspace_bytes, float* y_out, double* d_acc,
                                  uint32_t* d_flags, void* stream);

/*
 * iqq_quantize_qx_0_w_bf16 -- iqq_quantize_qx_0_w for weights stored as bf16 (the form a
 * checkpoint usually holds).  The quantization routine of [W] §一 takes binary32 values;
 * each bf16 is widened to binary32 exactly in the kernel (its bits are the binary32's high
 * half), so the blocks and flags are bit for bit those of iqq_quantize_qx_0_w (and _ws) on
 * the widened tensor, from half the bytes of x.
 *  x          [nrows, n_per_row] bf16, 16-byte aligned.
 *  workspace, workspace_bytes  optional, as for iqq_quantize_qx_0_w_ex.
 * Other arguments and errors as for iqq_quantize_qx_0_w.
 */
iqq_status iqq_quantize_qx_0_w_bf16(int bits, const void* x, const float* qw, void* out, int64_t nrows,
                                    int64_t n_per_row, int64_t rows_per_qw, int weight_mode, void* workspace,
                                    size_t workspace_bytes, uint32_t* d_flags, void* stream);

/*
 * iqq_quantize_qx_0_w_static -- iqq_quantize_qx_0_w_ws without a caller workspace: the
 * per-row sigma2 of wide rows goes to a library-owned device array of IQQ_STATIC_WS_ROWS
 * floats (a file-scope __device__ variable, one per device; nothing is allocated), and
 * tensors with more rows are processed in batches of that many rows.  Results are
 * identical to iqq_quantize_qx_0_w_ws.  The array is shared by every call on a device, so
 * calls must be ordered (one stream, or synchronized); concurrent calls on different
 * streams of one device are not supported.  Arguments and errors as iqq_quantize_qx_0_w.
 */
#define IQQ_STATIC_WS_ROWS 16384
iqq_status iqq_quantize_qx_0_w_static(int bits, const float* x, const float* qw, void* out, int64_t nrows,
                                      int64_t n_per_row, int64_t rows_per_qw, int weight_mode,
                                      uint32_t* d_flags, void* stream);

/*
 * iqq_quantize_q8_k128 -- Q8_K_128 activation quantization, [Q8] 修复方案:
 * 128-value blocks with a binary32 scale, int8 codes and one int16 sum of the
 * codes per 32 values that is not multiplied by d, so no fp16 quantity can
 * overflow.  amax = max|x|, d = amax/127, id = amax > 0 ? 127/amax : 0,
 * q = clamp(rint(x*id), -127, 127) (a NaN product gives 0),
 * bsums[i] = sum of q over values 32i..32i+31.
 *
 *  x          [nrows, n_per_row] float32, 16-byte aligned.
 *  out        nrows * n_per_row / 128 blocks of 140 bytes, 4-byte aligned:
 *             float d | int8 qs[128] | int16 bsums[4], little endian.
 *  n_per_row  must be a multiple of 128 (the ne00 % 128 == 0 rule of [Q8]).
 *  d_flags    optional; receives IQQ_FLAG_NONFINITE_INPUT.
 */
iqq_status iqq_quantize_q8_k128(const float* x, void* out, int64_t nrows, int64_t n_per_row,
                                uint32_t* d_flags, void* stream);

/*
 * iqq_quantize_q8_1 -- Q8_1 activation quantization, the format [Q8]
 * 修复前的数值隐患 describes and Q8_K_128 replaces: per 32 values a binary16
 * d = amax/127 and a binary16 s = d*sum(q), int8 codes as for Q8_K_128
 * (q = clamp(rint(x*id), -127, 127), id = amax > 0 ? 127/amax : 0).  s can
 * overflow binary16 although d fits; the number of such blocks (stored s
 * +-Inf, d finite) is added to *d_overflow.  Provided to measure that failure
 * next to Q8_K_128.
 *
 *  x          [nrows, n_per_row] float32, 16-byte aligned.
 *  out        nrows * n_per_row / 32 blocks of 36 bytes, 4-byte aligned:
 *             half d | half s | int8 qs[32], little endian.
 *  n_per_row  a multiple of 32.
 *  d_overflow optional device uint64 (8-byte aligned); the count is ADDED.
 *  d_flags    optional; receives IQQ_FLAG_NONFINITE_INPUT.
 */
#define IQQ_Q8_1_BLOCK_VALUES 32
#define IQQ_Q8_1_BLOCK_BYTES 36
iqq_status iqq_quantize_q8_1(const float* x, void* out, int64_t nrows, int64_t n_per_row,
                             unsigned long long* d_overflow, uint32_t* d_flags, void* stream);

/*
 * iqq_dequant_q4_0 -- y[r, 32b + i] = fp16(d) * (nibble_i - 8) for the Q4_0
 * blocks written by iqq_quantize_q4_0_w (the inverse map of [W] §一's
 * packing; the product is exact in binary32).
 *
 *  blocks     nrows * n_per_row / 32 blocks of 18 bytes, 2-byte aligned.
 *  y          [nrows, n_per_row] float32 output, 16-byte aligned.
 */
iqq_status iqq_dequant_q4_0(const void* blocks, float* y, int64_t nrows, int64_t n_per_row,
                            void* stream);

/*
 * iqq_dequant_qx_0 -- y = fp16(d) * l for blocks written by iqq_quantize_qx_0_w with
 * the same bits (4, 5, 6, 8); exact in binary32.  blocks 2-byte aligned, y 16-byte
 * aligned.
 */
iqq_status iqq_dequant_qx_0(int bits, const void* blocks, float* y, int64_t nrows, int64_t n_per_row,
                            void* stream);

/*
 * iqq_weighted_rmse_qx -- iqq_weighted_rmse for blocks of any of the 32-value formats
 * written by iqq_quantize_qx_0_w (bits 4, 5, 6, 8; y = fp16(d) * code as
 * iqq_dequant_qx_0).  Same arguments, accumulator and errors; bits outside {4, 5, 6, 8}
 * return IQQ_ERR_ARG.
 */
iqq_status iqq_weighted_rmse_qx(int bits, const float* x, const void* blocks, const float* qw, int64_t nrows,
                                int64_t n_per_row, int64_t rows_per_qw, double* d_acc, void* stream);

/*
 * iqq_dequant_rmse_qx -- iqq_dequant_qx_0 and iqq_weighted_rmse_qx in one pass: reads the
 * blocks and x once, writes y = fp16(d) * l (bit for bit iqq_dequant_qx_0's output) and
 * adds the round trip to d_acc exactly as iqq_weighted_rmse_qx does.  y is float32
 * [nrows, n_per_row], 16-byte aligned, required (NULL: IQQ_ERR_NULL); other arguments and
 * errors as for iqq_weighted_rmse_qx.
 */
iqq_status iqq_dequant_rmse_qx(int bits, const float* x, const void* blocks, const float* qw, int64_t nrows,
                               int64_t n_per_row, int64_t rows_per_qw, float* y, double* d_acc, void* stream);

/*
 * iqq_dequant_rmse_q4_0_batch -- iqq_dequant_rmse_qx (bits 4) on up to any number of
 * float32 tensors, 48 per launch: each tensor's CTAs are those of its own call, laid end to
 * end on one grid, so the start and drain of a launch are paid once per 48 tensors.  Each
 * tensor's y is bit for bit that of its own call, and all the tensors add to the one
 * accumulator as their calls would in turn (the binary64 sums and so d_acc[0..2] can differ
 * in the last bits with the order of the atomic adds, as between two runs of one call;
 * d_acc[3], a maximum, is the same).
 *  problems   host array of `count` descriptions (read before the call returns): x, blocks,
 *             qw, y, nrows, n_per_row and rows_per_qw of each tensor, as for
 *             iqq_dequant_rmse_qx (device pointers; tensors may share qw; the y must not
 *             overlap one another); y NULL adds only the round trip (iqq_weighted_rmse).
 *  d_acc      double[4] accumulator shared by all the tensors, as for iqq_weighted_rmse.
 * Errors: those of iqq_dequant_rmse_qx for any tensor (y excepted), and a tensor of 2^31/48
 * CTAs or more (IQQ_ERR_SHAPE), all checked before anything is enqueued; count < 0:
 * IQQ_ERR_SHAPE; problems NULL with count > 0: IQQ_ERR_NULL.
 */
typedef struct iqq_dequant_rmse_problem {
    const float* x;
    const void* blocks;
    const float* qw;
    float* y;
    int64_t nrows;
    int64_t n_per_row;
    int64_t rows_per_qw;
} iqq_dequant_rmse_problem;
iqq_status iqq_dequant_rmse_q4_0_batch(const iqq_dequant_rmse_problem* problems, int64_t count, double* d_acc,
                                       void* stream);

/*
 * iqq_dequant_rmse_qx_bf16 -- iqq_dequant_rmse_qx against x stored as bf16 [nrows,
 * n_per_row] (16-byte aligned), widened exactly to binary32: y and the accumulator are bit
 * for bit those of iqq_dequant_rmse_qx on the widened tensor.  Other arguments and errors
 * as for iqq_dequant_rmse_qx.
 */
iqq_status iqq_dequant_rmse_qx_bf16(int bits, const void* x, const void* blocks, const float* qw, int64_t nrows,
                                    int64_t n_per_row, int64_t rows_per_qw, float* y, double* d_acc,
                                    void* stream);

/*
 * iqq_gemv_q4_0_q8_k128 -- y[t][r] = dot(dequant(W row r), dequant(A row t)): Q4_0 weight
 * rows times Q8_K_128 activation rows (a matrix-vector product per token).  [Q8]
 * 修复前的数值隐患 describes the consumer of the activation blocks: unsigned weight codes
 * times int8 activation codes, corrected by the block sum; 修复方案 makes that sum an
 * unscaled int16 per 32 values, so the correction is exact.  Here, per 32-value block,
 * isum = sum(u*q) - 8*bsum with u = l + 8 the stored nibble, and the block's term
 * d8 * d4 * isum is formed exactly in binary64; the K/32 terms of a row are summed in
 * binary64 in a fixed order and rounded once to binary32.  The result is reproducible and
 * within (K/32 + 16) * 2^-53 * sum|terms| of the exact dot product before that rounding.
 *
 *  w_blocks  n_out rows of k/32 Q4_0 blocks (18 B, layout as iqq_quantize_q4_0_w),
 *            16-byte aligned.
 *  a_blocks  n_tok rows of k/128 Q8_K_128 blocks (140 B, layout as
 *            iqq_quantize_q8_k128), 4-byte aligned.
 *  y         float32 [n_tok][n_out], 4-byte aligned; fully overwritten.
 *  k         values per row: a multiple of 128, at most IQQ_GEMV_MAX_K.  k == 0 writes
 *            zeros (the empty dot product).
 *  d_flags   optional; receives IQQ_FLAG_WAIT_TIMEOUT.
 * Tokens are processed in tiles of up to 8 (fewer when a wide row's activations would not
 * fit in shared memory); a token count needing more than 65535 tiles returns
 * IQQ_ERR_SHAPE.  Blocks whose binary16 scale is not finite give unspecified values in the
 * rows that use them (iqq_quantize_q4_0_w flags such scales).
 */
#define IQQ_GEMV_MAX_K 65536
iqq_status iqq_gemv_q4_0_q8_k128(const void* w_blocks, const void* a_blocks, float* y, int64_t n_out,
                                 int64_t k, int64_t n_tok, uint32_t* d_flags, void* stream);

/*
 * iqq_gemv_q4_0_q8_k128_batch -- iqq_gemv_q4_0_q8_k128 for a list of independent problems
 * (for example every weight matrix of a model for one decode step) in as few launches as
 * possible: up to 64 problems per launch, one wave of CTAs each taking an equal share of
 * the launch's weight bytes (rows of one problem or of several).  Each problem's result is
 * exactly that of iqq_gemv_q4_0_q8_k128 (the per-row summation order does not depend on
 * the launch).
 *  problems  HOST array of count descriptors, read during the call and not kept; every
 *            field as for iqq_gemv_q4_0_q8_k128.  The outputs y must not overlap any
 *            problem's inputs or other outputs.
 * All problems are checked before anything is enqueued; the first failing check's status
 * is returned.
 */
typedef struct iqq_gemv_problem {
    const void* w_blocks;
    const void* a_blocks;
    float* y;
    int64_t n_out;
    int64_t k;
    int64_t n_tok;
} iqq_gemv_problem;
iqq_status iqq_gemv_q4_0_q8_k128_batch(const iqq_gemv_problem* problems, int64_t count, uint32_t* d_flags,
                                       void* stream);

/*
 * iqq_weighted_rmse -- round-trip error of Q4_0 blocks against the source,
 * weighted by the imatrix ([SVD] §3.2 rmse and maxerr; the weights are qw
 * alone, not the quantizer weights).  With e = x - dequant(blocks) rounded to
 * binary32, ADDS to the caller's binary64 accumulator
 *     d_acc[0] += sum qw*e^2,  d_acc[1] += sum qw,  d_acc[2] += sum e^2,
 *     d_acc[3]  = max(d_acc[3], max |e|).
 * The caller zeroes d_acc once and may accumulate over several tensors:
 * wrmse = sqrt(d_acc[0]/d_acc[1]), rmse = sqrt(d_acc[2]/count).  The sums use
 * binary64 atomics, so their rounding order is not fixed (relative
 * differences of order 1e-15 between runs).
 *
 *  x          [nrows, n_per_row] float32, 16-byte aligned.
 *  blocks     Q4_0 blocks of x, 2-byte aligned.
 *  qw         imatrix rows as in iqq_quantize_q4_0_w (NULL = 1), 16-byte aligned.
 *  d_acc      device double[4], 8-byte aligned.
 */
iqq_status iqq_weighted_rmse(const float* x, const void* blocks, const float* qw, int64_t nrows,
                             int64_t n_per_row, int64_t rows_per_qw, double* d_acc,
                             void* stream);

/* Static description of a status code (never NULL). */
const char* iqq_status_string(iqq_status status);

/* The cudaError_t of the most recent IQQ_ERR_CUDA on this host thread (0 if none). */
int iqq_last_cuda_error(void);

/* Library build string. */
const char* iqq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* IQQ_H */
