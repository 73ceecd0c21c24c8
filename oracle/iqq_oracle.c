/*
 * iqq_oracle.c -- plain, slow, single-threaded CPU oracle for the
 * imatrix-weighted Q4_0 quantizer, the Q8_K_128 activation quantizer,
 * Q4_0 dequantization and the round-trip weighted RMSE.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline / reference leg may load this file.  The CUDA
 * library never includes, links or calls it, and it includes nothing from
 * the CUDA library: the two share no code, header, table or constant.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math (see build.py).
 * Contraction is off, so every a*b+c below is two roundings unless it is an
 * explicit fmaf() call.  All float arithmetic is IEEE binary32 with
 * round-to-nearest-even (x86-64 SSE), sqrtf and '/' are correctly rounded,
 * rintf rounds half to even in the default rounding mode.
 *
 * Sources (page title, address, section):
 *  [W]   "ik_llama.cpp 量化权重之谜：weight[j] = qw[j] * sqrtf(sigma2 +
 *        xb[j]*xb[j])的由来与原理" (www.dpshk.com/news/4810665)
 *  [Q8]  "ik_llama.cpp 量化精度修复实录：用 Q8_K_128 替代 Q8_1 根治
 *        IQ1_S_R4 / IQ1_M_R4 的 fp16 溢出" (www.hnwysp.cn/news/39281)
 *  [SVD] "量化方法论实证：为什么 LQER/L²QER 难以改进 ik_llama.cpp 的
 *        k-quants 与 i-quants" (www.0539edu.com/news/4792009)
 *  [PTQ] "从零理解 LLM 量化：PTQ、QAT 与 ik_llama.cpp 量化体系的源码级导学"
 *        (m.nxbn.cn/news/53383)
 *
 * Where the pages leave a step open, the reading taken is stated beside the
 * step; every such reading is also listed in the design notes.
 *
 * Parity pins: every exported function is pinned by the CPU test suite
 * (closed forms, a library fp16 conversion, brute force on toy blocks, a
 * dense scale sweep, exact rational arithmetic and invariants).  The pages
 * print no worked quantization example, so the absolute values of the
 * scale search beyond those properties are "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORACLE_QK4_0 32     /* weights per Q4_0 block: "QK4_0" in [W] §一 */
#define ORACLE_Q4_0_BYTES 18 /* fp16 d + 16 bytes of nibbles */
#define ORACLE_QK8 128      /* Q8_K_128 block size, [Q8] 修复方案 */
#define ORACLE_Q8_BYTES 140 /* float d + int8 qs[128] + int16 bsums[4] */

#define FLAG_NONFINITE 1u
#define FLAG_NEG_QW 2u
#define FLAG_SCALE_OVERFLOW 4u

static uint32_t f32_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* ------------------------------------------------------------------ */
/* IEEE 754 binary16, written from the format's definition:            */
/* 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits; largest    */
/* finite 65504, smallest normal 2^-14, smallest subnormal 2^-24.      */
/* ------------------------------------------------------------------ */

/* Round-half-to-even of (m >> s) for s >= 1, m < 2^32. */
static uint32_t shift_rne(uint32_t m, int s)
{
    if (s >= 32) return 0;
    uint32_t q = m >> s;
    uint32_t rem = m & ((1u << s) - 1u);
    uint32_t half = 1u << (s - 1);
    if (rem > half || (rem == half && (q & 1u))) q += 1u;
    return q;
}

uint16_t oracle_fp16_from_float(float f)
{
    uint32_t u = f32_bits(f);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    uint32_t a = u & 0x7fffffffu;
    if (a > 0x7f800000u) {                 /* NaN: quiet NaN, keep top payload bits */
        return (uint16_t)(sign | 0x7e00u | ((a >> 13) & 0x3ffu));
    }
    if (a == 0x7f800000u) return (uint16_t)(sign | 0x7c00u);
    int e = (int)(a >> 23) - 127;          /* unbiased exponent of a normal float */
    uint32_t mant = (a & 0x7fffffu);
    if ((a >> 23) == 0) return sign;       /* binary32 subnormals are < 2^-126: round to 0 */
    mant |= 0x800000u;                     /* 24-bit significand, value = mant * 2^(e-23) */
    if (e >= -14) {
        /* normal binary16 candidate: keep 11 bits, round the low 13 */
        uint32_t q = shift_rne(mant, 13);  /* in [2^10, 2^11] */
        uint32_t be = (uint32_t)(e + 15);
        if (q == 0x800u) { q >>= 1; be += 1; }
        if (be >= 31) return (uint16_t)(sign | 0x7c00u);   /* overflow to infinity */
        return (uint16_t)(sign | (be << 10) | (q & 0x3ffu));
    }
    /* subnormal binary16: value / 2^-24 = mant * 2^(e+1), e+1 <= -14 */
    int s = -(e + 1);
    uint32_t q = shift_rne(mant, s);       /* q <= 2^10; q == 2^10 is the smallest normal */
    return (uint16_t)(sign | q);
}

float oracle_fp16_to_float(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int be = (h >> 10) & 0x1f;
    int fr = h & 0x3ff;
    float v;
    if (be == 0x1f) v = fr ? NAN : INFINITY;
    else if (be == 0) v = ldexpf((float)fr, -24);
    else v = ldexpf((float)(fr | 0x400), be - 25);
    return sign ? -v : v;
}

/* ------------------------------------------------------------------ */
/* Row energy sigma2, [W] §一: sigma2 = sum_x2 / n_per_row with        */
/* sum_x2 = sum_j x[j]^2 over the whole row.                           */
/* Reading: the products x*x are exact in binary64 and are summed in   */
/* binary64 left to right; the quotient is rounded once to binary32.   */
/* (The page's code sums in float; binary64 makes the result           */
/* independent of summation order to within one rounding.)             */
/* ------------------------------------------------------------------ */
float oracle_row_sigma2(const float *x, int64_t n)
{
    double s = 0.0;
    for (int64_t j = 0; j < n; ++j) s += (double)x[j] * (double)x[j];
    return (float)(s / (double)n);
}

/* ------------------------------------------------------------------ */
/* Importance weights of one block, [W] §一:                           */
/*   mode 0: weight[j] = qw[j] * sqrtf(sigma2 + xb[j]*xb[j])           */
/*   mode 1: weight[j] = qw[j]      (the variant [W] §一/§二 discusses) */
/* and the magnitude forms [W] §二 lists as tried before imatrix       */
/* existed (x^2, |x|, sigma^2 + x^2, sigma + |x|), here times qw:       */
/*   mode 2: qw * (x*x)        mode 3: qw * |x|                         */
/*   mode 4: qw * (sigma2 + x*x)   mode 5: qw * (sqrtf(sigma2) + |x|)   */
/* qw == NULL means qw[j] = 1 (the pure magnitude forms).  Each         */
/* operation rounds to binary32: t = x*x, u = sigma2 + t, s = sqrtf(u), */
/* w = qw*s; sigma = sqrtf(sigma2).                                     */
/* ------------------------------------------------------------------ */
void oracle_block_weights(const float *xb, const float *qwb, int n, float sigma2,
                          int weight_mode, float *w)
{
    const float sigma = sqrtf(sigma2);
    for (int j = 0; j < n; ++j) {
        float q = qwb ? qwb[j] : 1.0f;
        float x = xb[j];
        float t = x * x;
        float m;
        switch (weight_mode) {
        case 1: m = 1.0f; break;
        case 2: m = t; break;
        case 3: m = fabsf(x); break;
        case 4: m = sigma2 + t; break;
        case 5: m = sigma + fabsf(x); break;
        default: m = sqrtf(sigma2 + t); break;
        }
        w[j] = weight_mode == 1 ? q : q * m;
    }
}

/* ------------------------------------------------------------------ */
/* Weighted least-squares scale search for one block ("make_qx_quants" */
/* with nmax = 8, [W] §一): codes l in [-8, 7], sums                   */
/*   sumlx = sum w*x*l,  suml2 = sum w*l*l,  d = sumlx / suml2,        */
/* followed by greedy code moves driven by g = d*w*(x - d*l).          */
/*                                                                     */
/* Readings (the pages print the sums, the scale and the greedy        */
/* gradient, not the candidate set nor the stopping rule):             */
/*  - xmax is the signed value of the first element of largest |x|.    */
/*  - candidates k = -9..9: c_k = (float)(80+k)/10.0f,                 */
/*    iscale_k = -c_k/xmax, l = clamp(rint(iscale_k*x), -8, 7)         */
/*    (product rounded to binary32, rint = half to even).              */
/*  - wx[j] = w[j]*x[j] rounded once; sums run j = 0..n-1 from +0 with */
/*    sumlx = fmaf(wx, l, sumlx) and suml2 = fmaf(w, l*l, suml2).      */
/*  - score = (sumlx*sumlx)/suml2, -inf when suml2 <= 0; the strictly  */
/*    largest score wins, ties keep the lowest k.                      */
/*  - greedy: at most 5 passes over j = 0..n-1 (Gauss-Seidel).  At j:  */
/*    d = sumlx/suml2, g = d*(w*(x - d*l)); skip if g == 0; s = sign g;*/
/*    skip if l+s leaves [-8,7]; trial sumlx' = sumlx + s*wx,          */
/*    suml2' = fmaf(w, 2*s*l+1, suml2); accept iff suml2' > 0 and      */
/*    (sumlx'*sumlx')/suml2' > score.  A pass with no accepted move    */
/*    ends the search.                                                 */
/*  - final: sums recomputed from the final codes as above,            */
/*    d = sumlx/suml2.                                                 */
/*  - xmax == 0: d = 0, all codes 0, no search.                        */
/*  - every candidate score -inf (all weights 0 where l != 0): codes   */
/*    of k = 0, d = 1/iscale_0, no greedy.                             */
/*  - the fudge factor of [W] §四 has no printed value; it is 1 here.  */
/*                                                                     */
/* info (nullable) receives {k_sweep, passes, fallback, reserved}.     */
/* L_sweep (nullable) receives the codes chosen by the candidate sweep. */
/* Returns d (binary32).  n is 32 for Q4_0; small n serves the toy     */
/* brute-force checks.                                                 */
/* ------------------------------------------------------------------ */
static void candidate_codes(int n, int nmax, const float *xb, float iscale, float *l)
{
    const float lo = (float)(-nmax), hi = (float)(nmax - 1);
    for (int j = 0; j < n; ++j) {
        float v = iscale * xb[j];
        float r = rintf(v);
        l[j] = fminf(fmaxf(r, lo), hi);
    }
}

static void block_sums(int n, const float *wx, const float *w, const float *l,
                       float *sumlx, float *suml2)
{
    float a = 0.0f, b = 0.0f;
    for (int j = 0; j < n; ++j) {
        a = fmaf(wx[j], l[j], a);
        b = fmaf(w[j], l[j] * l[j], b);
    }
    *sumlx = a;
    *suml2 = b;
}

/* The same search for the other 32-value formats of the family (Q5_0, Q6_0,
 * Q8_0, [W] §一: "the same formula appears in quantize_row_q5_0_impl ..."):
 * nmax = 16, 32, 128 with codes in [-nmax, nmax-1].  Reading: the candidates
 * scale with nmax, c_k = (float)(nmax*(80+k)) / 80.0f (for nmax = 8 exactly
 * the Q4_0 set (80+k)/10); every other step is unchanged. */
float oracle_qx_block_search(int n, int nmax, const float *xb, const float *w, int8_t *L,
                             int8_t *L_sweep, int32_t *info)
{
    float wx[64], l[64], lbest[64];
    if (n <= 0 || n > 64) return NAN;
    if (nmax != 8 && nmax != 16 && nmax != 32 && nmax != 128) return NAN;
    const float lo = (float)(-nmax), hi = (float)(nmax - 1);
    if (info) { info[0] = 0; info[1] = 0; info[2] = 0; info[3] = 0; }

    float amax = 0.0f, xmax = 0.0f;
    for (int j = 0; j < n; ++j) {
        float a = fabsf(xb[j]);
        if (a > amax) { amax = a; xmax = xb[j]; }
    }
    if (amax == 0.0f) {
        for (int j = 0; j < n; ++j) { L[j] = 0; if (L_sweep) L_sweep[j] = 0; }
        return 0.0f;
    }
    for (int j = 0; j < n; ++j) wx[j] = w[j] * xb[j];

    float best = -INFINITY;
    int kbest = 0;
    for (int k = -9; k <= 9; ++k) {
        float c = (float)(nmax * (80 + k)) / 80.0f;
        float iscale = -c / xmax;
        candidate_codes(n, nmax, xb, iscale, l);
        float sumlx, suml2;
        block_sums(n, wx, w, l, &sumlx, &suml2);
        float score = suml2 > 0.0f ? (sumlx * sumlx) / suml2 : -INFINITY;
        if (score > best) {
            best = score;
            kbest = k;
            memcpy(lbest, l, sizeof(float) * (size_t)n);
        }
    }

    if (best == -INFINITY) {
        /* no candidate has a positive weighted code energy */
        float iscale0 = -(float)nmax / xmax;
        candidate_codes(n, nmax, xb, iscale0, l);
        for (int j = 0; j < n; ++j) {
            L[j] = (int8_t)l[j];
            if (L_sweep) L_sweep[j] = (int8_t)l[j];
        }
        if (info) { info[0] = 0; info[1] = 0; info[2] = 1; }
        return 1.0f / iscale0;
    }
    if (L_sweep) for (int j = 0; j < n; ++j) L_sweep[j] = (int8_t)lbest[j];

    float sumlx, suml2;
    block_sums(n, wx, w, lbest, &sumlx, &suml2);
    float score = best;
    int passes = 0;
    for (int pass = 0; pass < 5; ++pass) {
        int changed = 0;
        ++passes;
        for (int j = 0; j < n; ++j) {
            float d = sumlx / suml2;
            float g = d * (w[j] * (xb[j] - d * lbest[j]));
            if (g == 0.0f || g != g) continue;
            float s = g > 0.0f ? 1.0f : -1.0f;
            float ln = lbest[j] + s;
            if (ln < lo || ln > hi) continue;
            float nlx = sumlx + s * wx[j];
            float nl2 = fmaf(w[j], 2.0f * s * lbest[j] + 1.0f, suml2);
            if (!(nl2 > 0.0f)) continue;
            float nscore = (nlx * nlx) / nl2;
            if (nscore > score) {
                lbest[j] = ln;
                sumlx = nlx;
                suml2 = nl2;
                score = nscore;
                changed = 1;
            }
        }
        if (!changed) break;
    }
    block_sums(n, wx, w, lbest, &sumlx, &suml2);
    for (int j = 0; j < n; ++j) L[j] = (int8_t)lbest[j];
    if (info) { info[0] = kbest; info[1] = passes; info[2] = 0; }
    return sumlx / suml2;
}

float oracle_q4_0_block_search(int n, const float *xb, const float *w, int8_t *L,
                               int8_t *L_sweep, int32_t *info)
{
    return oracle_qx_block_search(n, 8, xb, w, L, L_sweep, info);
}

/* ------------------------------------------------------------------ */
/* Q4_0 block layout (reading; the pages name QK4_0 and the 4-bit      */
/* legacy family, [W] §一 and [PTQ] §2.1, not the byte order):         */
/*   bytes 0..1  : d as binary16, little endian                        */
/*   bytes 2..17 : qs[i] = (l[i]+8) | (l[i+16]+8) << 4, i = 0..15      */
/* Row r, block b sits at byte (r*nb + b)*18.                          */
/* ------------------------------------------------------------------ */
static void pack_q4_0(float d, const int8_t *L, uint8_t *blk, uint32_t *flags)
{
    uint16_t h = oracle_fp16_from_float(d);
    if ((h & 0x7fffu) == 0x7c00u && isfinite(d) && flags) *flags |= FLAG_SCALE_OVERFLOW;
    blk[0] = (uint8_t)(h & 0xff);
    blk[1] = (uint8_t)(h >> 8);
    for (int i = 0; i < 16; ++i)
        blk[2 + i] = (uint8_t)((L[i] + 8) | ((L[i + 16] + 8) << 4));
}

/* Whole-tensor imatrix-weighted Q4_0 quantization, [W] §一:           */
/* per row sigma2, per 32-block weights, search, pack.                 */
/* qw row for row r: qw + (rows_per_qw ? r/rows_per_qw : 0)*n_per_row. */
/* passes (nullable) receives the greedy pass count of every block.    */
/* Returns 0, or -1 for a shape the format cannot hold.                */
int oracle_quantize_q4_0_w(const float *x, const float *qw, uint8_t *out, int64_t nrows,
                           int64_t n_per_row, int64_t rows_per_qw, int weight_mode,
                           uint32_t *flags, int32_t *passes)
{
    if (n_per_row % ORACLE_QK4_0 != 0 || nrows < 0 || n_per_row < 0) return -1;
    if (weight_mode < 0 || weight_mode > 5) return -1;
    const int64_t nb = n_per_row / ORACLE_QK4_0;
    float w[ORACLE_QK4_0];
    int8_t L[ORACLE_QK4_0];
    int32_t info[4];
    for (int64_t r = 0; r < nrows; ++r) {
        const float *xr = x + r * n_per_row;
        const float *qr = qw ? qw + (rows_per_qw > 0 ? r / rows_per_qw : 0) * n_per_row : NULL;
        if (flags) {
            for (int64_t j = 0; j < n_per_row; ++j) {
                if (!isfinite(xr[j])) *flags |= FLAG_NONFINITE;
                if (qr && !isfinite(qr[j])) *flags |= FLAG_NONFINITE;
                if (qr && qr[j] < 0.0f) *flags |= FLAG_NEG_QW;
            }
        }
        float sigma2 = oracle_row_sigma2(xr, n_per_row);
        for (int64_t b = 0; b < nb; ++b) {
            const float *xb = xr + b * ORACLE_QK4_0;
            oracle_block_weights(xb, qr ? qr + b * ORACLE_QK4_0 : NULL, ORACLE_QK4_0, sigma2,
                                 weight_mode, w);
            float d = oracle_q4_0_block_search(ORACLE_QK4_0, xb, w, L, NULL, info);
            pack_q4_0(d, L, out + (r * nb + b) * ORACLE_Q4_0_BYTES, flags);
            if (passes) passes[r * nb + b] = info[1];
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* The other 32-value formats (reading; the pages name the types, not  */
/* their bytes).  n = l + nmax is the biased code.                     */
/*   bits 5 (Q5_0, 22 B): d16 | qh (u32 LE, bit j = (n_j >> 4) & 1)    */
/*                        | qs[16], qs[i] = (n_i & 15) | (n_{i+16} & 15) << 4 */
/*   bits 6 (Q6_0, 26 B): d16 | qh (u64 LE, bits 2j..2j+1 = n_j >> 4)  */
/*                        | qs[16] as for Q5_0                          */
/*   bits 8 (Q8_0, 34 B): d16 | int8 qs[32] = l_j                       */
/*   bits 4 (Q4_0, 18 B): as above                                      */
/* ------------------------------------------------------------------ */
int oracle_qx_block_bytes(int bits)
{
    switch (bits) {
    case 4: return 18;
    case 5: return 22;
    case 6: return 26;
    case 8: return 34;
    default: return -1;
    }
}

static int nmax_of(int bits) { return bits == 8 ? 128 : 1 << (bits - 1); }

static void pack_qx(int bits, float d, const int8_t *L, uint8_t *blk, uint32_t *flags)
{
    if (bits == 4) { pack_q4_0(d, L, blk, flags); return; }
    uint16_t h = oracle_fp16_from_float(d);
    if ((h & 0x7fffu) == 0x7c00u && isfinite(d) && flags) *flags |= FLAG_SCALE_OVERFLOW;
    blk[0] = (uint8_t)(h & 0xff);
    blk[1] = (uint8_t)(h >> 8);
    if (bits == 8) {
        for (int j = 0; j < 32; ++j) blk[2 + j] = (uint8_t)L[j];
        return;
    }
    const int nmax = nmax_of(bits);
    const int hb = bits == 5 ? 4 : 8;          /* bytes of high bits */
    uint64_t qh = 0;
    for (int j = 0; j < 32; ++j) {
        unsigned n = (unsigned)(L[j] + nmax);
        if (bits == 5) qh |= (uint64_t)((n >> 4) & 1u) << j;
        else qh |= (uint64_t)((n >> 4) & 3u) << (2 * j);
    }
    for (int b = 0; b < hb; ++b) blk[2 + b] = (uint8_t)(qh >> (8 * b));
    for (int i = 0; i < 16; ++i) {
        unsigned lo = (unsigned)(L[i] + nmax) & 15u, hi = (unsigned)(L[i + 16] + nmax) & 15u;
        blk[2 + hb + i] = (uint8_t)(lo | (hi << 4));
    }
}

static int unpack_code(int bits, const uint8_t *blk, int j)
{
    if (bits == 8) return (int8_t)blk[2 + j];
    const int nmax = nmax_of(bits);
    if (bits == 4) {
        int nib = j < 16 ? (blk[2 + j] & 0xf) : (blk[2 + j - 16] >> 4);
        return nib - nmax;
    }
    const int hb = bits == 5 ? 4 : 8;
    uint64_t qh = 0;
    for (int b = 0; b < hb; ++b) qh |= (uint64_t)blk[2 + b] << (8 * b);
    int low = j < 16 ? (blk[2 + hb + j] & 0xf) : (blk[2 + hb + j - 16] >> 4);
    int high = bits == 5 ? (int)((qh >> j) & 1u) : (int)((qh >> (2 * j)) & 3u);
    return (low | (high << 4)) - nmax;
}

/* Weighted quantization of a tensor to any of the 32-value formats. */
/* fudge: the importance's correction factor of [W] §四 (the fudge factor the code
 * takes from ggml_get_quantize_fudge_factor; its values are not printed).  Reading: §四
 * introduces it as a correction of the approximate (diagonal) Hessian, i.e. of the
 * importance, so it scales the sigma2 term of the forms that have one:
 * sigma2_used = fl(fudge * sigma2) for modes 0, 4 and 5; fudge = 1 changes nothing. */
int oracle_quantize_qx_0_w_f(int bits, const float *x, const float *qw, uint8_t *out, int64_t nrows,
                             int64_t n_per_row, int64_t rows_per_qw, int weight_mode, float fudge,
                             uint32_t *flags)
{
    const int bb = oracle_qx_block_bytes(bits);
    if (bb < 0 || n_per_row % 32 != 0 || nrows < 0 || n_per_row < 0) return -1;
    if (weight_mode < 0 || weight_mode > 5) return -1;
    const int nmax = nmax_of(bits);
    const int64_t nb = n_per_row / 32;
    float w[32];
    int8_t L[32];
    for (int64_t r = 0; r < nrows; ++r) {
        const float *xr = x + r * n_per_row;
        const float *qr = qw ? qw + (rows_per_qw > 0 ? r / rows_per_qw : 0) * n_per_row : NULL;
        if (flags) {
            for (int64_t j = 0; j < n_per_row; ++j) {
                if (!isfinite(xr[j])) *flags |= FLAG_NONFINITE;
                if (qr && !isfinite(qr[j])) *flags |= FLAG_NONFINITE;
                if (qr && qr[j] < 0.0f) *flags |= FLAG_NEG_QW;
            }
        }
        float sigma2 = fudge * oracle_row_sigma2(xr, n_per_row);
        for (int64_t b = 0; b < nb; ++b) {
            const float *xb = xr + b * 32;
            oracle_block_weights(xb, qr ? qr + b * 32 : NULL, 32, sigma2, weight_mode, w);
            float d = oracle_qx_block_search(32, nmax, xb, w, L, NULL, NULL);
            pack_qx(bits, d, L, out + (r * nb + b) * bb, flags);
        }
    }
    return 0;
}

int oracle_quantize_qx_0_w(int bits, const float *x, const float *qw, uint8_t *out, int64_t nrows,
                           int64_t n_per_row, int64_t rows_per_qw, int weight_mode,
                           uint32_t *flags)
{
    return oracle_quantize_qx_0_w_f(bits, x, qw, out, nrows, n_per_row, rows_per_qw, weight_mode, 1.0f,
                                    flags);
}

/* y = fp16_to_float(d) * l for any of the 32-value formats (exact in binary32). */
int oracle_dequant_qx_0(int bits, const uint8_t *blocks, float *y, int64_t nrows, int64_t n_per_row)
{
    const int bb = oracle_qx_block_bytes(bits);
    if (bb < 0 || n_per_row % 32 != 0) return -1;
    const int64_t nblk = nrows * (n_per_row / 32);
    for (int64_t g = 0; g < nblk; ++g) {
        const uint8_t *blk = blocks + g * bb;
        float d = oracle_fp16_to_float((uint16_t)(blk[0] | (blk[1] << 8)));
        for (int j = 0; j < 32; ++j) y[g * 32 + j] = d * (float)unpack_code(bits, blk, j);
    }
    return 0;
}

/* Dequantization of Q4_0 blocks: y = fp16_to_float(d) * (nibble - 8). */
/* The product is exact in binary32 (11-bit significand times |n|<=8). */
int oracle_dequant_q4_0(const uint8_t *blocks, float *y, int64_t nrows, int64_t n_per_row)
{
    if (n_per_row % ORACLE_QK4_0 != 0) return -1;
    const int64_t nblk = nrows * (n_per_row / ORACLE_QK4_0);
    for (int64_t g = 0; g < nblk; ++g) {
        const uint8_t *blk = blocks + g * ORACLE_Q4_0_BYTES;
        float d = oracle_fp16_to_float((uint16_t)(blk[0] | (blk[1] << 8)));
        for (int i = 0; i < 16; ++i) {
            int lo = blk[2 + i] & 0xf, hi = blk[2 + i] >> 4;
            y[g * 32 + i] = d * (float)(lo - 8);
            y[g * 32 + i + 16] = d * (float)(hi - 8);
        }
    }
    return 0;
}

/* Round-trip error reduction.  [SVD] §3.2 names the quantize-stats     */
/* statistics rmse = sqrt(total_error / num_samples) and maxerr; the    */
/* weighted form uses the imatrix entries as weights.  Reading: the     */
/* weights are qw alone (not the quantizer weights), e = x - y is       */
/* rounded once to binary32, and the sums are binary64:                 */
/*   acc[0] += qw*e*e, acc[1] += qw, acc[2] += e*e, acc[3] = max |e|.   */
/* acc accumulates (the caller zeroes it); wrmse = sqrt(acc0/acc1),     */
/* rmse = sqrt(acc2/(nrows*n_per_row)).  Any of the 32-value formats    */
/* (bits 4, 5, 6, 8), y = fp16(d) * code as oracle_dequant_qx_0.        */
int oracle_weighted_rmse_qx(int bits, const float *x, const uint8_t *blocks, const float *qw,
                            int64_t nrows, int64_t n_per_row, int64_t rows_per_qw, double *acc)
{
    const int bb = oracle_qx_block_bytes(bits);
    if (bb < 0 || n_per_row % 32 != 0) return -1;
    const int64_t nb = n_per_row / 32;
    for (int64_t r = 0; r < nrows; ++r) {
        const float *qr = qw ? qw + (rows_per_qw > 0 ? r / rows_per_qw : 0) * n_per_row : NULL;
        for (int64_t b = 0; b < nb; ++b) {
            const uint8_t *blk = blocks + (r * nb + b) * bb;
            float d = oracle_fp16_to_float((uint16_t)(blk[0] | (blk[1] << 8)));
            for (int i = 0; i < 32; ++i) {
                float y = d * (float)unpack_code(bits, blk, i);
                int64_t j = b * 32 + i;
                float e = x[r * n_per_row + j] - y;
                double ed = (double)e;
                double q = qr ? (double)qr[j] : 1.0;
                acc[0] += q * (ed * ed);
                acc[1] += q;
                acc[2] += ed * ed;
                if (fabs(ed) > acc[3]) acc[3] = fabs(ed);
            }
        }
    }
    return 0;
}

/* The Q4_0 form (18-byte blocks). */
int oracle_weighted_rmse(const float *x, const uint8_t *blocks, const float *qw,
                         int64_t nrows, int64_t n_per_row, int64_t rows_per_qw, double *acc)
{
    return oracle_weighted_rmse_qx(4, x, blocks, qw, nrows, n_per_row, rows_per_qw, acc);
}

/* ------------------------------------------------------------------ */
/* Q8_K_128 activation quantization, [Q8] 修复方案: blocks of 128       */
/* values, a binary32 scale, int8 codes, and one int16 sum of the codes */
/* per 32 values that is NOT multiplied by d.                           */
/* Readings: amax = max |x| (NaN ignored); d = amax/127;                */
/* id = amax > 0 ? 127/amax : 0; q = clamp(rint(x*id), -127, 127) with  */
/* a NaN product giving 0; bsums[i] = sum of q over values 32i..32i+31. */
/* Layout: float d (LE) | int8 qs[128] | int16 bsums[4] (LE) = 140 B.   */
/* Requires n_per_row % 128 == 0 (the selection rule of [Q8] 修复方案). */
/* ------------------------------------------------------------------ */
int oracle_quantize_q8_k128(const float *x, uint8_t *out, int64_t nrows, int64_t n_per_row,
                            uint32_t *flags)
{
    if (n_per_row % ORACLE_QK8 != 0 || nrows < 0 || n_per_row < 0) return -1;
    const int64_t nblk = nrows * (n_per_row / ORACLE_QK8);
    for (int64_t g = 0; g < nblk; ++g) {
        const float *xb = x + g * ORACLE_QK8;
        uint8_t *blk = out + g * ORACLE_Q8_BYTES;
        float amax = 0.0f;
        for (int j = 0; j < ORACLE_QK8; ++j) {
            float a = fabsf(xb[j]);
            if (!isfinite(xb[j]) && flags) *flags |= FLAG_NONFINITE;
            if (a > amax) amax = a;
        }
        float d = amax / 127.0f;
        float id = amax > 0.0f ? 127.0f / amax : 0.0f;
        int8_t q[ORACLE_QK8];
        for (int j = 0; j < ORACLE_QK8; ++j) {
            float v = xb[j] * id;
            if (v != v) { q[j] = 0; continue; }
            float r = fminf(fmaxf(rintf(v), -127.0f), 127.0f);
            q[j] = (int8_t)r;
        }
        memcpy(blk, &d, 4);
        memcpy(blk + 4, q, ORACLE_QK8);
        for (int i = 0; i < 4; ++i) {
            int s = 0;
            for (int j = 0; j < 32; ++j) s += q[32 * i + j];
            int16_t s16 = (int16_t)s;
            memcpy(blk + 132 + 2 * i, &s16, 2);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Q8_1 activation quantization, the format [Q8] 修复前的数值隐患       */
/* describes: blocks of 32 values with a binary16 scale d = x_max/127  */
/* and a binary16 sum s = d * sum(q).  s can overflow binary16 even    */
/* when d fits, which is the failure Q8_K_128 removes.                 */
/* Readings (same code rule as Q8_K_128): amax = max|x|, d = amax/127, */
/* id = amax > 0 ? 127/amax : 0, q = clamp(rint(x*id), -127, 127)      */
/* (a NaN product gives 0); s = d * (float)sum(q) in binary32; both     */
/* stored as binary16 RNE.  Layout: half d | half s | int8 qs[32]      */
/* = 36 bytes.  Returns the number of blocks whose stored s is +-Inf   */
/* while d is finite.                                                  */
/* ------------------------------------------------------------------ */
int64_t oracle_quantize_q8_1(const float *x, uint8_t *out, int64_t nrows, int64_t n_per_row)
{
    if (n_per_row % 32 != 0 || nrows < 0 || n_per_row < 0) return -1;
    const int64_t nblk = nrows * (n_per_row / 32);
    int64_t overflow = 0;
    for (int64_t g = 0; g < nblk; ++g) {
        const float *xb = x + g * 32;
        uint8_t *blk = out + g * 36;
        float amax = 0.0f;
        for (int j = 0; j < 32; ++j) {
            float a = fabsf(xb[j]);
            if (a > amax) amax = a;
        }
        float d = amax / 127.0f;
        float id = amax > 0.0f ? 127.0f / amax : 0.0f;
        int sum = 0;
        for (int j = 0; j < 32; ++j) {
            float v = xb[j] * id;
            int q = 0;
            if (v == v) q = (int)fminf(fmaxf(rintf(v), -127.0f), 127.0f);
            blk[4 + j] = (uint8_t)(int8_t)q;
            sum += q;
        }
        float sf = d * (float)sum;
        uint16_t hd = oracle_fp16_from_float(d), hs = oracle_fp16_from_float(sf);
        memcpy(blk, &hd, 2);
        memcpy(blk + 2, &hs, 2);
        if ((hs & 0x7fffu) == 0x7c00u && (hd & 0x7fffu) != 0x7c00u) ++overflow;
    }
    return overflow;
}

/* ------------------------------------------------------------------ */
/* Q4_0 x Q8_K_128 dot product (matrix-vector form).                   */
/* [Q8] 修复前的数值隐患 describes the consumer of the activation       */
/* blocks: weight codes times int8 activation codes, block by block.    */
/* The value computed is the plain definition -- the dot product of the */
/* two dequantized vectors:                                             */
/*   y[t][r] = sum_j  W~[r][j] * A~[t][j],                              */
/*   W~ = fp16_to_float(d4) * (nibble - 8)     (exact in binary32),     */
/*   A~ = d8 * q                               (exact in binary64).     */
/* Each product W~ * A~ needs at most 11+4+24+8 = 47 significant bits,  */
/* so it is exact in binary64; the K products are summed left to right  */
/* in binary64 (error <= K * 2^-53 * sum |products|).  absum receives    */
/* sum |W~ * A~| (the condition of the sum), and may be NULL.           */
/* Layouts: w is n_out rows of k/32 Q4_0 blocks (18 B each); a is n_tok */
/* rows of k/128 Q8_K_128 blocks (140 B each); y and absum are          */
/* [n_tok][n_out].  k must be a multiple of 128.                        */
/* ------------------------------------------------------------------ */
int oracle_dot_q4_0_q8_k128(const uint8_t *w, const uint8_t *a, double *y, double *absum,
                            int64_t n_out, int64_t k, int64_t n_tok)
{
    if (k % ORACLE_QK8 != 0 || n_out < 0 || k < 0 || n_tok < 0) return -1;
    const int64_t nb4 = k / ORACLE_QK4_0, nb8 = k / ORACLE_QK8;
    for (int64_t t = 0; t < n_tok; ++t) {
        const uint8_t *ar = a + t * nb8 * ORACLE_Q8_BYTES;
        for (int64_t r = 0; r < n_out; ++r) {
            const uint8_t *wr = w + r * nb4 * ORACLE_Q4_0_BYTES;
            double sum = 0.0, asum = 0.0;
            for (int64_t j = 0; j < k; ++j) {
                const uint8_t *wb = wr + (j / ORACLE_QK4_0) * ORACLE_Q4_0_BYTES;
                const int i = (int)(j % ORACLE_QK4_0);
                const int nib = i < 16 ? (wb[2 + i] & 0xf) : (wb[2 + i - 16] >> 4);
                const double wv = (double)oracle_fp16_to_float((uint16_t)(wb[0] | (wb[1] << 8)))
                                  * (double)(nib - 8);
                const uint8_t *ab = ar + (j / ORACLE_QK8) * ORACLE_Q8_BYTES;
                float d8;
                memcpy(&d8, ab, sizeof d8);
                const double av = (double)d8 * (double)(int8_t)ab[4 + j % ORACLE_QK8];
                const double p = wv * av;
                sum += p;
                asum += fabs(p);
            }
            y[t * n_out + r] = sum;
            if (absum) absum[t * n_out + r] = asum;
        }
    }
    return 0;
}

/* Layout constants, for the test suite's self-description checks. */
int oracle_q4_0_block_bytes(void) { return ORACLE_Q4_0_BYTES; }
int oracle_q8_k128_block_bytes(void) { return ORACLE_Q8_BYTES; }

/* Array forms of the binary16 conversions (used by the exhaustive pin). */
void oracle_fp16_from_float_array(const float *f, uint16_t *h, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) h[i] = oracle_fp16_from_float(f[i]);
}

void oracle_fp16_to_float_array(const uint16_t *h, float *f, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) f[i] = oracle_fp16_to_float(h[i]);
}
