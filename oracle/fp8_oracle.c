/*
 * fp8_oracle.c -- plain, slow, obviously correct CPU oracle for the FP8
 * scaled-quantization path (amax -> scale -> saturating RNE cast -> scaled
 * GEMM, delayed-scaling history, FP8 KV cache).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file.  It shares no code, header, table or constant generator with
 * the CUDA library; the only thing both sides share is the seeded synthetic
 * input generator, which holds none of the method's arithmetic.
 *
 * Sources (web pages on FP8 scaled quantization):
 *   [DeepL]  "DeepL押注FP8：大模型训练与推理统一精度实战解析"
 *            §2.1 format split (E4M3 forward, E5M2 gradients, bit layouts),
 *            §2.3 per-tensor / per-row / per-block scaling, delayed scaling
 *                 and the "deviation above a threshold" recovery check,
 *            §3.1 FP8 KV cache, §4.2 max-absolute-value statistics,
 *            §5.1 E5M2 overflow, §5.3 FP8 GEMM determinism.
 *   [H100]   "H100 FP8加速实测：新一代计算架构的飞跃" -- E5M2 reaches +-57344,
 *            FP8 multiply-accumulate on tensor cores.
 *   [Soup]   "FP8训练与QAT量化感知训练：如何在Hopper GPU上用Soup把大模型微调提速2倍",
 *            section "FP8 三种缩放配方怎么选": tensorwise single scale;
 *            rowwise per-row e4m3 scales that are powers of two.
 *   The bit-level format semantics the pages leave open (E4M3 without
 *   infinities, max 448, NaN code S.1111.111; E5M2 IEEE-like) follow the OCP
 *   8-bit floating point specification (Micikevicius et al. 2022, "FP8
 *   Formats for Deep Learning").
 *
 * Readings where the pages are silent (each is repeated in the design notes):
 *   - rounding is round-to-nearest, ties to the even code, and out-of-range
 *     magnitudes (and +-Inf) saturate to +-fmax;
 *   - amax ignores NaN and +-Inf (they are counted as non-finite);
 *   - amax == 0 gives scale 1; a scale that overflows fp32 is clamped;
 *   - s = fmax / amax as one correctly rounded fp32 division; the pow2 rule
 *     takes the largest power of two s with amax * s <= fmax;
 *   - the cast is y = fp32(x) * s (one rounded fp32 multiply), then RNE;
 *   - delayed scaling: the history starts at zero, the window statistic is
 *     the max, margin 0, and the recovery trigger is saturation
 *     (amax_t * s_t > fmax).
 *
 * Every floating-point step that decides a stored byte is done in the
 * precision the method fixes (fp32 for scale and product); every sum the
 * GEMM reference needs is done in fp64.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORC_E4M3 0
#define ORC_E5M2 1

/* ---------------------------------------------------------------- decode -- */

/* Value of one FP8 code, from its sign / exponent / mantissa fields
 * ([DeepL] §2.1: E4M3 = 1+4+3 bits, E5M2 = 1+5+2 bits).
 *   E4M3: bias 7, no infinities, S.1111.111 is NaN, all other codes finite.
 *   E5M2: bias 15, exponent 31 is Inf (mantissa 0) or NaN (mantissa != 0). */
double orc_decode(uint8_t code, int fmt)
{
    int sign = code >> 7;
    int mbits = (fmt == ORC_E4M3) ? 3 : 2;
    int ebits = (fmt == ORC_E4M3) ? 4 : 5;
    int bias = (fmt == ORC_E4M3) ? 7 : 15;
    int e = (code >> mbits) & ((1 << ebits) - 1);
    int m = code & ((1 << mbits) - 1);
    double mag;
    if (fmt == ORC_E4M3) {
        if (e == 15 && m == 7) return NAN;
    } else {
        if (e == 31) {
            if (m != 0) return NAN;
            return sign ? -INFINITY : INFINITY;
        }
    }
    if (e == 0)               /* subnormal: 0.m * 2^(1-bias) */
        mag = ldexp((double)m, 1 - bias - mbits);
    else                      /* normal: 1.m * 2^(e-bias) */
        mag = ldexp((double)((1 << mbits) + m), e - bias - mbits);
    return sign ? -mag : mag;
}

/* Largest finite magnitude code of a format: 448 (0x7E) and 57344 (0x7B). */
static uint8_t max_code(int fmt) { return fmt == ORC_E4M3 ? 0x7E : 0x7B; }

double orc_fmax(int fmt) { return orc_decode(max_code(fmt), fmt); }

/* Table of the non-negative finite values, index == code, built from
 * orc_decode (codes 0..max_code are monotone increasing). */
static double g_pos[2][128];
static int g_pos_ready[2];

static const double *pos_table(int fmt)
{
    if (!g_pos_ready[fmt]) {
        for (int c = 0; c <= max_code(fmt); ++c) g_pos[fmt][c] = orc_decode((uint8_t)c, fmt);
        g_pos_ready[fmt] = 1;
    }
    return g_pos[fmt];
}

/* ---------------------------------------------------------------- encode -- */

/* Saturating round-to-nearest-even cast of one fp32 value ([DeepL] §2.3:
 * scaled values are mapped into the range FP8 can express; §5.1: overflow is
 * the failure to avoid).  The result is the finite code nearest to y; on a tie
 * the code whose mantissa LSB is 0; magnitudes above the largest finite value
 * (and +-Inf) give +-fmax; NaN gives the format's NaN code 0x7F; the sign of a
 * zero result is kept. */
uint8_t orc_encode(float y, int fmt)
{
    if (isnan(y)) return 0x7F;
    uint8_t sign = signbit(y) ? 0x80 : 0x00;
    const double *v = pos_table(fmt);
    int top = max_code(fmt);
    double a = fabs((double)y);
    if (a >= v[top]) return (uint8_t)(sign | top);
    /* binary search: largest code lo with v[lo] <= a  (v[0] == 0 <= a) */
    int lo = 0, hi = top;          /* invariant: v[lo] <= a < v[hi] */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (v[mid] <= a) lo = mid; else hi = mid;
    }
    double dlo = a - v[lo];        /* exact: a and v[] are close binary numbers */
    double dhi = v[lo + 1] - a;
    int c;
    if (dlo < dhi) c = lo;
    else if (dhi < dlo) c = lo + 1;
    else c = (lo & 1) ? lo + 1 : lo;   /* tie: the even mantissa */
    return (uint8_t)(sign | c);
}

/* ------------------------------------------------------------ bf16 bits -- */

static float bf16_to_f32(uint16_t h)
{
    uint32_t b = (uint32_t)h << 16;
    float f;
    memcpy(&f, &b, 4);
    return f;
}

static float bits_to_f32(uint32_t b)
{
    float f;
    memcpy(&f, &b, 4);
    return f;
}

/* Round an fp32 value to bf16, nearest, ties to even: pick the nearer of the
 * two bf16 neighbours (truncation and the next value up in magnitude). */
uint16_t orc_f32_to_bf16(float f)
{
    if (isnan(f)) return (uint16_t)(signbit(f) ? 0xFFC0 : 0x7FC0);
    uint32_t b;
    memcpy(&b, &f, 4);
    uint32_t sign = b & 0x80000000u;
    uint32_t mag = b & 0x7FFFFFFFu;
    uint32_t lo = mag & 0xFFFF0000u;
    if (lo == mag) return (uint16_t)((sign | lo) >> 16);
    uint32_t hi = lo + 0x10000u;
    double a = (double)fabsf(f);
    double vlo = (double)bits_to_f32(lo);
    double vhi = (hi >= 0x7F800000u) ? ldexp(1.0, 128) : (double)bits_to_f32(hi);
    uint32_t r;
    if (a - vlo < vhi - a) r = lo;
    else if (vhi - a < a - vlo) r = hi;
    else r = (lo & 0x10000u) ? hi : lo;
    if (r > 0x7F800000u) r = 0x7F800000u;
    return (uint16_t)((sign | r) >> 16);
}

/* ------------------------------------------------------------------ amax -- */

static int bf16_finite(uint16_t h) { return (h & 0x7F80u) != 0x7F80u; }

/* amax = max |x| over the finite elements ([DeepL] §4.2: the maximum absolute
 * value of each tensor).  Non-finite elements are counted, not used. */
float orc_amax_bf16(const uint16_t *x, int64_t n, uint64_t *nonfinite)
{
    float m = 0.0f;
    uint64_t bad = 0;
    for (int64_t i = 0; i < n; ++i) {
        if (!bf16_finite(x[i])) { ++bad; continue; }
        float a = fabsf(bf16_to_f32(x[i]));
        if (a > m) m = a;
    }
    if (nonfinite) *nonfinite += bad;
    return m;
}

/* ---------------------------------------------------------------- scales -- */

/* Per-tensor / per-block scale ([DeepL] §2.3): s = fmax / amax, one correctly
 * rounded fp32 division; amax == 0 gives 1; overflow clamps to FLT_MAX. */
float orc_scale_from_amax(float amax, int fmt)
{
    if (!(amax > 0.0f)) return 1.0f;
    float fm = (float)orc_fmax(fmt);
    float s = fm / amax;
    if (isinf(s)) s = FLT_MAX;
    return s;
}

/* Power-of-two scale ([Soup] "FP8 三种缩放配方怎么选": rowwise scales are
 * powers of 2): the largest s = 2^k with amax * s <= fmax, found by exact
 * comparison in fp64 (amax * 2^k is exact); k is clamped to fp32's normal
 * range of powers of two. */
float orc_scale_pow2_from_amax(float amax, int fmt)
{
    if (!(amax > 0.0f)) return 1.0f;
    double fm = orc_fmax(fmt);
    int k = -200;
    for (int j = -200; j <= 200; ++j)
        if (ldexp((double)amax, j) <= fm) k = j;
    if (k > 127) k = 127;
    if (k < -126) k = -126;
    return (float)ldexp(1.0, k);
}

/* Dequantization scale d = 1 / s (correctly rounded fp32 division). */
float orc_inverse(float s) { return 1.0f / s; }

/* ------------------------------------------------------------------ cast -- */

/* q = cast(fp32(x) * s).  Counts elements whose scaled magnitude exceeds fmax
 * (they saturate) and non-finite inputs. */
static uint8_t cast_one(uint16_t xh, float s, int fmt, float fm, uint64_t *sat)
{
    float y = bf16_to_f32(xh) * s;
    if (sat && !isnan(y) && fabsf(y) > fm) ++*sat;
    return orc_encode(y, fmt);
}

/* ------------------------------------------------- tensorwise quantize -- */

/* Tensorwise quantization of a [rows, cols] bf16 tensor ([DeepL] §2.3
 * per-tensor scaling; [Soup] tensorwise recipe).
 *   scale_in == NULL: current scaling, s from this tensor's amax;
 *   scale_in != NULL: delayed scaling, s = *scale_in (from the history).
 * q is [rows, cols], or [cols, rows] when transpose_out is set.
 * Outputs: q, *scale_inv = 1/s, *amax_out = amax(x), counts[0] += non-finite,
 * counts[1] += saturated. */
void orc_quantize_tensorwise(const uint16_t *x, int64_t rows, int64_t cols, int fmt,
                             const float *scale_in, int transpose_out, uint8_t *q,
                             float *scale_inv, float *amax_out, uint64_t *counts)
{
    uint64_t nf = 0, sat = 0;
    float amax = orc_amax_bf16(x, rows * cols, &nf);
    float s = scale_in ? *scale_in : orc_scale_from_amax(amax, fmt);
    float fm = (float)orc_fmax(fmt);
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            uint8_t v = cast_one(x[r * cols + c], s, fmt, fm, &sat);
            if (transpose_out) q[c * rows + r] = v; else q[r * cols + c] = v;
        }
    if (scale_inv) *scale_inv = orc_inverse(s);
    if (amax_out) *amax_out = amax;
    if (counts) { counts[0] += nf; counts[1] += sat; }
}

/* ---------------------------------------------------- rowwise quantize -- */

/* One scale per row of a [rows, cols] tensor (leading dimension ld)
 * ([DeepL] §2.3 per-row; [Soup] rowwise recipe, pow2 scales when pow2 != 0).
 * q is dense [rows, cols]; scale_inv[r] = 1 / s_r.  counts (may be NULL):
 * counts[0] += non-finite inputs, counts[1] += saturated elements, as the
 * tensorwise quantizer counts them ([DeepL] §5.1: overflow and NaN are the
 * failures to watch). */
void orc_quantize_rowwise(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                          int fmt, int pow2, uint8_t *q, float *scale_inv, uint64_t *counts)
{
    float fm = (float)orc_fmax(fmt);
    uint64_t nf = 0, sat = 0;
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t *row = x + r * ld;
        float amax = orc_amax_bf16(row, cols, &nf);
        float s = pow2 ? orc_scale_pow2_from_amax(amax, fmt) : orc_scale_from_amax(amax, fmt);
        for (int64_t c = 0; c < cols; ++c) q[r * cols + c] = cast_one(row[c], s, fmt, fm, &sat);
        scale_inv[r] = orc_inverse(s);
    }
    if (counts) { counts[0] += nf; counts[1] += sat; }
}

/* -------------------------------------------------- blockwise quantize -- */

/* Per-block scaling ([DeepL] §2.3: the tensor is cut into small blocks, each
 * with its own scale).  Blocks are block_rows x 128 (block_rows = 1 for
 * activations, 128 for weights); edge blocks take amax over their valid
 * elements.  q is dense [rows, cols].
 * Scale layout (the GEMM's):
 *   block_rows == 1  : scale_inv[kb * rows + r]            ([ceil(cols/128), rows])
 *   block_rows == 128: scale_inv[rb * ceil(cols/128) + kb] ([ceil(rows/128), ceil(cols/128)])
 * counts (may be NULL): non-finite inputs and saturated elements, added. */
void orc_quantize_blockwise(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                            int fmt, int block_rows, int pow2, uint8_t *q, float *scale_inv,
                            uint64_t *counts)
{
    float fm = (float)orc_fmax(fmt);
    uint64_t nf = 0, sat = 0;
    int64_t nkb = (cols + 127) / 128;
    int64_t nrb = (rows + block_rows - 1) / block_rows;
    for (int64_t rb = 0; rb < nrb; ++rb)
        for (int64_t kb = 0; kb < nkb; ++kb) {
            int64_t r0 = rb * block_rows, r1 = r0 + block_rows;
            int64_t c0 = kb * 128, c1 = c0 + 128;
            if (r1 > rows) r1 = rows;
            if (c1 > cols) c1 = cols;
            float amax = 0.0f;
            for (int64_t r = r0; r < r1; ++r) {
                float a = orc_amax_bf16(x + r * ld + c0, c1 - c0, &nf);
                if (a > amax) amax = a;
            }
            float s = pow2 ? orc_scale_pow2_from_amax(amax, fmt) : orc_scale_from_amax(amax, fmt);
            for (int64_t r = r0; r < r1; ++r)
                for (int64_t c = c0; c < c1; ++c) q[r * cols + c] = cast_one(x[r * ld + c], s, fmt, fm, &sat);
            if (block_rows == 1) scale_inv[kb * rows + rb] = orc_inverse(s);
            else scale_inv[rb * nkb + kb] = orc_inverse(s);
        }
    if (counts) { counts[0] += nf; counts[1] += sat; }
}

/* ------------------------------------------------------------------ GEMM -- */

#define ORC_SCALE_TENSOR 0
#define ORC_SCALE_ROW 1
#define ORC_SCALE_BLOCK 2

/* One output element of the FP8 scaled GEMM D = A8 x B8^T with the scales
 * applied ([H100]: the multiply-accumulate runs on the 8-bit floats; [Soup]:
 * tensorwise / rowwise scaled matmuls; per-block scales from [DeepL] §2.3).
 * A is [M, K] and B is [N, K], both K-contiguous (leading dimension K).
 * Everything is exact products summed in fp64:
 *   tensor: D = da[0] * db[0] * sum_k a*b
 *   row:    D = da[m] * db[n] * sum_k a*b
 *   block:  D = sum_kb da[kb*M + m] * db[(n/128)*nkb + kb] * sum_{k in kb} a*b
 * mag is the same sum over |each scaled product| (the tolerance basis). */
static void gemm_one(const uint8_t *A, int fa, const uint8_t *B, int fb, int64_t M, int64_t N,
                     int64_t K, int mode, const float *da, const float *db, int64_t m, int64_t n,
                     double *val, double *mag)
{
    int64_t nkb = (K + 127) / 128;
    double acc = 0.0, accm = 0.0;
    if (mode == ORC_SCALE_BLOCK) {
        for (int64_t kb = 0; kb < nkb; ++kb) {
            double part = 0.0, partm = 0.0;
            int64_t k1 = (kb + 1) * 128 < K ? (kb + 1) * 128 : K;
            for (int64_t k = kb * 128; k < k1; ++k) {
                double p = orc_decode(A[m * K + k], fa) * orc_decode(B[n * K + k], fb);
                part += p;
                partm += fabs(p);
            }
            double sc = (double)da[kb * M + m] * (double)db[(n / 128) * nkb + kb];
            acc += sc * part;
            accm += fabs(sc) * partm;
        }
    } else {
        for (int64_t k = 0; k < K; ++k) {
            double p = orc_decode(A[m * K + k], fa) * orc_decode(B[n * K + k], fb);
            acc += p;
            accm += fabs(p);
        }
        double sc = (mode == ORC_SCALE_ROW) ? (double)da[m] * (double)db[n]
                                            : (double)da[0] * (double)db[0];
        acc *= sc;
        accm *= fabs(sc);
    }
    *val = acc;
    *mag = accm;
}

/* Full [M, N] reference output (fp64) and magnitudes. */
void orc_gemm_scaled(const uint8_t *A, int fa, const uint8_t *B, int fb, int64_t M, int64_t N,
                     int64_t K, int mode, const float *da, const float *db, double *D, double *mag)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            gemm_one(A, fa, B, fb, M, N, K, mode, da, db, m, n, &D[m * N + n], &mag[m * N + n]);
}

/* Listed output elements only (idx_m[i], idx_n[i]), for sampled checks at
 * sizes where the full product is too slow for a plain CPU loop. */
void orc_gemm_scaled_sampled(const uint8_t *A, int fa, const uint8_t *B, int fb, int64_t M,
                             int64_t N, int64_t K, int mode, const float *da, const float *db,
                             const int64_t *idx_m, const int64_t *idx_n, int64_t count,
                             double *val, double *mag)
{
    for (int64_t i = 0; i < count; ++i)
        gemm_one(A, fa, B, fb, M, N, K, mode, da, db, idx_m[i], idx_n[i], &val[i], &mag[i]);
}

/* The same GEMM accumulated the naive way in fp32 (kept to report how far
 * the tensor cores' fp32 accumulation sits from the plain sequential fp32
 * sum; the fp64 functions above stay the reference).  Each product of two
 * FP8 values is exact in fp32 (at most 4 x 4 significant bits, exponents in
 * range); the sum runs over k in order with one fp32 rounding per addition;
 * block mode sums each 128-wide K block alone, then adds sc * part (sc =
 * da * db rounded to fp32; multiply and add rounded separately); tensor and
 * row modes multiply the whole sum by the fp32 product of the two scales.
 * Returned as fp64 values of the fp32 results. */
static double gemm_one_f32(const uint8_t *A, int fa, const uint8_t *B, int fb, int64_t M, int64_t K,
                           int mode, const float *da, const float *db, int64_t m, int64_t n)
{
    int64_t nkb = (K + 127) / 128;
    float acc = 0.0f;
    if (mode == ORC_SCALE_BLOCK) {
        for (int64_t kb = 0; kb < nkb; ++kb) {
            float part = 0.0f;
            int64_t k1 = (kb + 1) * 128 < K ? (kb + 1) * 128 : K;
            for (int64_t k = kb * 128; k < k1; ++k)
                part += (float)(orc_decode(A[m * K + k], fa) * orc_decode(B[n * K + k], fb));
            float sc = da[kb * M + m] * db[(n / 128) * nkb + kb];
            float t = sc * part;
            acc = acc + t;
        }
    } else {
        for (int64_t k = 0; k < K; ++k)
            acc += (float)(orc_decode(A[m * K + k], fa) * orc_decode(B[n * K + k], fb));
        float sc = (mode == ORC_SCALE_ROW) ? da[m] * db[n] : da[0] * db[0];
        acc = acc * sc;
    }
    return (double)acc;
}

void orc_gemm_scaled_f32acc_sampled(const uint8_t *A, int fa, const uint8_t *B, int fb, int64_t M,
                                    int64_t N, int64_t K, int mode, const float *da, const float *db,
                                    const int64_t *idx_m, const int64_t *idx_n, int64_t count, double *val)
{
    (void)N;
    for (int64_t i = 0; i < count; ++i)
        val[i] = gemm_one_f32(A, fa, B, fb, M, K, mode, da, db, idx_m[i], idx_n[i]);
}

/* ------------------------------------------------------- delayed scaling -- */

/* Delayed-scaling update ([DeepL] §2.3: the scale for this step is predicted
 * from the statistics of the previous steps, and a deviation above a
 * threshold forces a recomputation).  Steps:
 *   saturated = amax_t * s_t > fmax (the scale in use could not hold amax_t);
 *   history[pos] = amax_t; pos = (pos + 1) % len;
 *   m = max(history); s' = fmax / m (m == 0 gives 1); d' = 1 / s'. */
void orc_amax_history_update(float *history, int32_t *pos, int len, float amax_cur, int fmt,
                             float *scale, float *scale_inv, uint32_t *saturated)
{
    float fm = (float)orc_fmax(fmt);
    float s_t = *scale;
    *saturated = (amax_cur * s_t > fm) ? 1u : 0u;
    history[*pos] = amax_cur;
    *pos = (*pos + 1) % len;
    float m = 0.0f;
    for (int i = 0; i < len; ++i)
        if (history[i] > m) m = history[i];
    *scale = orc_scale_from_amax(m, fmt);
    *scale_inv = orc_inverse(*scale);
}

/* ------------------------------------------------------------- KV cache -- */

/* FP8 KV cache ([DeepL] §3.1: K and V stored in FP8, halving memory).
 * x is [B, H, S, Dh] bf16; every (b, h) slice of S*Dh elements gets its own
 * per-tensor scale.  q is the same layout, scale_inv[b*H + h] = 1/s.
 * counts (may be NULL): non-finite inputs and saturated elements, added. */
void orc_kv_quant(const uint16_t *x, int64_t BH, int64_t SD, int fmt, uint8_t *q, float *scale_inv,
                  uint64_t *counts)
{
    float fm = (float)orc_fmax(fmt);
    uint64_t nf = 0, sat = 0;
    for (int64_t i = 0; i < BH; ++i) {
        const uint16_t *sl = x + i * SD;
        float amax = orc_amax_bf16(sl, SD, &nf);
        float s = orc_scale_from_amax(amax, fmt);
        for (int64_t j = 0; j < SD; ++j) q[i * SD + j] = cast_one(sl[j], s, fmt, fm, &sat);
        scale_inv[i] = orc_inverse(s);
    }
    if (counts) { counts[0] += nf; counts[1] += sat; }
}

/* Dequantization when the cache is read: x_hat = bf16(fp32(dec(q)) * d). */
void orc_kv_dequant(const uint8_t *q, const float *scale_inv, int64_t BH, int64_t SD, int fmt,
                    uint16_t *out)
{
    for (int64_t i = 0; i < BH; ++i)
        for (int64_t j = 0; j < SD; ++j) {
            float v = (float)orc_decode(q[i * SD + j], fmt);
            float y = v * scale_inv[i];
            out[i * SD + j] = orc_f32_to_bf16(y);
        }
}

/* ------------------------------------------------------ scale health check -- */

/* Health check of a set of scale factors ([DeepL] §6.2: periodically report
 * the min / max / mean of every layer's scales and watch for step changes,
 * the early sign of outliers or a distribution shift).
 *   valid entries: finite and > 0; stats = {min, max, mean} over them (mean =
 *   fp64 sum / count, rounded to fp32), all 0 when none is valid;
 *   counts[0] = entries whose ratio to prev (both valid) exceeds jump_ratio
 *   in either direction (fp32 divisions), 0 without prev;
 *   counts[1] = invalid entries. */
void orc_scale_stats(const float *s, const float *prev, int64_t n, float jump_ratio, float *stats,
                     uint32_t *counts)
{
    double sum = 0.0;
    float mn = 0.0f, mx = 0.0f;
    int64_t nv = 0;
    uint32_t jumps = 0, invalid = 0;
    for (int64_t i = 0; i < n; ++i) {
        float v = s[i];
        if (!(isfinite(v) && v > 0.0f)) { ++invalid; continue; }
        if (nv == 0 || v < mn) mn = v;
        if (nv == 0 || v > mx) mx = v;
        sum += (double)v;
        ++nv;
        if (prev) {
            float p = prev[i];
            if (isfinite(p) && p > 0.0f && (v / p > jump_ratio || p / v > jump_ratio)) ++jumps;
        }
    }
    stats[0] = mn;
    stats[1] = mx;
    stats[2] = nv ? (float)(sum / (double)nv) : 0.0f;
    counts[0] = jumps;
    counts[1] = invalid;
}

/* ------------------------------------------------------- paged KV cache -- */

/* Paged FP8 KV cache.  The cache is split into fixed-size blocks handed out on
 * demand ("ms-swift全链路能力解析：训练、推理、评测、量化与部署一体化解决方案", vLLM's block
 * KV cache) and stores K / V in FP8 ([DeepL] §3.1).  Tokens arrive a few at a
 * time, so a scale over a whole (sequence, head) slice is not known when a
 * token is written: each (token, head) row of Dh elements gets its own scale.
 *   x     [T, H, Dh] bf16, the new tokens' K (or V);
 *   slot  [T] int64, slot = block * block_size + offset; entries outside
 *         [0, nslots) are padding and write nothing;
 *   cache [nslots, H, Dh] FP8  (= [num_blocks, block_size, H, Dh]);
 *   scale_cache [nslots, H] fp32, 1/s of each written row. */
void orc_paged_kv_write(const uint16_t *x, const int64_t *slot, int64_t T, int64_t H, int64_t Dh,
                        int64_t nslots, int fmt, uint8_t *cache, float *scale_cache)
{
    float fm = (float)orc_fmax(fmt);
    for (int64_t t = 0; t < T; ++t) {
        int64_t sl = slot[t];
        if (sl < 0 || sl >= nslots) continue;
        for (int64_t h = 0; h < H; ++h) {
            const uint16_t *row = x + (t * H + h) * Dh;
            float s = orc_scale_from_amax(orc_amax_bf16(row, Dh, NULL), fmt);
            for (int64_t j = 0; j < Dh; ++j) cache[(sl * H + h) * Dh + j] = cast_one(row[j], s, fmt, fm, NULL);
            scale_cache[sl * H + h] = orc_inverse(s);
        }
    }
}

/* Read a sequence's tokens back through its block table, dequantized:
 *   token t of sequence b lives in block block_table[b][t / block_size] at
 *   offset t % block_size; out[b][t][h][:] = bf16(fp32(dec(q)) * scale_inv).
 *   out [B, S_out, H, Dh] bf16; positions t >= seq_lens[b], past the table's
 *   max_blocks * block_size, or in a block id outside [0, num_blocks) are 0. */
void orc_paged_kv_gather(const uint8_t *cache, const float *scale_cache, const int32_t *block_table,
                         const int32_t *seq_lens, int64_t B, int64_t max_blocks, int64_t H, int64_t Dh,
                         int64_t block_size, int64_t num_blocks, int64_t S_out, int fmt, uint16_t *out)
{
    for (int64_t b = 0; b < B; ++b)
        for (int64_t t = 0; t < S_out; ++t) {
            uint16_t *dst = out + (b * S_out + t) * H * Dh;
            int64_t blk = -1;
            if (t < seq_lens[b] && t / block_size < max_blocks) blk = block_table[b * max_blocks + t / block_size];
            if (blk < 0 || blk >= num_blocks) {
                memset(dst, 0, (size_t)(H * Dh) * sizeof(uint16_t));
                continue;
            }
            int64_t sl = blk * block_size + t % block_size;
            for (int64_t h = 0; h < H; ++h)
                for (int64_t j = 0; j < Dh; ++j) {
                    float v = (float)orc_decode(cache[(sl * H + h) * Dh + j], fmt);
                    dst[h * Dh + j] = orc_f32_to_bf16(v * scale_cache[sl * H + h]);
                }
        }
}

/* ------------------------------------- backward operands and wgrad GEMM -- */

/* Rowwise quantization of the transpose ("FP8训练与QAT量化感知训练：…用Soup
 * 把大模型微调提速2倍", section "FP8 三种缩放配方怎么选": the rowwise recipes
 * scale every row of each GEMM operand).  The backward GEMMs contract over a
 * dimension that is not contiguous in memory -- tokens for the weight
 * gradient dW = dY^T X, output channels for the data gradient dX = dY W --
 * so their K-major operands are transposes: qT[c][r] = cast(x[r][c], s_c)
 * with s_c from the amax of COLUMN c of x (a row of x^T), scale_inv[c] = 1/s_c.
 * x [rows, cols] with leading dimension ld; qT [cols, rows].
 * counts (may be NULL): non-finite inputs and saturated elements, added. */
void orc_quantize_rowwise_transpose(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, int fmt,
                                    int pow2, uint8_t *qT, float *scale_inv, uint64_t *counts)
{
    float fm = (float)orc_fmax(fmt);
    uint64_t nf = 0, sat = 0;
    for (int64_t c = 0; c < cols; ++c) {
        float amax = 0.0f;
        for (int64_t r = 0; r < rows; ++r) {
            uint16_t h = x[r * ld + c];
            if (!bf16_finite(h)) { ++nf; continue; }
            float a = fabsf(bf16_to_f32(h));
            if (a > amax) amax = a;
        }
        float s = pow2 ? orc_scale_pow2_from_amax(amax, fmt) : orc_scale_from_amax(amax, fmt);
        for (int64_t r = 0; r < rows; ++r) qT[c * rows + r] = cast_one(x[r * ld + c], s, fmt, fm, &sat);
        scale_inv[c] = orc_inverse(s);
    }
    if (counts) { counts[0] += nf; counts[1] += sat; }
}

/* Weight gradient kept in high precision (the same section: the
 * rowwise_with_gw_hp recipe keeps the weight-gradient GEMM out of FP8):
 *   dW[m][n] = sum_t dY[t][m] * X[t][n]   over the T token rows,
 * from the bf16 tensors as stored (token-major, dY [T, M], X [T, N]); exact
 * products summed in fp64.  mag[m][n] = sum_t |dY[t][m] * X[t][n]| (the
 * tolerance basis).  Sampled at (idx_m[i], idx_n[i]). */
void orc_gemm_bf16_wgrad_sampled(const uint16_t *dY, const uint16_t *X, int64_t T, int64_t M, int64_t N,
                                 const int64_t *idx_m, const int64_t *idx_n, int64_t count, double *val,
                                 double *mag)
{
    for (int64_t i = 0; i < count; ++i) {
        int64_t m = idx_m[i], n = idx_n[i];
        double acc = 0.0, mg = 0.0;
        for (int64_t t = 0; t < T; ++t) {
            double p = (double)bf16_to_f32(dY[t * M + m]) * (double)bf16_to_f32(X[t * N + n]);
            acc += p;
            mg += fabs(p);
        }
        val[i] = acc;
        mag[i] = mg;
    }
}
