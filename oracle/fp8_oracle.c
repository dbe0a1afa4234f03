/*
 * Plain, slow, single-threaded CPU oracle for FP8 training quantisation of
 * MoE expert GEMMs and for the FP8 scaled grouped GEMM that consumes it.
 *
 * THIS IS TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load it.  It shares no code, header, table
 * or helper with the CUDA library; it is written directly from the format
 * definitions and from the steps the pages list, in their order.
 *
 * Sources (web pages; cited by title and section):
 *  [AIR]  "FP8 su GPU AMD: i guadagni di TorchTitan e TorchAO ora sono nel
 *          mainline PyTorch" (ai-radar.it)
 *         - intro, second paragraph: activations take one scale per row,
 *           expert weights one scale per column, and an int32 tensor of
 *           offsets routes the tokens to the experts.
 *         - section "La correttezza del formato viene prima del tuning":
 *           e4m3fnuz has maximum 240 and no NaN/Inf encodings; scaling against
 *           the wrong maximum clips silently.
 *         - section "Il guadagno vero è nel movimento dei dati", first
 *           paragraph: the chain is absmax per row or column, derivation of
 *           the scale, clamp, cast to FP8.
 *  [ABP]  "AMD Boosts PyTorch FP8 Training on Instinct GPUs", third
 *         paragraph: FNUZ = Finite, No NaN, Unsigned Zero.
 *
 * Readings where the pages are silent (each one also listed in the design
 * notes of the repository):
 *  - e4m3fn (OCP): bias 7, largest finite 448, NaN = S.1111.111, has -0.
 *  - e4m3fnuz: bias 8, largest finite 240 (0x7F), NaN only 0x80, no -0.
 *  - encode = round to nearest, ties to even mantissa, in ONE rounding from
 *    the fp32 value, saturating at the largest finite value (infinities
 *    included); NaN encodes as a NaN code: 0x7F for e4m3fn (0xFF, the other
 *    e4m3fn NaN, is an equally valid result), 0x80 for e4m3fnuz.
 *  - absmax = the largest |x| over the values that are not NaN (a NaN
 *    compares false and is skipped).
 *  - scale s = fp32(fmax / max(amax, 1e-12f)) with IEEE round-to-nearest;
 *    y = fp32(x * s); y is clamped to [-fmax, fmax]; q = encode(y).
 *    The quantisation scale s is what is stored (x ~ decode(q) / s).
 *  - offsets hold E cumulative group ends (no leading zero).  Group e spans
 *    rows [start_e, end_e) with start_0 = 0, start_e = end_{e-1},
 *    end_e = clamp(offsets[e], start_e, rows_total).
 *  - GEMM reference: operands dequantised in fp64 (decode(q)/s), products
 *    summed in fp64; the tolerance is 1e-3 * sum |a||b| per element.
 *
 * Build: plain C11, no fast-math, no FP contraction (see oracle/build.py).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORC_FMT_E4M3FN 0
#define ORC_FMT_E4M3FNUZ 1
#define ORC_LAYOUT_SAME 0
#define ORC_LAYOUT_TRANSPOSED 1

/* exponent bias and largest finite magnitude of each e4m3 variant */
static int fmt_bias(int fmt) { return fmt == ORC_FMT_E4M3FNUZ ? 8 : 7; }
static double fmt_max(int fmt) { return fmt == ORC_FMT_E4M3FNUZ ? 240.0 : 448.0; }

double oracle_fp8_max(int fmt) { return fmt_max(fmt); }

/* Value of an 8-bit code: sign | 4-bit exponent | 3-bit mantissa.
 * Exponent field 0 is subnormal: m/8 * 2^(1-bias); otherwise
 * (1 + m/8) * 2^(e-bias).  NaN codes return NaN. */
double oracle_fp8_decode(uint8_t code, int fmt)
{
    int bias = fmt_bias(fmt);
    int sign = code >> 7;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    if (fmt == ORC_FMT_E4M3FN && (code & 0x7F) == 0x7F) return NAN;
    if (fmt == ORC_FMT_E4M3FNUZ && code == 0x80) return NAN;
    double mag;
    if (e == 0)
        mag = ldexp((double)m, 1 - bias - 3);
    else
        mag = ldexp((double)(8 + m), e - bias - 3);
    return sign ? -mag : mag;
}

/* Round-to-nearest-even encode of an fp32 value onto the finite e4m3 grid,
 * saturating at +-max.  Within one binade the representable magnitudes are
 * consecutive integer multiples of a power-of-two spacing, so rounding the
 * quotient a/spacing to the nearest integer (ties to even) is exactly the
 * mantissa-level RNE; subnormals share the spacing of the first normal
 * binade.  a/spacing is exact in double because a is an fp32 value and the
 * spacing is a power of two. */
uint8_t oracle_fp8_encode(float y, int fmt)
{
    /* NaN (the pages never meet one) goes to a NaN code: 0x7F for e4m3fn
     * (0xFF is NaN too; the sign of a NaN is not portable), 0x80, the only
     * NaN, for e4m3fnuz */
    if (isnan(y)) return (uint8_t)(fmt == ORC_FMT_E4M3FNUZ ? 0x80 : 0x7F);
    int bias = fmt_bias(fmt);
    double maxv = fmt_max(fmt);
    int neg = signbit(y) ? 1 : 0;
    double a = fabs((double)y);
    double min_normal = ldexp(1.0, 1 - bias);
    double sub_step = ldexp(1.0, 1 - bias - 3);
    double step;
    int ex;
    if (a < min_normal) {
        step = sub_step;
    } else {
        (void)frexp(a, &ex);          /* a = f * 2^ex, f in [0.5, 1) */
        step = ldexp(1.0, ex - 1 - 3);  /* binade [2^(ex-1), 2^ex), 8 steps */
    }
    double v = nearbyint(a / step) * step; /* default mode: ties to even */
    if (v > maxv) v = maxv;
    if (v == 0.0) {
        /* e4m3fn keeps the sign of zero; e4m3fnuz has a single zero */
        return (uint8_t)((neg && fmt == ORC_FMT_E4M3FN) ? 0x80 : 0x00);
    }
    unsigned code;
    if (v < min_normal) {
        code = (unsigned)(v / sub_step); /* exponent field 0, mantissa m */
    } else {
        (void)frexp(v, &ex);
        int e = ex - 1 + bias;
        int m = (int)(v / ldexp(1.0, ex - 1 - 3)) - 8;
        code = ((unsigned)e << 3) | (unsigned)m;
    }
    return (uint8_t)(code | (neg ? 0x80u : 0u));
}

static float bf16_to_f32(uint16_t h)
{
    uint32_t bits = (uint32_t)h << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return f;
}

/* The scaling maximum: an explicit override when > 0, else the format's own
 * maximum.  The override exists only to reproduce the format-mismatch case
 * (scaling against 448 while encoding e4m3fnuz, or 240 with e4m3fn). */
static float scaling_max(int fmt, float scale_max)
{
    return scale_max > 0.0f ? scale_max : (float)fmt_max(fmt);
}

/* amax -> scale, step two of the chain */
static float scale_from_amax(float amax, float smax)
{
    const float eps = 1e-12f;
    float a = amax < eps ? eps : amax;
    float s = smax / a; /* IEEE fp32 division, round to nearest */
    return s;
}

/* scale -> clamp -> cast, steps three and four; counts saturation. */
static uint8_t cast_one(float x, float s, float smax, int fmt, float sat_thr,
                        unsigned long long *sat)
{
    float y = x * s; /* fp32 product, round to nearest */
    if (fabsf(y) > sat_thr) (*sat)++;
    if (y > smax) y = smax;
    if (y < -smax) y = -smax;
    return oracle_fp8_encode(y, fmt);
}

/* Elements whose pre-clamp |y| lies more than one fp32 ulp above the
 * encoding's largest finite value are counted as saturated. */
static float saturation_threshold(int fmt)
{
    return nextafterf((float)fmt_max(fmt), INFINITY);
}

/* Rowwise quantisation ([AIR] intro: one scale per activation row).
 * x: bf16 bits [rows, ld_x]; q: codes [rows, ld_q]; scales: [rows]. */
void oracle_quant_rowwise(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld_x,
                          uint8_t *q, int64_t ld_q, float *scales, int fmt,
                          float scale_max, unsigned long long *sat_count)
{
    float smax = scaling_max(fmt, scale_max);
    float thr = saturation_threshold(fmt);
    unsigned long long sat = 0;
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t *xr = x + r * ld_x;
        float amax = 0.0f; /* absmax: exact in fp32 */
        for (int64_t c = 0; c < cols; ++c) {
            float v = fabsf(bf16_to_f32(xr[c]));
            if (v > amax) amax = v;
        }
        float s = scale_from_amax(amax, smax);
        scales[r] = s;
        for (int64_t c = 0; c < cols; ++c)
            q[r * ld_q + c] = cast_one(bf16_to_f32(xr[c]), s, smax, fmt, thr, &sat);
    }
    if (sat_count) *sat_count += sat;
}

/* Group bounds from cumulative ends, clamped so that they are monotone and
 * inside [0, rows_total]. */
void oracle_group_bounds(const int32_t *offsets, int32_t num_groups, int64_t rows_total,
                         int64_t *start, int64_t *end)
{
    int64_t prev = 0;
    for (int32_t e = 0; e < num_groups; ++e) {
        int64_t hi = offsets[e];
        if (hi < prev) hi = prev;
        if (hi > rows_total) hi = rows_total;
        start[e] = prev;
        end[e] = hi;
        prev = hi;
    }
}

/* Jagged column-wise quantisation ([AIR] intro: one scale per column of
 * each expert's block; groups from the offsets tensor).  For every group e
 * and column c the absmax is taken over the group's rows only.
 * layout SAME:       q[r * ld_q + c]
 * layout TRANSPOSED: q[c * ld_q + r]   (the contraction axis of the backward
 *                    GEMM becomes contiguous; no separate transposed copy)
 * scales: [num_groups, cols].  start/end: caller scratch of num_groups. */
void oracle_quant_colwise_jagged(const uint16_t *x, int64_t rows_total, int64_t cols,
                                 int64_t ld_x, const int32_t *offsets, int32_t num_groups,
                                 uint8_t *q, int64_t ld_q, int layout, float *scales, int fmt,
                                 float scale_max, unsigned long long *sat_count,
                                 int64_t *start, int64_t *end)
{
    float smax = scaling_max(fmt, scale_max);
    float thr = saturation_threshold(fmt);
    unsigned long long sat = 0;
    oracle_group_bounds(offsets, num_groups, rows_total, start, end);
    for (int32_t e = 0; e < num_groups; ++e) {
        for (int64_t c = 0; c < cols; ++c) {
            float amax = 0.0f;
            for (int64_t r = start[e]; r < end[e]; ++r) {
                float v = fabsf(bf16_to_f32(x[r * ld_x + c]));
                if (v > amax) amax = v;
            }
            float s = scale_from_amax(amax, smax);
            scales[(int64_t)e * cols + c] = s;
            for (int64_t r = start[e]; r < end[e]; ++r) {
                uint8_t code = cast_one(bf16_to_f32(x[r * ld_x + c]), s, smax, fmt, thr, &sat);
                if (layout == ORC_LAYOUT_TRANSPOSED)
                    q[c * ld_q + r] = code;
                else
                    q[r * ld_q + c] = code;
            }
        }
    }
    if (sat_count) *sat_count += sat;
}

/* FP8 scaled grouped GEMM, token-jagged form (forward and input gradient):
 *   C[m, n] = sum_k (decode(qa[m,k]) / sa[m]) * (decode(qb_e[n,k]) / sb[e,n])
 * where e is the group holding row m.  Evaluated in fp64 at the sample
 * points (rows[i], cols[i]).  Rows outside every group get NaN (the GPU
 * leaves them unwritten).  bound[i] = 1e-3 * sum |a||b|. */
void oracle_gemm_m_jagged_sample(const uint8_t *qa, int64_t ld_a, const float *sa,
                                 const uint8_t *qb, int64_t ld_b, int64_t b_group_stride,
                                 const float *sb, int64_t sb_group_stride,
                                 const int32_t *offsets, int32_t num_groups, int64_t m_total,
                                 int64_t k, int fmt, const int64_t *rows, const int64_t *cols,
                                 int64_t n_samples, double *c_ref, double *bound,
                                 int64_t *start, int64_t *end)
{
    oracle_group_bounds(offsets, num_groups, m_total, start, end);
    for (int64_t i = 0; i < n_samples; ++i) {
        int64_t m = rows[i], n = cols[i];
        int32_t g = -1;
        for (int32_t e = 0; e < num_groups; ++e)
            if (m >= start[e] && m < end[e]) { g = e; break; }
        if (g < 0) { c_ref[i] = NAN; bound[i] = 0.0; continue; }
        double acc = 0.0, mag = 0.0;
        double inv_sa = 1.0 / (double)sa[m];
        double inv_sb = 1.0 / (double)sb[(int64_t)g * sb_group_stride + n];
        const uint8_t *arow = qa + m * ld_a;
        const uint8_t *brow = qb + (int64_t)g * b_group_stride + n * ld_b;
        for (int64_t kk = 0; kk < k; ++kk) {
            double a = oracle_fp8_decode(arow[kk], fmt) * inv_sa;
            double b = oracle_fp8_decode(brow[kk], fmt) * inv_sb;
            acc += a * b;
            mag += fabs(a * b);
        }
        c_ref[i] = acc;
        bound[i] = 1e-3 * mag;
    }
}

/* FP8 scaled grouped GEMM, contraction-jagged form (weight gradient):
 *   C[e, i, j] = sum_{m in group e} (decode(qa[i,m]) / sa[e,i]) * (decode(qb[j,m]) / sb[e,j])
 * qa: [n, ld_a], qb: [k, ld_b], both with the token axis contiguous (the
 * transposed output of the jagged column-wise quantisation).
 * Sample points (grp[i], rows[i], cols[i]).  An empty group gives 0. */
void oracle_gemm_k_jagged_sample(const uint8_t *qa, int64_t ld_a, const float *sa,
                                 int64_t sa_group_stride, const uint8_t *qb, int64_t ld_b,
                                 const float *sb, int64_t sb_group_stride,
                                 const int32_t *offsets, int32_t num_groups, int64_t m_total,
                                 int fmt, const int64_t *grp, const int64_t *rows,
                                 const int64_t *cols, int64_t n_samples, double *c_ref,
                                 double *bound, int64_t *start, int64_t *end)
{
    oracle_group_bounds(offsets, num_groups, m_total, start, end);
    for (int64_t s = 0; s < n_samples; ++s) {
        int64_t e = grp[s], i = rows[s], j = cols[s];
        double inv_sa = 1.0 / (double)sa[e * sa_group_stride + i];
        double inv_sb = 1.0 / (double)sb[e * sb_group_stride + j];
        double acc = 0.0, mag = 0.0;
        for (int64_t m = start[e]; m < end[e]; ++m) {
            double a = oracle_fp8_decode(qa[i * ld_a + m], fmt) * inv_sa;
            double b = oracle_fp8_decode(qb[j * ld_b + m], fmt) * inv_sb;
            acc += a * b;
            mag += fabs(a * b);
        }
        c_ref[s] = acc;
        bound[s] = 1e-3 * mag;
    }
}

/* The encoder applied to every element of an fp32 array (plain loop). */
void oracle_fp8_encode_array(const float *y, int64_t n, uint8_t *q, int fmt)
{
    for (int64_t i = 0; i < n; ++i) q[i] = oracle_fp8_encode(y[i], fmt);
}

/* ------------------------------------------------------------------------
 * MXFP8: microscaled FP8 ("AMD Primus adds FP8/MXFP8 kernels ...", section
 * "What Primus adds for MoE training on MI355X": MXFP8 grouped GEMM and
 * quantisation kernels; "AMD Boosts PyTorch FP8 Training on Instinct GPUs",
 * last paragraph; "FP8 su GPU AMD ...", section "Cosa significa per chi
 * gestisce cluster locali": MXFP8 as the next, finer-grained format).
 * The pages name the format and do not define it; the reading taken is the
 * OCP Microscaling Formats (MX) v1.0 definition of MXFP8 with e4m3 elements:
 *  - a block is 32 consecutive elements along the contraction axis;
 *  - its shared scale is X = 2^E, E = floor(log2(amax)) - 8 (8 = the
 *    exponent of e4m3fn's largest normal binade), stored as the E8M0 byte
 *    E + 127, E clamped to [-127, 127];
 *  - element code = encode(x / X): the quotient is clamped to +-448 and
 *    rounded to nearest even (the e4m3fn encoder above);
 *  - value = decode(code) * X.
 * Readings for the cases the definition leaves open (same as the per-row
 * path where they overlap): amax skips NaN; an all-zero (or all-NaN) block
 * takes E = -127; an infinite amax takes E = 127.
 * ------------------------------------------------------------------------ */

/* E of a block from its absmax (an exact fp32 value). */
static int mx_exponent(float amax)
{
    if (!(amax > 0.0f)) return -127;
    if (isinf(amax)) return 127;
    int ex;
    (void)frexp((double)amax, &ex); /* amax = f * 2^ex, f in [0.5, 1): floor(log2) = ex - 1 */
    int e = ex - 1 - 8;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

/* Code of one element of a block with exponent e: x / 2^e is exact in
 * double; as an fp32 value it is exact too wherever it can reach a nonzero
 * code (a bf16 value times a power of two keeps its 8 significant bits, and
 * magnitudes from 2^-10 up lie in fp32's normal range). */
static uint8_t mx_encode_one(float x, int e)
{
    double y = ldexp((double)x, -e);
    if (y > 448.0) y = 448.0;
    if (y < -448.0) y = -448.0;
    return oracle_fp8_encode((float)y, ORC_FMT_E4M3FN);
}

/* Scale byte of the block x[0], x[stride], ... (n <= 32 elements; the
 * missing ones of a partial block count as zeros). */
static uint8_t mx_block_scale(const uint16_t *x, int64_t stride, int64_t n, int *e_out)
{
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float v = fabsf(bf16_to_f32(x[i * stride]));
        if (v > amax) amax = v;
    }
    int e = mx_exponent(amax);
    *e_out = e;
    return (uint8_t)(e + 127);
}

/* MX quantisation along rows: blocks of 32 consecutive columns.
 * x: bf16 bits [rows, ld_x], cols a multiple of 32; q: codes [rows, ld_q];
 * sc: E8M0 bytes [rows, ld_s], sc[r, b] for columns [32b, 32b + 32). */
void oracle_mx_quant_rowwise(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld_x,
                             uint8_t *q, int64_t ld_q, uint8_t *sc, int64_t ld_s)
{
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < cols / 32; ++b) {
            const uint16_t *xb = x + r * ld_x + 32 * b;
            int e;
            sc[r * ld_s + b] = mx_block_scale(xb, 1, 32, &e);
            for (int64_t i = 0; i < 32; ++i)
                q[r * ld_q + 32 * b + i] = mx_encode_one(bf16_to_f32(xb[i]), e);
        }
    }
}

/* Padded start of each group: P_0 = 0, P_e = sum_{j<e} round_up(size_j, 128). */
static void padded_starts(const int64_t *start, const int64_t *end, int32_t num_groups,
                          int64_t *pstart)
{
    int64_t p = 0;
    for (int32_t e = 0; e < num_groups; ++e) {
        pstart[e] = p;
        p += (end[e] - start[e] + 127) / 128 * 128;
    }
}

/* MX quantisation along the tokens of each expert group, written transposed
 * in the padded layout: column c, token t of group e (t < size_e) goes to
 * q[c, P_e + t]; the tokens [size_e, round_up(size_e, 128)) hold zero codes.
 * Blocks are 32 consecutive tokens from the group's start; a group's last
 * block may be partial (its missing tokens are the zero padding).  Scales:
 * sc[c, P_e / 32 + b] for the group's blocks b < round_up(size_e, 128) / 32
 * (padding-only blocks: amax 0, E = -127).  Tokens past the last group are
 * not written.  start/end/pstart: caller scratch of num_groups. */
void oracle_mx_quant_colwise_padded(const uint16_t *x, int64_t rows_total, int64_t cols,
                                    int64_t ld_x, const int32_t *offsets, int32_t num_groups,
                                    uint8_t *q, int64_t ld_q, uint8_t *sc, int64_t ld_s,
                                    int64_t *start, int64_t *end, int64_t *pstart)
{
    oracle_group_bounds(offsets, num_groups, rows_total, start, end);
    padded_starts(start, end, num_groups, pstart);
    for (int32_t g = 0; g < num_groups; ++g) {
        int64_t size = end[g] - start[g];
        int64_t padded = (size + 127) / 128 * 128;
        for (int64_t c = 0; c < cols; ++c) {
            for (int64_t b = 0; b < padded / 32; ++b) {
                int64_t t0 = 32 * b;
                int64_t n = size - t0;
                if (n > 32) n = 32;
                if (n < 0) n = 0;
                int e;
                sc[c * ld_s + pstart[g] / 32 + b] =
                    mx_block_scale(x + (start[g] + t0) * ld_x + c, ld_x, n, &e);
                for (int64_t i = 0; i < 32; ++i) {
                    int64_t t = t0 + i;
                    q[c * ld_q + pstart[g] + t] =
                        t < size ? mx_encode_one(bf16_to_f32(x[(start[g] + t) * ld_x + c]), e)
                                 : (uint8_t)0;
                }
            }
        }
    }
}

/* Value of an MX element: decode(code) * 2^(scale byte - 127). */
static double mx_value(uint8_t code, uint8_t scale)
{
    return ldexp(oracle_fp8_decode(code, ORC_FMT_E4M3FN), (int)scale - 127);
}

/* MX grouped GEMM, token-jagged form:
 *   C[m, n] = sum_k value(qa[m,k], sa[m, k/32]) * value(qb_e[n,k], sb_e[n, k/32])
 * with e the group of row m; fp64 at the sample points; rows outside every
 * group give NaN.  bound[i] = 1e-3 * sum |a||b|. */
void oracle_mx_gemm_m_jagged_sample(const uint8_t *qa, int64_t ld_a, const uint8_t *sa,
                                    int64_t ld_sa, const uint8_t *qb, int64_t ld_b,
                                    int64_t b_group_stride, const uint8_t *sb, int64_t ld_sb,
                                    int64_t sb_group_stride, const int32_t *offsets,
                                    int32_t num_groups, int64_t m_total, int64_t k,
                                    const int64_t *rows, const int64_t *cols, int64_t n_samples,
                                    double *c_ref, double *bound, int64_t *start, int64_t *end)
{
    oracle_group_bounds(offsets, num_groups, m_total, start, end);
    for (int64_t i = 0; i < n_samples; ++i) {
        int64_t m = rows[i], n = cols[i];
        int32_t g = -1;
        for (int32_t e = 0; e < num_groups; ++e)
            if (m >= start[e] && m < end[e]) { g = e; break; }
        if (g < 0) { c_ref[i] = NAN; bound[i] = 0.0; continue; }
        const uint8_t *arow = qa + m * ld_a;
        const uint8_t *asc = sa + m * ld_sa;
        const uint8_t *brow = qb + (int64_t)g * b_group_stride + n * ld_b;
        const uint8_t *bsc = sb + (int64_t)g * sb_group_stride + n * ld_sb;
        double acc = 0.0, mag = 0.0;
        for (int64_t kk = 0; kk < k; ++kk) {
            double a = mx_value(arow[kk], asc[kk / 32]);
            double b = mx_value(brow[kk], bsc[kk / 32]);
            acc += a * b;
            mag += fabs(a * b);
        }
        c_ref[i] = acc;
        bound[i] = 1e-3 * mag;
    }
}

/* MX grouped GEMM, contraction-jagged form on the padded transposed layout
 * (weight gradient):
 *   C[e, i, j] = sum_{t < size_e} value(qa[i, P_e + t], sa[i, (P_e + t)/32])
 *                                 * value(qb[j, P_e + t], sb[j, (P_e + t)/32])
 * Sample points (grp[s], rows[s], cols[s]); an empty group gives 0. */
void oracle_mx_gemm_k_jagged_padded_sample(const uint8_t *qa, int64_t ld_a, const uint8_t *sa,
                                           int64_t ld_sa, const uint8_t *qb, int64_t ld_b,
                                           const uint8_t *sb, int64_t ld_sb,
                                           const int32_t *offsets, int32_t num_groups,
                                           int64_t m_total, const int64_t *grp,
                                           const int64_t *rows, const int64_t *cols,
                                           int64_t n_samples, double *c_ref, double *bound,
                                           int64_t *start, int64_t *end, int64_t *pstart)
{
    oracle_group_bounds(offsets, num_groups, m_total, start, end);
    padded_starts(start, end, num_groups, pstart);
    for (int64_t s = 0; s < n_samples; ++s) {
        int64_t e = grp[s], i = rows[s], j = cols[s];
        double acc = 0.0, mag = 0.0;
        for (int64_t t = pstart[e]; t < pstart[e] + (end[e] - start[e]); ++t) {
            double a = mx_value(qa[i * ld_a + t], sa[i * ld_sa + t / 32]);
            double b = mx_value(qb[j * ld_b + t], sb[j * ld_sb + t / 32]);
            acc += a * b;
            mag += fabs(a * b);
        }
        c_ref[s] = acc;
        bound[s] = 1e-3 * mag;
    }
}
