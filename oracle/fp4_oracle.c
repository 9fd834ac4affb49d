/*
 * fp4_oracle.c -- plain, slow CPU oracle for block-scaled 4-bit quantization.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or constant with the
 * CUDA library: every format below is enumerated here from its definition.
 *
 * Sources (web pages; cited by title and section):
 *   [NVFP4]  "Why Gated DeltaNet Survives 4-Bit Quantization: NVFP4 W4A4 ..."
 *            review, section 1 (Key Terms): NVFP4 = E2M1 values, one E4M3
 *            scale per 16 elements.
 *   [RaZeR]  "RaZeR - Redundant Zero Remapping" technical summary,
 *            section 1 (the E2M1 value set, the always-positive scale),
 *            section 2.1 (E3M3 weight scales, E4M3 activation scales),
 *            section 2.2 (remapping -0 to a per-block special value chosen
 *            by minimum mean squared error).
 *   [MACaQ]  "MACaQ: Fast, Model Agnostic Calibrated Quantization ..."
 *            review, section 1 (MXFP4, online scaling and micro-rotation,
 *            Hessian-weighted exponent selection, Flip-Refinement) and
 *            section 3 (Method).
 *   [Finer]  "Finer is Better (with the Right Scaling)" summary,
 *            Methodology items 1-2 (abs-max, prevent-zero, 4-over-6,
 *            brute force, hierarchical scaling).
 *
 * The pages fix the formats and name the rules but give no arithmetic.  The
 * readings taken here (all decisions in IEEE fp32 round-to-nearest-even, the
 * per-block squared error accumulated with fmaf in element order) are listed
 * in the repository's design notes.  This file must be compiled with
 * -ffp-contract=off and without fast-math so that every expression below is
 * exactly the sequence of fp32 roundings it spells out.
 *
 * Parity status: every function here is pinned by a CPU test against a
 * property the pages or the mathematics fix (see tests/test_oracle_*.py).
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* Formats                                                             */
/* ------------------------------------------------------------------ */

/* E2M1 magnitudes, [RaZeR] section 1: {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
 * Code = sign << 3 | magnitude index. */
static const float E2M1_MAG[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

float oracle_e2m1_value(int code)
{
    float m = E2M1_MAG[code & 7];
    return (code & 8) ? -m : m;
}

/* Nearest E2M1 magnitude index to a >= 0; ties go to the even index;
 * anything at or above 6 (including +inf) saturates to index 7. */
static int e2m1_nearest_mag(float a)
{
    if (!(a < 6.0f))
        return 7;
    for (int m = 0; m < 7; ++m) {
        double twice_mid = (double)E2M1_MAG[m] + (double)E2M1_MAG[m + 1];
        double twice_a = 2.0 * (double)a;   /* exact */
        if (twice_a < twice_mid)
            return m;
        if (twice_a == twice_mid)
            return (m % 2 == 0) ? m : m + 1;
    }
    return 7;
}

int oracle_e2m1_encode(float y)
{
    return (signbit(y) ? 8 : 0) | e2m1_nearest_mag(fabsf(y));
}

/* OCP E4M3 (FN): 1 sign, 4 exponent (bias 7), 3 mantissa bits; exponent
 * field 0 is subnormal; 0x7F / 0xFF are NaN, so the largest finite is 448.
 * Only the non-negative half is used for scales ([RaZeR] section 1). */
float oracle_e4m3_value(int code)
{
    int e = (code >> 3) & 0xF, m = code & 7;
    double v = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return (float)((code & 0x80) ? -v : v);
}

/* E3M3, [RaZeR] section 2.1: a 6-bit unsigned scale, 3 exponent bits
 * (bias 3) and 3 mantissa bits, exponent field 0 subnormal, no NaN/Inf
 * codes.  Values 2^-5 ... 30. */
float oracle_e3m3_value(int code)
{
    int e = (code >> 3) & 7, m = code & 7;
    double v = (e == 0) ? ldexp((double)m / 8.0, -2) : ldexp(1.0 + (double)m / 8.0, e - 3);
    return (float)v;
}

/* E8M0 (MX shared scale, [MACaQ] section 1): value 2^(byte-127); 0xFF NaN. */
double oracle_e8m0_value(int byte) { return ldexp(1.0, byte - 127); }

/* Round a non-negative r to the nearest value of an ascending code table
 * value(0..last), ties to the even code, saturating at value(last). */
static int nearest_code(float r, float (*value)(int), int last)
{
    if (!(r < value(last)))
        return last;
    for (int c = 0; c < last; ++c) {
        double lo = value(c), hi = value(c + 1);
        if ((double)r < hi) {
            double twice_r = 2.0 * (double)r, twice_mid = lo + hi;   /* exact */
            if (twice_r < twice_mid)
                return c;
            if (twice_r > twice_mid)
                return c + 1;
            return (c % 2 == 0) ? c : c + 1;
        }
    }
    return last;
}

int oracle_e4m3_encode(float r) { return nearest_code(r, oracle_e4m3_value, 0x7E); }
int oracle_e3m3_encode(float r) { return nearest_code(r, oracle_e3m3_value, 63); }

/* UE5M3, the wide-exponent block scale [Finer] compares E4M3 + 4-over-6 +
 * hierarchical scaling against (findings: format compatibility; the page
 * gives no bit layout).  Read as an unsigned 8-bit float: 5 exponent bits
 * with bias 15 over 3 mantissa bits, subnormals at exponent 0, and -- as in
 * the OCP E4M3FN convention -- the all-ones code not a number, so codes
 * 0..254 span 0, 2^-17 .. 1.75 * 2^16 = 114688. */
float oracle_ue5m3_value(int code)
{
    int e = (code >> 3) & 31, m = code & 7;
    if (e == 0)
        return ldexpf((float)m, -17);
    return ldexpf(1.0f + (float)m / 8.0f, e - 15);
}

int oracle_ue5m3_encode(float r) { return nearest_code(r, oracle_ue5m3_value, 0xFE); }

/* ------------------------------------------------------------------ */
/* Shared pieces of the NVFP4 / RaZeR quantizers                        */
/* ------------------------------------------------------------------ */

enum { SF_E4M3 = 0, SF_E3M3 = 1, SF_E8M0 = 2, SF_UE5M3 = 3 };
enum { RULE_ABSMAX = 0, RULE_PREVENT_ZERO = 1, RULE_FOUR_OVER_SIX = 2,
       RULE_BRUTE_FORCE = 3, RULE_HESSIAN_EXP = 4 };

/* Largest finite scale of each format (448 for E4M3, 30 for E3M3). */
static float scale_max(int sf)
{
    if (sf == SF_UE5M3)
        return 114688.0f;
    return sf == SF_E3M3 ? 30.0f : 448.0f;
}

/* Per-tensor FP32 global scale of hierarchical scaling ([Finer] method 2):
 * g = amax / (6 * S_max), so that the largest block maps to the largest
 * scale.  A tensor of zeros (or one so small that g underflows) gets g = 1. */
float oracle_global_scale(float amax, int sf)
{
    float denom = 6.0f * scale_max(sf);
    float g = amax / denom;
    if (!(g > 0.0f))
        g = 1.0f;
    return g;
}

float oracle_amax(const float *x, int64_t n)
{
    float a = 0.0f;
    for (int64_t i = 0; i < n; ++i)
        a = fmaxf(a, fabsf(x[i]));
    return a;
}

/* Quantize one block of n elements with the decoded block-scale value sc and
 * global scale g.  If special is non-NULL this is a RaZeR block: the -0 code
 * stands for *special instead of zero.  Writes the unpacked 4-bit codes and
 * the dequantized values; returns the block's squared error accumulated in
 * element order (the decision metric of every rule). */
static float quantize_block(const float *x, int n, float sc, float g,
                            const float *special, uint8_t *code, float *deq)
{
    float S = sc * g;                                       /* effective scale */
    float inv = (S == 0.0f) ? 0.0f : fminf(1.0f / S, FLT_MAX);
    float acc = 0.0f;
    for (int i = 0; i < n; ++i) {
        float y = x[i] * inv;
        int m = e2m1_nearest_mag(fabsf(y));
        int c = (signbit(y) ? 8 : 0) | m;
        float v = oracle_e2m1_value(c);
        if (special) {
            /* [RaZeR] 2.2: -0 is no longer a zero.  Values that round to
             * zero take +0; a value takes the special code when the special
             * value (same sign) is strictly nearer than the E2M1 neighbour. */
            if (m == 0) {
                c = 0;
                v = 0.0f;
            } else if (signbit(y) == signbit(*special)) {
                float ay = fabsf(y);
                float d_special = fabsf(ay - fabsf(*special));
                float d_grid = fabsf(ay - E2M1_MAG[m]);
                if (d_special < d_grid) {
                    c = 8;
                    v = *special;
                }
            }
        }
        float d = v * S;
        float e = x[i] - d;
        acc = fmaf(e, e, acc);
        code[i] = (uint8_t)c;
        deq[i] = d;
    }
    return acc;
}

static float block_absmax(const float *x, int n)
{
    float a = 0.0f;
    for (int i = 0; i < n; ++i)
        a = fmaxf(a, fabsf(x[i]));
    return a;
}

/* Abs-max scale target ([Finer] method 2, standard abs-max): the block max
 * divided by M times the global scale, rounded to the scale format. */
static int absmax_scale_code(float a, float M, float g, int sf)
{
    float r = a / (M * g);
    if (sf == SF_UE5M3)
        return oracle_ue5m3_encode(r);
    return sf == SF_E3M3 ? oracle_e3m3_encode(r) : oracle_e4m3_encode(r);
}

static float scale_value(int code, int sf)
{
    if (sf == SF_UE5M3)
        return oracle_ue5m3_value(code);
    return sf == SF_E3M3 ? oracle_e3m3_value(code) : oracle_e4m3_value(code);
}

static void pack_codes(const uint8_t *c, int n, uint8_t *out)
{
    for (int i = 0; i < n; i += 2)
        out[i / 2] = (uint8_t)((c[i] & 0xF) | ((c[i + 1] & 0xF) << 4));
}

/* ------------------------------------------------------------------ */
/* NVFP4 block-scaled quantization with a choice of scale rule          */
/* ------------------------------------------------------------------ */

/* x: rows x cols fp32 row-major; blocks of `block` contiguous elements along
 * a row.  Outputs: codes (rows*cols/2 bytes, element 2i in the low nibble),
 * scales (rows*cols/block E4M3 bytes, row-major), deq and mse (nullable).
 * Returns 0, or -1 on a bad argument. */
int oracle_block_fp4_quantize(const float *x, int64_t rows, int64_t cols, int block, int rule,
                              int sf, float g, uint8_t *codes, uint8_t *scales, float *deq,
                              float *mse);

int oracle_nvfp4_quantize(const float *x, int64_t rows, int64_t cols, int block,
                          int rule, float g, uint8_t *codes, uint8_t *scales,
                          float *deq, float *mse)
{
    return oracle_block_fp4_quantize(x, rows, cols, block, rule, SF_E4M3, g, codes, scales, deq,
                                     mse);
}

/* The same with the scale format as a parameter: SF_E4M3 (NVFP4) or
 * SF_UE5M3; the rules are unchanged, brute force runs over every finite
 * positive code of the format in ascending order. */
int oracle_block_fp4_quantize(const float *x, int64_t rows, int64_t cols, int block, int rule,
                              int sf, float g, uint8_t *codes, uint8_t *scales, float *deq,
                              float *mse)
{
    if (block != 4 && block != 8 && block != 16 && block != 32)
        return -1;
    if (sf != SF_E4M3 && sf != SF_UE5M3)
        return -1;
    const int last = sf == SF_UE5M3 ? 0xFE : 0x7E;
    if (cols % block != 0 || rule < RULE_ABSMAX || rule > RULE_BRUTE_FORCE)
        return -1;
    const int64_t nblk = rows * (cols / block);
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nblk; ++b) {
        const float *xb = x + b * block;
        uint8_t cbest[32], ctry[32];
        float dbest[32], dtry[32];
        float a = block_absmax(xb, block);
        int sc_code;
        float sse;
        if (rule == RULE_ABSMAX || rule == RULE_PREVENT_ZERO) {
            sc_code = absmax_scale_code(a, 6.0f, g, sf);
            if (rule == RULE_PREVENT_ZERO && sc_code == 0)
                sc_code = 1;     /* smallest positive scale (E4M3: 2^-9) */
            sse = quantize_block(xb, block, scale_value(sc_code, sf), g, NULL, cbest, dbest);
        } else if (rule == RULE_FOUR_OVER_SIX) {
            int c6 = absmax_scale_code(a, 6.0f, g, sf);
            int c4 = absmax_scale_code(a, 4.0f, g, sf);
            float sse6 = quantize_block(xb, block, scale_value(c6, sf), g, NULL, cbest, dbest);
            float sse4 = quantize_block(xb, block, scale_value(c4, sf), g, NULL, ctry, dtry);
            sc_code = c6;
            sse = sse6;
            if (sse4 < sse6) {
                sc_code = c4;
                sse = sse4;
                memcpy(cbest, ctry, sizeof cbest);
                memcpy(dbest, dtry, sizeof dbest);
            }
        } else { /* brute force: every finite positive scale, ascending */
            sc_code = -1;
            sse = 0.0f;
            for (int c = 1; c <= last; ++c) {
                float s = quantize_block(xb, block, scale_value(c, sf), g, NULL, ctry, dtry);
                if (sc_code < 0 || s < sse) {
                    sc_code = c;
                    sse = s;
                    memcpy(cbest, ctry, sizeof cbest);
                    memcpy(dbest, dtry, sizeof dbest);
                }
            }
        }
        pack_codes(cbest, block, codes + b * (block / 2));
        scales[b] = (uint8_t)sc_code;
        if (deq)
            memcpy(deq + b * block, dbest, (size_t)block * sizeof(float));
        if (mse)
            mse[b] = sse * (1.0f / (float)block);
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* RaZeR: redundant-zero remapping, blocks of 16                        */
/* ------------------------------------------------------------------ */

/* sf = SF_E3M3 (weights: 6-bit scale, 2 selector bits, 4 specials) or
 * SF_E4M3 (activations: 8-bit scale whose sign bit selects one of 2
 * specials).  Scale = abs-max in that format.  For each special value the
 * block is quantized and scored by its squared error; the lowest wins, ties
 * to the earlier table entry.  meta byte = sel << 6 | e3m3  or
 * sel << 7 | e4m3. */
int oracle_razer_quantize(const float *x, int64_t rows, int64_t cols, int sf,
                          const float *specials, int n_special, float g,
                          uint8_t *codes, uint8_t *meta, float *deq, float *mse)
{
    const int B = 16;
    if (cols % B != 0)
        return -1;
    if (!((sf == SF_E3M3 && n_special >= 1 && n_special <= 4) ||
          (sf == SF_E4M3 && n_special >= 1 && n_special <= 2)))
        return -1;
    const int64_t nblk = rows * (cols / B);
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nblk; ++b) {
        const float *xb = x + b * B;
        uint8_t cbest[16], ctry[16];
        float dbest[16], dtry[16];
        float a = block_absmax(xb, B);
        int sc_code = absmax_scale_code(a, 6.0f, g, sf);
        float sc = scale_value(sc_code, sf);
        int sel = -1;
        float sse = 0.0f;
        for (int k = 0; k < n_special; ++k) {
            float s = quantize_block(xb, B, sc, g, &specials[k], ctry, dtry);
            if (sel < 0 || s < sse) {
                sel = k;
                sse = s;
                memcpy(cbest, ctry, sizeof cbest);
                memcpy(dbest, dtry, sizeof dbest);
            }
        }
        pack_codes(cbest, B, codes + b * (B / 2));
        meta[b] = (uint8_t)(sf == SF_E3M3 ? (sel << 6) | sc_code : (sel << 7) | sc_code);
        if (deq)
            memcpy(deq + b * B, dbest, sizeof dbest);
        if (mse)
            mse[b] = sse * (1.0f / 16.0f);
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* MXFP4 with online scaling and size-32 block-Hadamard ([MACaQ])       */
/* ------------------------------------------------------------------ */

/* fp32 nearest to 1/sqrt(32) = 2^-2.5, the normalisation of H_32. */
static float hadamard32_norm(void) { return (float)(1.0 / sqrt(32.0)); }

/* Online transform of one row: u_j = x_j * t_j (if t given), then per
 * 32-column block the Sylvester Hadamard butterflies for strides
 * 1, 2, 4, 8, 16, then the 1/sqrt(32) normalisation ([MACaQ] section 1,
 * "Online Scaling & Micro-Rotation"). */
static void transform_row(const float *x, int64_t cols, const float *t, int hadamard, float *u)
{
    for (int64_t j = 0; j < cols; ++j)
        u[j] = t ? x[j] * t[j] : x[j];
    if (!hadamard)
        return;
    const float c = hadamard32_norm();
    for (int64_t k = 0; k < cols; k += 32) {
        float *v = u + k;
        for (int h = 1; h < 32; h <<= 1)
            for (int i = 0; i < 32; ++i)
                if ((i & h) == 0) {
                    float p = v[i], q = v[i + h];
                    v[i] = p + q;
                    v[i + h] = p - q;
                }
        for (int i = 0; i < 32; ++i)
            v[i] = v[i] * c;
    }
}

int oracle_mx_transform(const float *x, int64_t rows, int64_t cols, const float *t,
                        int hadamard, float *out)
{
    if (cols % 32 != 0)
        return -1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        transform_row(x + r * cols, cols, t, hadamard, out + r * cols);
    return 0;
}

/* OCP MX shared exponent: floor(log2(block max)) minus 2 (the largest E2M1
 * exponent), clamped to the E8M0 range; an all-zero block gets -127. */
static int mx_standard_exponent(float a)
{
    if (a == 0.0f)
        return -127;
    int e = ilogbf(a) - 2;
    return e < -127 ? -127 : (e > 127 ? 127 : e);
}

/* One MX block with exponent e: codes, dequantized values, ordered SSE. */
static float mx_block(const float *y, int e, uint8_t *code, float *deq)
{
    float acc = 0.0f;
    for (int i = 0; i < 32; ++i) {
        float q = ldexpf(y[i], -e);
        int c = oracle_e2m1_encode(q);
        float d = ldexpf(oracle_e2m1_value(c), e);
        float err = y[i] - d;
        acc = fmaf(err, err, acc);
        code[i] = (uint8_t)c;
        deq[i] = d;
    }
    return acc;
}

/* Hessian-weighted error d^T H d of a block error d under the 32x32 block
 * H (row-major), accumulated in order: v_i = sum_j H_ij d_j, then
 * sum_i d_i v_i ([MACaQ] section 1, Hessian-Weighted Exponent Selection). */
static float hessian_cost(const float *H, const float *d)
{
    float cost = 0.0f;
    for (int i = 0; i < 32; ++i) {
        float v = 0.0f;
        for (int j = 0; j < 32; ++j)
            v = fmaf(H[i * 32 + j], d[j], v);
        cost = fmaf(d[i], v, cost);
    }
    return cost;
}

/* x: rows x cols fp32; t: per-column scale (nullable); hadamard: apply the
 * block rotation; rule: RULE_ABSMAX (OCP exponent) or RULE_HESSIAN_EXP
 * (offsets 0, +1, -1 around it, scored by d^T H'_k d with hess holding
 * cols/32 blocks of 32x32 fp32).  Outputs codes, E8M0 bytes, deq and mse
 * (both in the transformed domain, nullable). */
int oracle_mxfp4_quantize(const float *x, int64_t rows, int64_t cols, const float *t,
                          int hadamard, int rule, const float *hess, uint8_t *codes,
                          uint8_t *scales, float *deq, float *mse)
{
    if (cols % 32 != 0 || (rule != RULE_ABSMAX && rule != RULE_HESSIAN_EXP))
        return -1;
    if (rule == RULE_HESSIAN_EXP && !hess)
        return -1;
    const int64_t kb = cols / 32;
    int bad = 0;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        float *u = (float *)malloc((size_t)cols * sizeof(float));
        if (!u) {
#pragma omp atomic write
            bad = 1;
            continue;
        }
        transform_row(x + r * cols, cols, t, hadamard, u);
        for (int64_t k = 0; k < kb; ++k) {
            const float *y = u + k * 32;
            uint8_t cbest[32], ctry[32];
            float dbest[32], dtry[32], err[32];
            int e0 = mx_standard_exponent(block_absmax(y, 32));
            int e = e0;
            float sse = mx_block(y, e0, cbest, dbest);
            if (rule == RULE_HESSIAN_EXP) {
                const int offsets[3] = {0, 1, -1};
                float best = 0.0f;
                int have = 0;
                for (int o = 0; o < 3; ++o) {
                    int ec = e0 + offsets[o];
                    if (ec < -127 || ec > 127)
                        continue;
                    float s = mx_block(y, ec, ctry, dtry);
                    for (int i = 0; i < 32; ++i)
                        err[i] = y[i] - dtry[i];
                    float cost = hessian_cost(hess + k * 1024, err);
                    if (!have || cost < best) {
                        have = 1;
                        best = cost;
                        e = ec;
                        sse = s;
                        memcpy(cbest, ctry, sizeof cbest);
                        memcpy(dbest, dtry, sizeof dbest);
                    }
                }
            }
            int64_t b = r * kb + k;
            pack_codes(cbest, 32, codes + b * 16);
            scales[b] = (uint8_t)(e + 127);
            if (deq)
                memcpy(deq + b * 32, dbest, sizeof dbest);
            if (mse)
                mse[b] = sse * (1.0f / 32.0f);
        }
        free(u);
    }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------ */
/* Flip-Refinement ([MACaQ] section 1 Key Terms, section 3 Method)      */
/* ------------------------------------------------------------------ */

/* The E2M1 values in increasing order as one ladder of 15 levels (+0 and
 * -0 are the same level, index 7).  A move takes one element to the
 * neighbouring level below or above. */
static int e2m1_level(int code)
{
    int m = code & 7;
    return (code & 8) ? 7 - m : 7 + m;
}

static int e2m1_code_of_level(int level)
{
    return level >= 7 ? level - 7 : (8 | (7 - level));
}

/* Starting from the codes of an MX quantization (exponents fixed), each
 * output row runs a greedy coordinate descent on
 *   f = sum_k d_k^T H'_k d_k,   d = u - deq(codes),
 * u the transformed row and H'_k the 32x32 diagonal blocks of the layer
 * Hessian.  A step evaluates, for every element i and both neighbouring
 * levels, the closed-form decrease of f when the element's dequantized value
 * moves by D = (v' - v) 2^e:
 *   gain = 2 D g_i - D^2 H_ii,   g = H' d   (the block's gradient / 2),
 * takes the largest gain if it is positive (ties: lowest element, then the
 * downward move), updates the code, and updates the block's g in place:
 *   g_j <- g_j - D H_ji.
 * A row stops after max_moves accepted moves or when no move has a
 * positive gain.  g starts as the fma chain v_i = sum_j H_ij d_j in j order
 * (the exponent selection's order); gain = 2*(D*g_i) - (D*D)*H_ii with each
 * product and the difference rounded to fp32.  codes are updated in place;
 * moves (nullable) receives the accepted move count per row. */
int oracle_mxfp4_flip_refine(const float *x, int64_t rows, int64_t cols, const float *t,
                             int hadamard, const float *hess, int max_moves, uint8_t *codes,
                             const uint8_t *scales, int32_t *moves)
{
    if (cols % 32 != 0 || !hess || max_moves < 0)
        return -1;
    const int64_t kb = cols / 32;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        float *u = (float *)malloc((size_t)cols * sizeof(float));
        float *g = (float *)malloc((size_t)cols * sizeof(float));
        uint8_t *c = (uint8_t *)malloc((size_t)cols);
        if (!u || !g || !c) {
#pragma omp atomic write
            bad = 1;
            free(u);
            free(g);
            free(c);
            continue;
        }
        transform_row(x + r * cols, cols, t, hadamard, u);
        for (int64_t j = 0; j < cols; ++j) {
            uint8_t byte = codes[(r * cols + j) / 2];
            c[j] = (uint8_t)((j & 1) ? (byte >> 4) : (byte & 15));
        }
        /* g = H'_k d per block */
        for (int64_t k = 0; k < kb; ++k) {
            const int e = (int)scales[r * kb + k] - 127;
            float d[32];
            for (int j = 0; j < 32; ++j)
                d[j] = u[k * 32 + j] - ldexpf(oracle_e2m1_value(c[k * 32 + j]), e);
            const float *H = hess + k * 1024;
            for (int i = 0; i < 32; ++i) {
                float v = 0.0f;
                for (int j = 0; j < 32; ++j)
                    v = fmaf(H[i * 32 + j], d[j], v);
                g[k * 32 + i] = v;
            }
        }
        int32_t n = 0;
        while (n < max_moves) {
            float best = 0.0f;
            int64_t bi = -1;
            int blevel = 0;
            for (int64_t i = 0; i < cols; ++i) {
                const int64_t k = i / 32;
                const int e = (int)scales[r * kb + k] - 127;
                const float Hii = hess[k * 1024 + (i % 32) * 33];
                const int level = e2m1_level(c[i]);
                const float v = oracle_e2m1_value(c[i]);
                for (int dir = -1; dir <= 1; dir += 2) {
                    const int nl = level + dir;
                    if (nl < 0 || nl > 14)
                        continue;
                    const float vn = oracle_e2m1_value(e2m1_code_of_level(nl));
                    const float D = ldexpf(vn - v, e);
                    const float gain = 2.0f * (D * g[i]) - (D * D) * Hii;
                    if (gain > best) {
                        best = gain;
                        bi = i;
                        blevel = nl;
                    }
                }
            }
            if (bi < 0)
                break;
            const int64_t k = bi / 32;
            const int e = (int)scales[r * kb + k] - 127;
            const float D = ldexpf(oracle_e2m1_value(e2m1_code_of_level(blevel)) -
                                       oracle_e2m1_value(c[bi]), e);
            c[bi] = (uint8_t)e2m1_code_of_level(blevel);
            const float *H = hess + k * 1024;
            const int i = (int)(bi % 32);
            for (int j = 0; j < 32; ++j)
                g[k * 32 + j] = fmaf(-D, H[j * 32 + i], g[k * 32 + j]);
            ++n;
        }
        for (int64_t j = 0; j < cols; j += 2)
            codes[(r * cols + j) / 2] = (uint8_t)(c[j] | (c[j + 1] << 4));
        if (moves)
            moves[r] = n;
        free(u);
        free(g);
        free(c);
    }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------ */
/* Dequantization with per-block MSE                                    */
/* ------------------------------------------------------------------ */

/* codes/scales as produced above.  sf: SF_E4M3 / SF_E3M3 (value * scale *
 * global scale; RaZeR when specials != NULL, selector in the meta byte's
 * top bits) or SF_E8M0 (value * 2^e, block 32).  ref (nullable) is the
 * fp32 tensor the block MSE is measured against. */
int oracle_dequant_mse(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t cols,
                       int block, int sf, const float *specials, int n_special, float g,
                       const float *ref, float *deq, float *mse)
{
    if (cols % block != 0 || block < 4 || block > 32 || (block & (block - 1)))
        return -1;
    if (sf == SF_E8M0 && (block != 32 || specials))
        return -1;
    if (specials && (block != 16 || sf == SF_UE5M3))
        return -1;
    if (mse && !ref)
        return -1;
    const int64_t nblk = rows * (cols / block);
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nblk; ++b) {
        uint8_t sb = scales[b];
        int sc_code = sb, sel = 0;
        if (specials) {
            sel = sf == SF_E3M3 ? (sb >> 6) : (sb >> 7);
            sc_code = sf == SF_E3M3 ? (sb & 0x3F) : (sb & 0x7F);
        }
        float acc = 0.0f;
        for (int i = 0; i < block; ++i) {
            int64_t idx = b * block + i;
            uint8_t byte = codes[idx / 2];
            int c = (idx % 2 == 0) ? (byte & 0xF) : (byte >> 4);
            float d;
            if (sf == SF_E8M0) {
                d = ldexpf(oracle_e2m1_value(c), (int)sb - 127);
            } else {
                float S = scale_value(sc_code, sf) * g;
                float v = (specials && c == 8) ? specials[sel < n_special ? sel : 0]
                                               : oracle_e2m1_value(c);
                d = v * S;
            }
            if (deq)
                deq[idx] = d;
            if (ref) {
                float e = ref[idx] - d;
                acc = fmaf(e, e, acc);
            }
        }
        if (mse)
            mse[b] = acc * (1.0f / (float)block);
    }
    return 0;
}

/* Threads used by the parallel loops above (1 = serial). */
void oracle_set_threads(int n)
{
#ifdef _OPENMP
    omp_set_num_threads(n > 0 ? n : 1);
#else
    (void)n;
#endif
}

int oracle_get_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
