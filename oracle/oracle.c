/*
 * oracle.c -- plain, slow, fp64 CPU oracle for the fused
 * "W-way reduce + residual add + RMSNorm" step and its variants.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or
 * calls this file; only the tests, the smoke check and the bench's CPU
 * baseline leg do.  It shares no code, header, table or helper with the
 * CUDA library.
 *
 * Sources (vLLM pull-request reports on prhub.com.cn):
 *   [P1] PR #54787 report, "ROCm AITER fused allreduce+RMSNorm fast path":
 *        sections "实现拆解" (implementation) and "关键源码片段"
 *        (fused_allreduce_gemma_rms_norm: explicit all_reduce followed by
 *        GemmaRMSNorm with the residual; gemma_norm => weight bias 1.0).
 *   [P2] PR #44849 report, "[ROCm][MiniMax-M2] Dispatch fused QK-norm +
 *        AllReduce via AITER": section "关键源码片段"
 *        (_minimax_qk_norm_fusion and its sequential RMSNorm + AllReduce
 *        fallback: q and k are normalised over the full TP width).
 *   [P3] PR #50802 report, "AITER add-RMSNorm dead-residual fusion":
 *        sections "实现拆解" and "关键源码片段" (output-only pattern keeps
 *        only the RMSNorm output; the no-residual all_reduce -> rms_norm site;
 *        per-group FP8 quantisation of the normalised output).
 *
 * Every function below is the plain definition written out: exact widening
 * of the 16-bit inputs to fp64, a left-to-right fp64 sum, the mean of
 * squares, one sqrt and one division per row.  No blocking, no fusion, no
 * reordering.  Rounding of results to 16-bit formats and the e4m3 encoder are
 * written here from the IEEE-754 / OCP-FP8 format definitions.
 *
 * Parity pins (tests/test_oracle_pins.py) tie each function to something
 * other than itself: torch's rms_norm in fp64 for W=1 and zero residual,
 * exact rational arithmetic on small inputs, permutation and scale
 * invariances, the row-RMS identity, exhaustive e4m3 and 16-bit rounding
 * checks against torch's CPU casts, and hand-derived closed forms.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORACLE_BF16 0
#define ORACLE_FP16 1

/* ------------------------------------------------------------------ */
/* 16-bit float formats, from their bit layouts.                        */
/*   bf16: 1 sign, 8 exponent (bias 127), 7 fraction bits.              */
/*   fp16: 1 sign, 5 exponent (bias 15), 10 fraction bits.              */
/* ------------------------------------------------------------------ */

static double decode_fields(uint32_t sign, uint32_t exp, uint32_t frac,
                            int exp_bits, int frac_bits)
{
    const int bias = (1 << (exp_bits - 1)) - 1;
    const uint32_t exp_all_ones = (1u << exp_bits) - 1u;
    double mag;
    if (exp == exp_all_ones) {
        mag = frac ? NAN : INFINITY;
    } else if (exp == 0) {
        /* subnormal: frac * 2^(1 - bias - frac_bits) */
        mag = ldexp((double)frac, 1 - bias - frac_bits);
    } else {
        mag = ldexp((double)((1u << frac_bits) | frac), (int)exp - bias - frac_bits);
    }
    return sign ? -mag : mag;
}

double oracle_decode16(uint16_t bits, int dtype)
{
    if (dtype == ORACLE_BF16)
        return decode_fields(bits >> 15, (bits >> 7) & 0xFFu, bits & 0x7Fu, 8, 7);
    return decode_fields(bits >> 15, (bits >> 10) & 0x1Fu, bits & 0x3FFu, 5, 10);
}

/*
 * Round a finite or infinite double to the nearest value of a binary format
 * with `exp_bits` exponent bits and `frac_bits` fraction bits, ties to even,
 * with gradual underflow and overflow to infinity (IEEE-754 default
 * rounding).  Returns the encoded bits.
 */
static uint32_t round_to_format(double x, int exp_bits, int frac_bits)
{
    const int bias = (1 << (exp_bits - 1)) - 1;
    const uint32_t exp_all_ones = (1u << exp_bits) - 1u;
    const uint32_t sign_bit = 1u << (exp_bits + frac_bits);
    uint32_t sign = 0;
    if (isnan(x))
        return (exp_all_ones << frac_bits) | (1u << (frac_bits - 1));
    if (signbit(x)) {
        sign = sign_bit;
        x = -x;
    }
    if (isinf(x))
        return sign | (exp_all_ones << frac_bits);
    if (x == 0.0)
        return sign;

    /* x = m * 2^e with m in [0.5, 1) */
    int e;
    (void)frexp(x, &e);
    /* unbiased exponent of the leading bit is e-1; the quantum (value of the
     * last fraction bit) is 2^(e-1-frac_bits) for normals and the fixed
     * subnormal quantum 2^(1-bias-frac_bits) below the normal range. */
    int lead = e - 1;
    int min_normal_exp = 1 - bias;
    int q_exp = (lead < min_normal_exp ? min_normal_exp : lead) - frac_bits;
    /* scaled = x / quantum, exact in double (power-of-two scaling) */
    double scaled = ldexp(x, -q_exp);
    double fl = floor(scaled);
    double rem = scaled - fl;                 /* exact */
    double n = fl;
    if (rem > 0.5 || (rem == 0.5 && fmod(fl, 2.0) != 0.0))
        n = fl + 1.0;
    /* value = n * 2^q_exp; renormalise if rounding carried into a new binade */
    double val = ldexp(n, q_exp);
    if (val == 0.0)                            /* rounded down to zero */
        return sign;
    int e2;
    (void)frexp(val, &e2);
    int lead2 = e2 - 1;
    if (lead2 > bias)                          /* above the largest finite */
        return sign | (exp_all_ones << frac_bits);
    if (lead2 < min_normal_exp) {              /* subnormal (or zero) */
        uint32_t frac = (uint32_t)ldexp(val, -(min_normal_exp - frac_bits));
        return sign | frac;
    }
    uint32_t biased = (uint32_t)(lead2 + bias);
    uint32_t frac = (uint32_t)(ldexp(val, -(lead2 - frac_bits)) - ldexp(1.0, frac_bits));
    return sign | (biased << frac_bits) | frac;
}

uint16_t oracle_round16(double x, int dtype)
{
    if (dtype == ORACLE_BF16)
        return (uint16_t)round_to_format(x, 8, 7);
    return (uint16_t)round_to_format(x, 5, 10);
}

/* ------------------------------------------------------------------ */
/* FP8 e4m3fn (OCP 8-bit floating point, "FN" variant):                */
/*   1 sign, 4 exponent (bias 7), 3 fraction bits; no infinities;      */
/*   S.1111.111 is NaN; largest finite 1.75 * 2^8 = 448; smallest      */
/*   subnormal 2^-9.                                                   */
/* ------------------------------------------------------------------ */

double oracle_e4m3_decode(uint8_t code)
{
    uint32_t sign = code >> 7, exp = (code >> 3) & 0xFu, frac = code & 7u;
    double mag;
    if (exp == 0xFu && frac == 7u)
        mag = NAN;
    else if (exp == 0)
        mag = ldexp((double)frac, -9);          /* frac * 2^(1-7-3) */
    else
        mag = ldexp((double)(8u | frac), (int)exp - 7 - 3);
    return sign ? -mag : mag;
}

/*
 * Encode with round-to-nearest-even and saturation to +-448 ("satfinite":
 * values beyond the largest finite magnitude, infinities included, clamp to
 * it; NaN maps to the NaN code 0x7F with the sign kept).
 */
uint8_t oracle_e4m3_encode(double x)
{
    uint8_t sign = 0;
    if (isnan(x))
        return signbit(x) ? 0xFF : 0x7F;
    if (signbit(x)) {
        sign = 0x80;
        x = -x;
    }
    if (x >= 448.0)
        return sign | 0x7E;
    if (x == 0.0)
        return sign;
    int e;
    (void)frexp(x, &e);
    int lead = e - 1;
    int q_exp = (lead < -6 ? -6 : lead) - 3;   /* min normal exponent 1-7 = -6 */
    double scaled = ldexp(x, -q_exp);
    double fl = floor(scaled);
    double rem = scaled - fl;
    double n = fl;
    if (rem > 0.5 || (rem == 0.5 && fmod(fl, 2.0) != 0.0))
        n = fl + 1.0;
    double val = ldexp(n, q_exp);
    if (val >= 448.0)                          /* 448 is representable; above clamps */
        return sign | 0x7E;
    if (val == 0.0)                            /* rounded down to zero */
        return sign;
    int e2;
    (void)frexp(val, &e2);
    int lead2 = e2 - 1;
    if (lead2 < -6) {
        uint32_t frac = (uint32_t)ldexp(val, 9);
        return sign | (uint8_t)frac;
    }
    uint32_t biased = (uint32_t)(lead2 + 7);
    uint32_t frac = (uint32_t)(ldexp(val, -(lead2 - 3)) - 8.0);
    return sign | (uint8_t)((biased << 3) | frac);
}

/* ------------------------------------------------------------------ */
/* [P1] explicit all_reduce + (Gemma)RMSNorm with residual;            */
/* [P3] output-only and no-residual forms.                             */
/* ------------------------------------------------------------------ */

/*
 * For each token t (row of length H):
 *   r[h]  = residual[h] + sum_{w=0}^{W-1} P_w[h]        (residual optional)
 *   ms    = (1/H) * sum_h r[h]^2
 *   y[h]  = r[h] / sqrt(ms + eps) * (gemma ? 1 + weight[h] : weight[h])
 * y and r are returned unrounded in fp64; rounding to the output format is
 * oracle_round16's job.  inv_rms[t] = 1/sqrt(ms+eps) when requested.
 */
void oracle_ar_add_rmsnorm(const uint16_t *const *partials, int W,
                           const uint16_t *residual, const uint16_t *weight,
                           int64_t T, int64_t H, double eps, int gemma, int dtype,
                           double *y, double *r_out, double *inv_rms)
{
    for (int64_t t = 0; t < T; ++t) {
        double sumsq = 0.0;
        for (int64_t h = 0; h < H; ++h) {
            double r = residual ? oracle_decode16(residual[t * H + h], dtype) : 0.0;
            for (int w = 0; w < W; ++w)
                r += oracle_decode16(partials[w][t * H + h], dtype);
            if (r_out)
                r_out[t * H + h] = r;
            sumsq += r * r;
        }
        double ms = sumsq / (double)H;
        double denom = sqrt(ms + eps);
        if (inv_rms)
            inv_rms[t] = 1.0 / denom;
        for (int64_t h = 0; h < H; ++h) {
            double r = residual ? oracle_decode16(residual[t * H + h], dtype) : 0.0;
            for (int w = 0; w < W; ++w)
                r += oracle_decode16(partials[w][t * H + h], dtype);
            double wv = oracle_decode16(weight[h], dtype);
            double weff = gemma ? 1.0 + wv : wv;
            y[t * H + h] = r / denom * weff;
        }
    }
}

/*
 * [P3] per-group FP8 quantisation of the normalised output, groups of
 * `group` consecutive elements along H:
 *   amax  = max |y| over the group
 *   scale = amax / 448                     (scales64: the exact fp64 value)
 * The e4m3 code is a decision taken in fp32, as the GPU takes it:
 *   y32 = fl32(y), amax32 = max |y32|, s32 = fl32(amax32 / 448),
 *   q   = e4m3_rne_satfinite(fl32(y32 / s32)),   q = 0 when amax32 == 0.
 * scales32 receives s32.
 */
void oracle_quant_fp8_group(const double *y, int64_t T, int64_t H, int group,
                            uint8_t *q, double *scales64, float *scales32)
{
    int64_t G = H / group;
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t g = 0; g < G; ++g) {
            const double *yg = y + t * H + g * group;
            double amax = 0.0;
            float amax32 = 0.0f;
            for (int i = 0; i < group; ++i) {
                double a = fabs(yg[i]);
                if (a > amax)
                    amax = a;
                float a32 = fabsf((float)yg[i]);
                if (a32 > amax32)
                    amax32 = a32;
            }
            volatile float s32 = amax32 / 448.0f;
            if (scales64)
                scales64[t * G + g] = amax / 448.0;
            if (scales32)
                scales32[t * G + g] = s32;
            for (int i = 0; i < group; ++i) {
                uint8_t code = 0;
                if (amax32 > 0.0f) {
                    volatile float quot = (float)yg[i] / s32;
                    code = oracle_e4m3_encode((double)quot);
                }
                q[t * H + g * group + i] = code;
            }
        }
    }
}

/*
 * [P2] MiniMax sharded QK-norm.  Shard w holds, per token, a row
 *   [ q_w (qs) | k_w (ks) | v_w (ks) ],  qs = q_size/W, ks = kv_size/W,
 * and the full q of a token is concat_w q_w (likewise k).  Each is
 * RMS-normalised over its FULL width with the full weight vector; shard w's
 * output is its own slice:
 *   inv_q = 1/sqrt((1/q_size) * sum over all shards of q^2 + eps)
 *   q_out[w][t][j] = q_w[t][j] * inv_q * q_weight[w*qs + j]
 * and the same for k with kv_size and k_weight.  v is not an output.
 * q_out is laid out [W][T][qs], k_out [W][T][ks], both fp64, unrounded.
 */
void oracle_qk_norm_sharded(const uint16_t *const *qkv, int W,
                            const uint16_t *q_weight, const uint16_t *k_weight,
                            int64_t T, int64_t q_size, int64_t kv_size,
                            double eps, int dtype, double *q_out, double *k_out)
{
    int64_t qs = q_size / W, ks = kv_size / W, row = qs + 2 * ks;
    for (int64_t t = 0; t < T; ++t) {
        double ssq_q = 0.0, ssq_k = 0.0;
        for (int w = 0; w < W; ++w) {
            const uint16_t *x = qkv[w] + t * row;
            for (int64_t j = 0; j < qs; ++j) {
                double v = oracle_decode16(x[j], dtype);
                ssq_q += v * v;
            }
            for (int64_t j = 0; j < ks; ++j) {
                double v = oracle_decode16(x[qs + j], dtype);
                ssq_k += v * v;
            }
        }
        double den_q = sqrt(ssq_q / (double)q_size + eps);
        double den_k = sqrt(ssq_k / (double)kv_size + eps);
        for (int w = 0; w < W; ++w) {
            const uint16_t *x = qkv[w] + t * row;
            for (int64_t j = 0; j < qs; ++j)
                q_out[((int64_t)w * T + t) * qs + j] =
                    oracle_decode16(x[j], dtype) / den_q *
                    oracle_decode16(q_weight[w * qs + j], dtype);
            for (int64_t j = 0; j < ks; ++j)
                k_out[((int64_t)w * T + t) * ks + j] =
                    oracle_decode16(x[qs + j], dtype) / den_k *
                    oracle_decode16(k_weight[w * ks + j], dtype);
        }
    }
}

/* Vectorised helpers for the tests: round / decode whole arrays. */
void oracle_round16_array(const double *x, int64_t n, int dtype, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_round16(x[i], dtype);
}

void oracle_decode16_array(const uint16_t *x, int64_t n, int dtype, double *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_decode16(x[i], dtype);
}

void oracle_e4m3_encode_array(const double *x, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_e4m3_encode(x[i]);
}

void oracle_e4m3_decode_array(const uint8_t *x, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_e4m3_decode(x[i]);
}
