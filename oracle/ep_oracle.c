/*
 * ep_oracle.c -- plain, slow, single-threaded CPU oracle for the MoE
 * layout / dispatch / combine path (token-choice and expert-choice).
 *
 * TEST INFRASTRUCTURE ONLY.  This file exists so that the tests, the
 * smoke check and the CPU-baseline leg of the benchmark have an
 * independent statement of what the GPU library must compute.  Nothing
 * in the product path links, loads or calls it, and it shares no code,
 * header, table or constant generator with the CUDA library.
 *
 * Every routine is the plain definition written out as loops, in the
 * order the definition states it; there is no blocking, fusion or
 * reordering.  Sources (page title, section):
 *
 *   [README]  "DeepEP-Ascend" README (sgl-kernel-npu, python/deep_ep),
 *             section "API Overview" (get_dispatch_layout / dispatch /
 *             combine / low_latency_dispatch / low_latency_combine rows),
 *             section "Quantization Modes in Normal Dispatch",
 *             section "Environment Variables" (MOE_EXPERT_TOKEN_NUMS_TYPE,
 *             MOE_ENABLE_TOPK_NEG_ONE).
 *   [EC]      DeepEP issue #595 "Support Expert-Choice Routing via Native
 *             Expert-Centric API ([num_experts, capacity])", sections
 *             "Background", "Current Limitation & Performance Bottleneck",
 *             "Proposed Solutions" (Solution 1 and Solution 2).
 *
 * Readings of points the pages leave open (they are listed with reasons
 * in the design notes): order inside an expert is ascending token, then
 * ascending k; logical rank r owns experts [r*E/R, (r+1)*E/R); one copy
 * per (token, expert) pair; FP8 scale = amax/448 per 128 channels and
 * q = e4m3_rne_satfinite(x * (448/amax)); the other quantisation modes of
 * the README table are read in the same way (dynamic symmetric scale from
 * the amax of the row for the per-token modes; the OCP Microscaling shared
 * exponent for the MX modes, see below); combine is an fmaf chain from
 * 0.0f in ascending k; an expert-choice token's slots are taken in
 * ascending slot id s = e*C + c.
 *
 * Parity pins: every function here is checked by the CPU test-suite
 * against brute-force enumeration, closed forms, invariants and library
 * conversions (torch's bf16 / float8_e4m3fn / float8_e5m2 casts); none is
 * unpinned.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <float.h>

/* Interface constants: the same numeric values as the library's public
 * enums (dtype, buffer layout); written out here on their own. */
#define OR_BF16 0
#define OR_FP32 1
#define OR_FP8_E4M3 2
#define OR_INT8_PER_TOKEN 3
#define OR_FP8_E4M3_PER_TOKEN 4
#define OR_MXFP8_E4M3 5
#define OR_MXFP8_E5M2 6
#define OR_MXFP4_E2M1 7
#define OR_COMPACT 0
#define OR_PADDED 1

/* ---------------------------------------------------------------------
 * Number formats.
 * bfloat16: the top 16 bits of an IEEE binary32; narrowing rounds to
 * nearest, ties to even.
 * float8 e4m3 ("E4M3FN"): 1 sign, 4 exponent (bias 7), 3 mantissa bits;
 * no infinities; S.1111.111 is NaN; largest finite 1.75 * 2^8 = 448;
 * exponent field 0 encodes subnormals m/8 * 2^-6.  The README's FP8
 * quantization modes name this format (float8_e4m3fn).
 * ------------------------------------------------------------------- */

float oracle_bf16_to_f32(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if (isnan(f))
        return (uint16_t)(((u >> 16) & 0x8000u) | 0x7FC0u);
    /* keep the upper half; add half an ulp of the kept part, minus one
     * when the kept part is even, so that exact halves go to even */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

float oracle_e4m3_to_f32(uint8_t c)
{
    int s = (c >> 7) & 1;
    int e = (c >> 3) & 0xF;
    int m = c & 7;
    float v;
    if (e == 0xF && m == 7)
        return s ? -NAN : NAN;
    if (e == 0)
        v = ldexpf((float)m / 8.0f, -6);
    else
        v = ldexpf(1.0f + (float)m / 8.0f, e - 7);
    return s ? -v : v;
}

/* Round to nearest e4m3 value, ties to even mantissa; any magnitude above
 * 448 saturates to 448 (the "satfinite" reading). */
uint8_t oracle_f32_to_e4m3(float f)
{
    uint8_t sign = signbit(f) ? 0x80 : 0x00;
    float a = fabsf(f);
    if (isnan(f))
        return (uint8_t)(sign | 0x7F);
    if (a == 0.0f)
        return sign;
    if (a > 448.0f)
        return (uint8_t)(sign | 0x7E);
    if (a < ldexpf(1.0f, -6)) {
        /* subnormal range: value = m * 2^-9, m in [0, 8]; m == 8 is the
         * smallest normal (code 0x08) so the code is m itself */
        float q = ldexpf(a, 9); /* exact: scaling by a power of two */
        int m = (int)nearbyintf(q);
        return (uint8_t)(sign | (uint8_t)m);
    }
    int ex;
    float fr = frexpf(a, &ex); /* a = fr * 2^ex, fr in [0.5, 1) */
    int unb = ex - 1;          /* a = (2*fr) * 2^unb, 2*fr in [1, 2) */
    float q = fr * 16.0f;      /* mantissa in units of 1/8: [8, 16) */
    int m = (int)nearbyintf(q);
    if (m == 16) {
        m = 8;
        unb += 1;
    }
    int code = ((unb + 7) << 3) | (m - 8);
    if (code > 0x7E)
        code = 0x7E;
    return (uint8_t)(sign | (uint8_t)code);
}

/* ---------------------------------------------------------------------
 * More element formats of the README's quantization table
 * ("Quantization Modes in Normal Dispatch": int8, float8_e5m2,
 * float4_e2m1fn_x2, float8_e8m0fnu scales).  The bit layouts are those of
 * the OCP 8-bit floating point and Microscaling (MX) v1.0 specifications.
 *
 * float8 e5m2: 1 sign, 5 exponent (bias 15), 2 mantissa bits; exponent
 * field 31 holds infinities and NaNs; largest finite 1.75 * 2^15 = 57344;
 * exponent field 0 encodes subnormals m/4 * 2^-14.
 * float4 e2m1: 1 sign, 2 exponent (bias 1), 1 mantissa bit; no infinities
 * or NaN; the magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6.
 * int8: two's complement; the symmetric range [-127, 127] is used.
 * ------------------------------------------------------------------- */

float oracle_e5m2_to_f32(uint8_t c)
{
    int s = (c >> 7) & 1;
    int e = (c >> 2) & 0x1F;
    int m = c & 3;
    float v;
    if (e == 0x1F)
        v = (m == 0) ? INFINITY : NAN;
    else if (e == 0)
        v = ldexpf((float)m / 4.0f, -14);
    else
        v = ldexpf(1.0f + (float)m / 4.0f, e - 15);
    return s ? -v : v;
}

/* Round to nearest e5m2 value, ties to even mantissa; magnitudes above
 * 57344 saturate to 57344 (satfinite). */
uint8_t oracle_f32_to_e5m2(float f)
{
    uint8_t sign = signbit(f) ? 0x80 : 0x00;
    float a = fabsf(f);
    if (isnan(f))
        return (uint8_t)(sign | 0x7F);
    if (a == 0.0f)
        return sign;
    if (a > 57344.0f)
        return (uint8_t)(sign | 0x7B);
    if (a < ldexpf(1.0f, -14)) {
        /* subnormal range: value = m * 2^-16, m in [0, 4]; m == 4 is the
         * smallest normal (code 0x04) */
        int m = (int)nearbyintf(ldexpf(a, 16));
        return (uint8_t)(sign | (uint8_t)m);
    }
    int ex;
    float fr = frexpf(a, &ex); /* a = fr * 2^ex, fr in [0.5, 1) */
    int unb = ex - 1;
    int m = (int)nearbyintf(fr * 8.0f); /* significand in units of 1/4: [4, 8] */
    if (m == 8) {
        m = 4;
        unb += 1;
    }
    int code = ((unb + 15) << 2) | (m - 4);
    if (code > 0x7B)
        code = 0x7B;
    return (uint8_t)(sign | (uint8_t)code);
}

/* 4-bit code (low nibble) -> value. */
float oracle_e2m1_to_f32(uint8_t c)
{
    int s = (c >> 3) & 1;
    int e = (c >> 1) & 3;
    int m = c & 1;
    float v = (e == 0) ? 0.5f * (float)m : ldexpf(1.0f + 0.5f * (float)m, e - 1);
    return s ? -v : v;
}

/* Round to nearest e2m1 value, ties to even mantissa; magnitudes above 6
 * saturate to 6.  Returns the 4-bit code in the low nibble. */
uint8_t oracle_f32_to_e2m1(float f)
{
    uint8_t sign = signbit(f) ? 0x8 : 0x0;
    float a = fabsf(f);
    if (isnan(f) || a > 6.0f)
        return (uint8_t)(sign | 0x7);
    if (a == 0.0f)
        return sign;
    if (a < 1.0f) {
        /* subnormal range: value = m * 0.5, m in [0, 2]; m == 2 is 1.0 (code 2) */
        int m = (int)nearbyintf(ldexpf(a, 1));
        return (uint8_t)(sign | (uint8_t)m);
    }
    int ex;
    float fr = frexpf(a, &ex);
    int unb = ex - 1;
    int m = (int)nearbyintf(fr * 4.0f); /* significand in units of 1/2: [2, 4] */
    if (m == 4) {
        m = 2;
        unb += 1;
    }
    int code = ((unb + 1) << 1) | (m - 2);
    if (code > 7)
        code = 7;
    return (uint8_t)(sign | (uint8_t)code);
}

/* Round to nearest integer, ties to even (the default rounding mode of
 * nearbyintf), clamped to [-127, 127]. */
int8_t oracle_f32_to_int8(float f)
{
    if (isnan(f))
        return 0;
    float r = nearbyintf(f);
    if (r > 127.0f)
        r = 127.0f;
    if (r < -127.0f)
        r = -127.0f;
    return (int8_t)r;
}

void oracle_f32_to_e5m2_array(const float* in, uint8_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_f32_to_e5m2(in[i]);
}

void oracle_e5m2_to_f32_array(const uint8_t* in, float* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_e5m2_to_f32(in[i]);
}

void oracle_f32_to_e2m1_array(const float* in, uint8_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_f32_to_e2m1(in[i]);
}

void oracle_e2m1_to_f32_array(const uint8_t* in, float* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_e2m1_to_f32(in[i]);
}

void oracle_f32_to_int8_array(const float* in, int8_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_f32_to_int8(in[i]);
}

void oracle_f32_to_bf16_array(const float* in, uint16_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_f32_to_bf16(in[i]);
}

void oracle_f32_to_e4m3_array(const float* in, uint8_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_f32_to_e4m3(in[i]);
}

void oracle_e4m3_to_f32_array(const uint8_t* in, float* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_e4m3_to_f32(in[i]);
}

/* ---------------------------------------------------------------------
 * FP8 e4m3 quantization of one bf16 row, one fp32 scale per 128 channels.
 * For group g: amax = max |x|; scale = amax / 448; inv = 448 / amax;
 * q = e4m3_rne_satfinite(x * inv).  amax == 0 gives scale 0 and all
 * codes 0x00.  inv is clamped to FLT_MAX so that a tiny amax cannot make
 * it infinite (0 * inf would otherwise be NaN).
 * [README] "Quantization Modes in Normal Dispatch" (FP8 e4m3 payload with
 * float32 scales); the 128-channel granularity and amax/448 are the
 * low-latency FP8 workload's definition.
 * ------------------------------------------------------------------- */
void oracle_fp8_quant_row(const uint16_t* xrow, int32_t hidden, uint8_t* q, float* scales)
{
    int32_t groups = hidden / 128;
    for (int32_t g = 0; g < groups; ++g) {
        float amax = 0.0f;
        for (int32_t i = 0; i < 128; ++i) {
            float v = fabsf(oracle_bf16_to_f32(xrow[g * 128 + i]));
            if (v > amax)
                amax = v;
        }
        if (amax == 0.0f) {
            scales[g] = 0.0f;
            for (int32_t i = 0; i < 128; ++i)
                q[g * 128 + i] = 0x00;
            continue;
        }
        float scale = amax / 448.0f;
        float inv = 448.0f / amax;
        if (inv > FLT_MAX)
            inv = FLT_MAX;
        scales[g] = scale;
        for (int32_t i = 0; i < 128; ++i) {
            float xv = oracle_bf16_to_f32(xrow[g * 128 + i]);
            float prod = xv * inv;
            q[g * 128 + i] = oracle_f32_to_e4m3(prod);
        }
    }
}

/* ---------------------------------------------------------------------
 * Per-token modes of the README table: "int8" (INT8 dynamic, per-token
 * float32 scale) and "pertoken_fp8_e4m3" (scalar FP8, per-token float32
 * scale).  One scale for the whole row, from the amax of the row, in the
 * same way as the 128-channel FP8 mode: scale = amax / qmax, inv = qmax /
 * amax (clamped to FLT_MAX), q = encode(x * inv), with qmax = 127 (int8,
 * round to nearest even, clamped to [-127, 127]) or 448 (e4m3
 * satfinite).  amax == 0 gives scale 0 and all-zero codes.
 * ------------------------------------------------------------------- */
static float row_amax(const uint16_t* xrow, int32_t n)
{
    float amax = 0.0f;
    for (int32_t i = 0; i < n; ++i) {
        float v = fabsf(oracle_bf16_to_f32(xrow[i]));
        if (v > amax)
            amax = v;
    }
    return amax;
}

void oracle_int8_quant_row(const uint16_t* xrow, int32_t hidden, int8_t* q, float* scale)
{
    float amax = row_amax(xrow, hidden);
    if (amax == 0.0f) {
        *scale = 0.0f;
        for (int32_t i = 0; i < hidden; ++i)
            q[i] = 0;
        return;
    }
    float inv = 127.0f / amax;
    if (inv > FLT_MAX)
        inv = FLT_MAX;
    *scale = amax / 127.0f;
    for (int32_t i = 0; i < hidden; ++i)
        q[i] = oracle_f32_to_int8(oracle_bf16_to_f32(xrow[i]) * inv);
}

void oracle_fp8_pertoken_quant_row(const uint16_t* xrow, int32_t hidden, uint8_t* q, float* scale)
{
    float amax = row_amax(xrow, hidden);
    if (amax == 0.0f) {
        *scale = 0.0f;
        for (int32_t i = 0; i < hidden; ++i)
            q[i] = 0x00;
        return;
    }
    float inv = 448.0f / amax;
    if (inv > FLT_MAX)
        inv = FLT_MAX;
    *scale = amax / 448.0f;
    for (int32_t i = 0; i < hidden; ++i)
        q[i] = oracle_f32_to_e4m3(oracle_bf16_to_f32(xrow[i]) * inv);
}

/* ---------------------------------------------------------------------
 * MX modes of the README table ("mx_fp8_e4m3", "mx_fp8_e5m2",
 * "mx_fp4_e2m1": per 32 elements, float8_e8m0fnu scale).  The README gives
 * the formats and the block size but not the scale rule; the rule here is
 * the OCP Microscaling v1.0 conversion: for each block of 32 elements,
 *   X = floor(log2(amax)) - emax,  emax = exponent of the element format's
 *       largest normal (e4m3: 8, e5m2: 15, e2m1: 2),
 * clamped to the E8M0 range [-127, 127] (amax == 0 gives -127); the scale
 * byte is X + 127 (the block's scale is 2^X) and every element becomes
 * encode(x * 2^-X), rounding to nearest even and saturating at the element
 * format's largest finite value.  e2m1 codes are packed two per byte,
 * element 2i in the low nibble and 2i+1 in the high nibble.
 * ------------------------------------------------------------------- */
int32_t oracle_mx_shared_exp(float amax, int32_t emax_elem)
{
    if (amax == 0.0f)
        return -127;
    int ex;
    frexpf(amax, &ex); /* amax = fr * 2^ex, fr in [0.5, 1): floor(log2 amax) = ex - 1 */
    int32_t X = (ex - 1) - emax_elem;
    if (X < -127)
        X = -127;
    if (X > 127)
        X = 127;
    return X;
}

void oracle_mx_quant_row(int32_t dtype, const uint16_t* xrow, int32_t hidden, uint8_t* q, uint8_t* scales)
{
    int32_t emax = dtype == OR_MXFP8_E4M3 ? 8 : (dtype == OR_MXFP8_E5M2 ? 15 : 2);
    for (int32_t g = 0; g < hidden / 32; ++g) {
        float amax = row_amax(xrow + g * 32, 32);
        int32_t X = oracle_mx_shared_exp(amax, emax);
        scales[g] = (uint8_t)(X + 127);
        for (int32_t i = 0; i < 32; ++i) {
            int32_t h = g * 32 + i;
            float v = ldexpf(oracle_bf16_to_f32(xrow[h]), -X); /* exact: a power-of-two scaling */
            if (dtype == OR_MXFP8_E4M3) {
                q[h] = oracle_f32_to_e4m3(v);
            } else if (dtype == OR_MXFP8_E5M2) {
                q[h] = oracle_f32_to_e5m2(v);
            } else {
                uint8_t c = oracle_f32_to_e2m1(v);
                if (h % 2 == 0)
                    q[h / 2] = c;
                else
                    q[h / 2] = (uint8_t)(q[h / 2] | (c << 4));
            }
        }
    }
}

/* Bytes of codes and of scales that one quantised row of `hidden`
 * channels takes in each output format (0 scale bytes for bf16). */
int64_t oracle_row_code_bytes(int32_t dtype, int32_t hidden)
{
    if (dtype == OR_BF16)
        return 2 * (int64_t)hidden;
    if (dtype == OR_MXFP4_E2M1)
        return hidden / 2;
    return hidden;
}

int64_t oracle_row_scale_bytes(int32_t dtype, int32_t hidden)
{
    switch (dtype) {
    case OR_FP8_E4M3:
        return 4 * (int64_t)(hidden / 128);
    case OR_INT8_PER_TOKEN:
    case OR_FP8_E4M3_PER_TOKEN:
        return 4;
    case OR_MXFP8_E4M3:
    case OR_MXFP8_E5M2:
    case OR_MXFP4_E2M1:
        return hidden / 32;
    default:
        return 0;
    }
}

/* One bf16 row in output format `dtype`: codes into q, scales into
 * `scales` (layouts as above). */
void oracle_quant_row(int32_t dtype, const uint16_t* xrow, int32_t hidden, uint8_t* q, void* scales)
{
    switch (dtype) {
    case OR_FP8_E4M3:
        oracle_fp8_quant_row(xrow, hidden, q, (float*)scales);
        break;
    case OR_INT8_PER_TOKEN:
        oracle_int8_quant_row(xrow, hidden, (int8_t*)q, (float*)scales);
        break;
    case OR_FP8_E4M3_PER_TOKEN:
        oracle_fp8_pertoken_quant_row(xrow, hidden, q, (float*)scales);
        break;
    default:
        oracle_mx_quant_row(dtype, xrow, hidden, q, (uint8_t*)scales);
        break;
    }
}

/* ---------------------------------------------------------------------
 * Token-choice layout.  [README] "API Overview", get_dispatch_layout:
 * per-rank token counts, per-expert token counts and is_token_in_rank;
 * "Environment Variables": MOE_EXPERT_TOKEN_NUMS_TYPE (count form and
 * prefix-sum form -- both are produced here: counts[E] and offsets[E+1])
 * and MOE_ENABLE_TOPK_NEG_ONE (-1 = token not sent to any expert).
 * slot[t,k] = number of earlier pairs (t',k') < (t,k), in token-major
 * order, routed to the same expert; -1 for a pair that is not routed.
 * An id outside [-1, E) is treated as -1 and counted in the return value.
 * ------------------------------------------------------------------- */
int64_t oracle_tc_layout(const int64_t* topk_idx, int32_t T, int32_t K, int32_t E, int32_t R,
                         int32_t* counts, int32_t* offsets, int32_t* rank_counts,
                         uint8_t* is_token_in_rank, int32_t* slot)
{
    int64_t bad = 0;
    int32_t per_rank = E / R;
    for (int32_t e = 0; e < E; ++e)
        counts[e] = 0;
    for (int32_t r = 0; r < R; ++r)
        rank_counts[r] = 0;
    for (int32_t t = 0; t < T; ++t) {
        uint32_t mask = 0;
        for (int32_t k = 0; k < K; ++k) {
            int64_t e = topk_idx[(int64_t)t * K + k];
            if (e >= 0 && e < E) {
                slot[(int64_t)t * K + k] = counts[e];
                counts[e] += 1;
                mask |= 1u << (uint32_t)(e / per_rank);
            } else {
                slot[(int64_t)t * K + k] = -1;
                if (e != -1)
                    bad += 1;
            }
        }
        for (int32_t r = 0; r < R; ++r) {
            uint8_t bit = (uint8_t)((mask >> r) & 1u);
            is_token_in_rank[(int64_t)t * R + r] = bit;
            rank_counts[r] += bit;
        }
    }
    offsets[0] = 0;
    for (int32_t e = 0; e < E; ++e)
        offsets[e + 1] = offsets[e] + counts[e];
    return bad;
}

/* Destination row of pair (t,k) routed to expert e with rank `s` inside
 * it: compact buffers are the per-expert segments laid end to end;
 * padded (low-latency) buffers give every expert max_tokens rows.
 * Returns -1 when the pair has no row. */
static int64_t pair_row(int64_t e, int32_t s, int32_t E, const int32_t* offsets, int32_t mode,
                        int32_t max_tokens, int64_t num_rows)
{
    int64_t row;
    if (e < 0 || e >= E || s < 0)
        return -1;
    if (mode == OR_PADDED) {
        if (s >= max_tokens)
            return -2;
        row = e * (int64_t)max_tokens + s;
    } else {
        row = (int64_t)offsets[e] + s;
    }
    if (row >= num_rows)
        return -2;
    return row;
}

/* ---------------------------------------------------------------------
 * Token-choice dispatch.  [README] "API Overview", dispatch (normal) and
 * low_latency_dispatch (per-expert buffers of num_max_dispatch_tokens_per
 * _rank rows); "Quantization Modes in Normal Dispatch" (bf16 payload, or
 * one of the quantised formats above with its scales).  For every routed
 * pair (t,k), row pair_row(...) of recv receives x[t] (bf16 copy) or its
 * encoding by oracle_quant_row, and the same row of recv_scales its
 * scales; recv_src[row] = t and recv_weights[row] = w[t,k] when those
 * outputs are requested.  Returns the number of pairs that had no room
 * (padded slot >= max_tokens, or row beyond num_recv_rows).
 * ------------------------------------------------------------------- */
int64_t oracle_tc_dispatch(const uint16_t* x, int32_t T, int32_t H, const int64_t* topk_idx, int32_t K,
                           int32_t E, const int32_t* slot, const int32_t* offsets, int32_t mode,
                           int32_t max_tokens, int64_t num_recv_rows, int32_t out_dtype,
                           const float* topk_weights, void* recv, void* recv_scales,
                           int32_t* recv_src, float* recv_weights)
{
    int64_t overflow = 0;
    int64_t code_bytes = oracle_row_code_bytes(out_dtype, H);
    int64_t scale_bytes = oracle_row_scale_bytes(out_dtype, H);
    uint8_t* qrow = NULL;
    uint8_t* srow = NULL;
    if (out_dtype != OR_BF16) {
        qrow = (uint8_t*)malloc((size_t)code_bytes + 1);
        srow = (uint8_t*)malloc((size_t)scale_bytes + 4);
    }
    for (int32_t t = 0; t < T; ++t) {
        for (int32_t k = 0; k < K; ++k) {
            int64_t e = topk_idx[(int64_t)t * K + k];
            int32_t s = slot[(int64_t)t * K + k];
            int64_t row = pair_row(e, s, E, offsets, mode, max_tokens, num_recv_rows);
            if (row == -2) {
                overflow += 1;
                continue;
            }
            if (row < 0)
                continue;
            if (out_dtype != OR_BF16) {
                oracle_quant_row(out_dtype, x + (int64_t)t * H, H, qrow, srow);
                memcpy((uint8_t*)recv + row * code_bytes, qrow, (size_t)code_bytes);
                memcpy((uint8_t*)recv_scales + row * scale_bytes, srow, (size_t)scale_bytes);
            } else {
                memcpy((uint16_t*)recv + row * H, x + (int64_t)t * H, sizeof(uint16_t) * (size_t)H);
            }
            if (recv_src)
                recv_src[row] = t;
            if (recv_weights)
                recv_weights[row] = topk_weights[(int64_t)t * K + k];
        }
    }
    free(qrow);
    free(srow);
    return overflow;
}

/* ---------------------------------------------------------------------
 * Token-choice combine.  [README] "API Overview", combine (reduce with
 * the dispatch handle) and low_latency_combine (takes topk_weights: a
 * weighted reduce); [EC] Solution 2 (skip -1 padding).
 * out[t] = sum over k ascending of w[t,k] * y[row(t,k)], skipping pairs
 * with no row, as the chain acc = fmaf(w, y, acc) from acc = 0.0f in
 * fp32; written as fp32 or rounded once to bf16.  `tokens` (optional)
 * selects which tokens to compute; out row i belongs to tokens[i].
 * ------------------------------------------------------------------- */
void oracle_tc_combine(const uint16_t* y, int64_t num_y_rows, int32_t H, int32_t T, const int64_t* topk_idx,
                       int32_t K, int32_t E, const int32_t* slot, const int32_t* offsets, int32_t mode,
                       int32_t max_tokens, const float* topk_weights, const int32_t* tokens,
                       int32_t n_tokens, int32_t out_dtype, void* out)
{
    float* acc = (float*)malloc(sizeof(float) * (size_t)H);
    int32_t n = tokens ? n_tokens : T;
    for (int32_t i = 0; i < n; ++i) {
        int32_t t = tokens ? tokens[i] : i;
        for (int32_t h = 0; h < H; ++h)
            acc[h] = 0.0f;
        for (int32_t k = 0; k < K; ++k) {
            int64_t e = topk_idx[(int64_t)t * K + k];
            int32_t s = slot[(int64_t)t * K + k];
            int64_t row = pair_row(e, s, E, offsets, mode, max_tokens, num_y_rows);
            if (row < 0)
                continue;
            float w = topk_weights[(int64_t)t * K + k];
            for (int32_t h = 0; h < H; ++h)
                acc[h] = fmaf(w, oracle_bf16_to_f32(y[row * H + h]), acc[h]);
        }
        for (int32_t h = 0; h < H; ++h) {
            if (out_dtype == OR_FP32)
                ((float*)out)[(int64_t)i * H + h] = acc[h];
            else
                ((uint16_t*)out)[(int64_t)i * H + h] = oracle_f32_to_bf16(acc[h]);
        }
    }
    free(acc);
}

/* ---------------------------------------------------------------------
 * Per-rank (deduplicated) dispatch and rank-level combine.  [README] "API
 * Overview": normal-mode dispatch sends tokens to expert *ranks* and returns
 * the received tokens with their top-k information; combine reduces the
 * tokens coming back from the ranks, using the dispatch handle; the layout
 * gives is_token_in_rank.  Reading: a token travels once to every rank
 * that holds at least one of its experts (is_token_in_rank[t, r] = 1).
 * Rank r's received rows are its tokens in ascending token order, and the
 * ranks' row ranges are laid end to end: rank_offsets[R+1] is the exclusive
 * scan of the per-rank token counts and rank_row[t, r] is token t's row
 * (rank_offsets[r] + number of earlier tokens of rank r), -1 where t does
 * not go to r.  Each received row carries the token's K entries as seen by
 * the rank: the local expert id e - r*E/R for an expert of rank r and its
 * gate weight, else -1 and 0.  The rank-level combine adds, for each token,
 * the rows its ranks send back, in ascending rank order, in fp32 from 0
 * (the gate weights were applied on the ranks), written as fp32 or rounded
 * once to bf16.
 * ------------------------------------------------------------------- */
void oracle_rank_layout(const uint8_t* is_token_in_rank, int32_t T, int32_t R, int32_t* rank_offsets,
                        int32_t* rank_row)
{
    int32_t* count = (int32_t*)calloc((size_t)R + 1, sizeof(int32_t));
    for (int32_t t = 0; t < T; ++t) {
        for (int32_t r = 0; r < R; ++r) {
            if (is_token_in_rank[(int64_t)t * R + r]) {
                rank_row[(int64_t)t * R + r] = count[r];
                count[r] += 1;
            } else {
                rank_row[(int64_t)t * R + r] = -1;
            }
        }
    }
    rank_offsets[0] = 0;
    for (int32_t r = 0; r < R; ++r)
        rank_offsets[r + 1] = rank_offsets[r] + count[r];
    for (int32_t t = 0; t < T; ++t)
        for (int32_t r = 0; r < R; ++r)
            if (rank_row[(int64_t)t * R + r] >= 0)
                rank_row[(int64_t)t * R + r] += rank_offsets[r];
    free(count);
}

void oracle_rank_dispatch(const uint16_t* x, int32_t T, int32_t H, const int64_t* topk_idx, int32_t K,
                          int32_t E, int32_t R, const int32_t* rank_row, const float* topk_weights,
                          uint16_t* recv, int64_t* recv_topk_idx, float* recv_topk_weights, int32_t* recv_src)
{
    int32_t per_rank = E / R;
    for (int32_t t = 0; t < T; ++t) {
        for (int32_t r = 0; r < R; ++r) {
            int64_t row = rank_row[(int64_t)t * R + r];
            if (row < 0)
                continue;
            memcpy(recv + row * H, x + (int64_t)t * H, sizeof(uint16_t) * (size_t)H);
            if (recv_src)
                recv_src[row] = t;
            for (int32_t k = 0; k < K; ++k) {
                int64_t e = topk_idx[(int64_t)t * K + k];
                int local = e >= 0 && e < E && e / per_rank == r;
                if (recv_topk_idx)
                    recv_topk_idx[row * K + k] = local ? e - (int64_t)r * per_rank : -1;
                if (recv_topk_weights)
                    recv_topk_weights[row * K + k] = local ? topk_weights[(int64_t)t * K + k] : 0.0f;
            }
        }
    }
}

void oracle_rank_combine(const uint16_t* y, int32_t H, int32_t T, int32_t R, const int32_t* rank_row,
                         const int32_t* tokens, int32_t n_tokens, int32_t out_dtype, void* out)
{
    float* acc = (float*)malloc(sizeof(float) * (size_t)H);
    int32_t n = tokens ? n_tokens : T;
    for (int32_t i = 0; i < n; ++i) {
        int32_t t = tokens ? tokens[i] : i;
        for (int32_t h = 0; h < H; ++h)
            acc[h] = 0.0f;
        for (int32_t r = 0; r < R; ++r) {
            int64_t row = rank_row[(int64_t)t * R + r];
            if (row < 0)
                continue;
            for (int32_t h = 0; h < H; ++h)
                acc[h] = acc[h] + oracle_bf16_to_f32(y[row * H + h]);
        }
        for (int32_t h = 0; h < H; ++h) {
            if (out_dtype == OR_FP32)
                ((float*)out)[(int64_t)i * H + h] = acc[h];
            else
                ((uint16_t*)out)[(int64_t)i * H + h] = oracle_f32_to_bf16(acc[h]);
        }
    }
    free(acc);
}

/* ---------------------------------------------------------------------
 * Expert-choice layout.  [EC] "Proposed Solutions", Solution 1: the
 * routing is token_indices[E, C] (expert e picked token token_indices[e,c]
 * in slot c); no [T, K] inverse table with padding is built.  What the
 * combine needs instead is each token's own list of slots, stored as a
 * CSR: token_offsets[T+1] (exclusive scan of the number of slots that
 * picked each token) and token_slots (slot ids s = e*C + c, ascending
 * within a token).  counts[e] = number of valid entries in row e;
 * is_token_in_rank / rank_counts as for token choice.  An id outside
 * [-1, T) is treated as an empty slot and counted in the return value.
 * ------------------------------------------------------------------- */
int64_t oracle_ec_layout(const int32_t* token_indices, int32_t T, int32_t E, int32_t C, int32_t R,
                         int32_t* counts, int32_t* rank_counts, uint8_t* is_token_in_rank,
                         int32_t* token_offsets, int32_t* token_slots)
{
    int64_t bad = 0;
    int32_t per_rank = E / R;
    int64_t S = (int64_t)E * C;
    int32_t* deg = (int32_t*)calloc((size_t)T + 1, sizeof(int32_t));
    int32_t* fill = (int32_t*)calloc((size_t)T + 1, sizeof(int32_t));
    uint32_t* mask = (uint32_t*)calloc((size_t)T + 1, sizeof(uint32_t));
    for (int32_t e = 0; e < E; ++e)
        counts[e] = 0;
    for (int64_t s = 0; s < S; ++s) {
        int32_t t = token_indices[s];
        int32_t e = (int32_t)(s / C);
        if (t >= 0 && t < T) {
            deg[t] += 1;
            counts[e] += 1;
            mask[t] |= 1u << (uint32_t)(e / per_rank);
        } else if (t != -1) {
            bad += 1;
        }
    }
    token_offsets[0] = 0;
    for (int32_t t = 0; t < T; ++t)
        token_offsets[t + 1] = token_offsets[t] + deg[t];
    for (int64_t s = 0; s < S; ++s) {
        int32_t t = token_indices[s];
        if (t >= 0 && t < T) {
            token_slots[token_offsets[t] + fill[t]] = (int32_t)s;
            fill[t] += 1;
        }
    }
    for (int32_t r = 0; r < R; ++r)
        rank_counts[r] = 0;
    for (int32_t t = 0; t < T; ++t) {
        for (int32_t r = 0; r < R; ++r) {
            uint8_t bit = (uint8_t)((mask[t] >> r) & 1u);
            is_token_in_rank[(int64_t)t * R + r] = bit;
            rank_counts[r] += bit;
        }
    }
    free(deg);
    free(fill);
    free(mask);
    return bad;
}

/* Expert-choice dispatch.  [EC] Solution 1 (dispatch_expert_choice):
 * recv[e*C + c] = x[token_indices[e, c]]; rows of empty slots untouched. */
void oracle_ec_dispatch(const uint16_t* x, int32_t T, int32_t H, const int32_t* token_indices,
                        int32_t E, int32_t C, uint16_t* recv)
{
    int64_t S = (int64_t)E * C;
    for (int64_t s = 0; s < S; ++s) {
        int32_t t = token_indices[s];
        if (t >= 0 && t < T)
            memcpy(recv + s * H, x + (int64_t)t * H, sizeof(uint16_t) * (size_t)H);
    }
}

/* Expert-choice combine.  [EC] "Current Limitation" point 2 and Solution
 * 1: the reduce runs over the slots that picked the token, with no
 * [T, K] padding and no cap on their number.  out[t] = fmaf chain over
 * the token's CSR slots s in ascending order of expert_weights[s] *
 * y[s]; a token no expert picked gets zeros. */
void oracle_ec_combine(const uint16_t* y, int32_t H, int32_t T, const int32_t* token_offsets,
                       const int32_t* token_slots, const float* expert_weights, const int32_t* tokens,
                       int32_t n_tokens, int32_t out_dtype, void* out)
{
    float* acc = (float*)malloc(sizeof(float) * (size_t)H);
    int32_t n = tokens ? n_tokens : T;
    for (int32_t i = 0; i < n; ++i) {
        int32_t t = tokens ? tokens[i] : i;
        for (int32_t h = 0; h < H; ++h)
            acc[h] = 0.0f;
        for (int32_t j = token_offsets[t]; j < token_offsets[t + 1]; ++j) {
            int64_t s = token_slots[j];
            float w = expert_weights[s];
            for (int32_t h = 0; h < H; ++h)
                acc[h] = fmaf(w, oracle_bf16_to_f32(y[s * H + h]), acc[h]);
        }
        for (int32_t h = 0; h < H; ++h) {
            if (out_dtype == OR_FP32)
                ((float*)out)[(int64_t)i * H + h] = acc[h];
            else
                ((uint16_t*)out)[(int64_t)i * H + h] = oracle_f32_to_bf16(acc[h]);
        }
    }
    free(acc);
}
