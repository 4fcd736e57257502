/*
 * CPU oracle for one packed FP4 mixture-of-experts FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, single-threaded
 * definition that the CUDA library is checked against.  Only the test suite,
 * the smoke check and the benchmark's CPU-baseline / reference legs load it.
 * It shares no code, header, table or helper with the CUDA library and must
 * never be reached from the library's own code path.
 *
 * What it computes (the packed MoE decode layer of "FireEcho Engine",
 * sections "The Goliath Kernel: Why It's Fast" and "Speed Optimization
 * History"; the SiLU(gate)*up product of "FastInfer", section "Confirmed
 * elementwise SwiGLU scheduling"):
 *
 *   0. router GEMM (when the logits are not given): logits[t][e] =
 *      sum_h x[t][h] W_r[e][h], one bf16 row of W_r per expert, in fp64;
 *   1. router: per token, experts ordered by (logit descending, index
 *      ascending); the first k are the token's slots j = 0..k-1; the slot
 *      weights are the softmax of the k selected logits (fp64, stored fp32);
 *   2. grouping: pair p = t*k + j goes to expert idx[t][j]; counts, the
 *      exclusive scan of the counts, and the pair ids ordered by
 *      (expert, pair id);
 *   3. dequantisation: W[e][k][n] = E2M1(code) * bf16 scale of the 32-element
 *      group of k that holds k; two codes per byte, the low nibble holding
 *      the even k; all experts in one [E, K/2, N] code buffer and one
 *      [E, K/32, N] scale buffer (FireEcho's packed [E, K//2, N] expert
 *      buffer); an expert may instead hold INT2 codes, W = (q - 1.5) * the
 *      same group scale, four codes per byte (orc_moe_forward_fmt);
 *   4. gate_up: g[n] = sum_k x[k] W[k][n], u[n] = sum_k x[k] W[k][I+n]
 *      (gate columns first, then up columns, one fused matrix);
 *      act[n] = silu(g[n]) * u[n], silu(v) = v / (1 + exp(-v));
 *   5. down: o[h] = sum_i act[i] Wd[i][h];
 *   6. combine: y[t][h] = sum_j w[t][j] o_j[h], slot order, in fp64; the
 *      bfloat16 copy is rounded once, to nearest even.
 *
 * The E2M1 code table, the group of 32, the nibble order, the router rule
 * and the scale rule max|w|/6 are the format this library implements; the
 * pages themselves only sketch the in-register dequantisation.  Every sum is
 * accumulated in fp64 in the obvious order; nothing is blocked, fused or
 * reordered.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_EINVAL (-1)
#define ORC_ENOMEM (-2)

/* ---------------------------------------------------------------------- */
/* E2M1: 1 sign bit (bit 3), then the magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 */
/* for magnitude codes 0..7.                                                 */
/* ---------------------------------------------------------------------- */
static const float orc_e2m1_magnitude[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

double orc_e2m1_decode(int code)
{
    double m = orc_e2m1_magnitude[code & 7];
    return (code & 8) ? -m : m;
}

/* bfloat16 helpers (the oracle's own) */
static float orc_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static uint16_t orc_f32_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return 0x7FC0; /* NaN */
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* fp64 -> bfloat16, round to nearest even, without double rounding: round to
 * float with round-to-odd (sticky last bit) first, which keeps the final
 * 8-bit rounding exact because float has more than 8 + 2 significant bits. */
uint16_t orc_f64_to_bf16_rne(double y)
{
    if (isnan(y)) return 0x7FC0;
    float f = (float)y;
    if (isinf(f) || (double)f == y) return orc_f32_to_bf16_rne(f);
    if (fabs((double)f) > fabs(y)) f = nextafterf(f, 0.0f);
    uint32_t u;
    memcpy(&u, &f, 4);
    u |= 1u;
    memcpy(&f, &u, 4);
    return orc_f32_to_bf16_rne(f);
}

/* ---------------------------------------------------------------------- */
/* Quantiser (load-time packer): scale = bf16_rne(max|w| / 6) per group of  */
/* 32 along K, code = nearest E2M1 value to w / scale in float32, exact     */
/* midpoints to the even mantissa bit, ratios beyond 6 clamp to 6, a zero  */
/* magnitude is code 0, an all-zero group has scale 0 and codes 0.          */
/* ---------------------------------------------------------------------- */
int orc_e2m1_encode(float r)
{
    float a = fabsf(r);
    int m;
    if (a <= 0.25f) m = 0;        /* tie 0.25 -> 0   */
    else if (a < 0.75f) m = 1;    /* tie 0.75 -> 1.0 */
    else if (a <= 1.25f) m = 2;   /* tie 1.25 -> 1.0 */
    else if (a < 1.75f) m = 3;    /* tie 1.75 -> 2.0 */
    else if (a <= 2.5f) m = 4;    /* tie 2.5  -> 2.0 */
    else if (a < 3.5f) m = 5;     /* tie 3.5  -> 4.0 */
    else if (a <= 5.0f) m = 6;    /* tie 5.0  -> 4.0 */
    else m = 7;                   /* (5, inf) -> 6.0 */
    if (m == 0) return 0;
    return (r < 0.0f) ? (m | 8) : m;
}

int orc_quantize(const float* W, int64_t E, int64_t K, int64_t N, uint8_t* codes, uint16_t* scales)
{
    if (!W || !codes || !scales || E < 0 || K <= 0 || N <= 0 || K % 32) return ORC_EINVAL;
    const int64_t G = K / 32;
    memset(codes, 0, (size_t)(E * (K / 2) * N));
    for (int64_t e = 0; e < E; ++e)
        for (int64_t g = 0; g < G; ++g)
            for (int64_t n = 0; n < N; ++n) {
                float mx = 0.0f;
                for (int64_t kk = 0; kk < 32; ++kk) {
                    float a = fabsf(W[(e * K + g * 32 + kk) * N + n]);
                    if (a > mx) mx = a;
                }
                uint16_t sb = orc_f32_to_bf16_rne(mx / 6.0f);
                scales[(e * G + g) * N + n] = sb;
                float s = orc_bf16_to_f32(sb);
                for (int64_t kk = 0; kk < 32; ++kk) {
                    int64_t k = g * 32 + kk;
                    int code = (s == 0.0f) ? 0 : orc_e2m1_encode(W[(e * K + k) * N + n] / s);
                    uint8_t* byte = &codes[(e * (K / 2) + k / 2) * N + n];
                    if (k % 2 == 0) *byte = (uint8_t)((*byte & 0xF0) | code);
                    else            *byte = (uint8_t)((*byte & 0x0F) | (code << 4));
                }
            }
    return ORC_OK;
}

/* Dequantised weight W[k][n] of one expert's [K/2, N] codes / [K/32, N]
 * scales: an exact float32 product (at most 2 + 8 significant bits). */
static float orc_weight(const uint8_t* codes, const uint16_t* scales, int64_t N, int64_t k, int64_t n)
{
    uint8_t byte = codes[(k / 2) * N + n];
    int code = (k % 2 == 0) ? (byte & 0x0F) : (byte >> 4);
    return (float)orc_e2m1_decode(code) * orc_bf16_to_f32(scales[(k / 32) * N + n]);
}

float orc_dequant(const uint8_t* codes, const uint16_t* scales, int64_t N, int64_t k, int64_t n)
{
    return orc_weight(codes, scales, N, k, n);
}

/* ---------------------------------------------------------------------- */
/* Router: top-k by logit, ties to the lower expert index, softmax over the */
/* k selected logits.                                                       */
/* ---------------------------------------------------------------------- */
static int orc_before(const float* l, int a, int b)
{
    /* does expert a come before expert b in (logit desc, index asc) order */
    if (l[a] > l[b]) return 1;
    if (l[a] < l[b]) return 0;
    return a < b;
}

int orc_route(const float* logits, int T, int E, int k, int32_t* idx, float* w)
{
    if (T < 0 || E <= 0 || k < 1 || k > E || (T > 0 && (!logits || !idx || !w))) return ORC_EINVAL;
    char* taken = (char*)malloc((size_t)E);
    if (!taken) return ORC_ENOMEM;
    for (int t = 0; t < T; ++t) {
        const float* l = logits + (int64_t)t * E;
        memset(taken, 0, (size_t)E);
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e)
                if (!taken[e] && (best < 0 || orc_before(l, e, best))) best = e;
            taken[best] = 1;
            idx[(int64_t)t * k + j] = best;
        }
        double l0 = l[idx[(int64_t)t * k]];
        double den = 0.0;
        for (int j = 0; j < k; ++j) den += exp((double)l[idx[(int64_t)t * k + j]] - l0);
        for (int j = 0; j < k; ++j)
            w[(int64_t)t * k + j] = (float)(exp((double)l[idx[(int64_t)t * k + j]] - l0) / den);
    }
    free(taken);
    return ORC_OK;
}

/* ---------------------------------------------------------------------- */
/* INT2 scalar codes ("FireEcho Engine", sections "Quantization Formats":   */
/* INT2, 2 bits, 8x, scalar, for the coldest experts; and "FE-XC / INT2 Cold */
/* Expert Demotion": a scalar 2-bit format for rarely used experts).  The    */
/* pages give no code table; the reading here is the symmetric four-level   */
/* scalar quantiser: a 2-bit unsigned code q decodes to (q - 1.5) times the */
/* bf16 scale of its 32-element group along K, s = bf16_rne(max|w| / 1.5),  */
/* the code of r = w / s is the nearest level, a tie (r = -1, 0 or 1) going */
/* to the level above.  Four codes per byte: the code of k = 4 r + i sits  */
/* in bits 2i and 2i + 1 of byte row r; layout [E][K/4][N], scales          */
/* [E][K/32][N] as for E2M1.                                                */
/* ---------------------------------------------------------------------- */
double orc_int2_decode(int q) { return (double)(q & 3) - 1.5; }

int orc_int2_encode(float r)
{
    if (r < -1.0f) return 0;
    if (r < 0.0f) return 1;
    if (r < 1.0f) return 2;
    return 3;
}

int orc_quantize_int2(const float* W, int64_t E, int64_t K, int64_t N, uint8_t* codes, uint16_t* scales)
{
    if (E < 0 || K <= 0 || N <= 0 || K % 32 || !W || !codes || !scales) return ORC_EINVAL;
    memset(codes, 0, (size_t)(E * (K / 4) * N));
    for (int64_t e = 0; e < E; ++e)
        for (int64_t g = 0; g < K / 32; ++g)
            for (int64_t n = 0; n < N; ++n) {
                float mx = 0.0f;
                for (int64_t kk = 0; kk < 32; ++kk) {
                    const float a = fabsf(W[(e * K + g * 32 + kk) * N + n]);
                    if (a > mx) mx = a;
                }
                const uint16_t sb = orc_f32_to_bf16_rne(mx / 1.5f);
                scales[(e * (K / 32) + g) * N + n] = sb;
                const float sv = orc_bf16_to_f32(sb);
                for (int64_t kk = 0; kk < 32; ++kk) {
                    const int64_t k = g * 32 + kk;
                    const int q = sv != 0.0f ? orc_int2_encode(W[(e * K + k) * N + n] / sv) : 2;
                    codes[(e * (K / 4) + k / 4) * N + n] |= (uint8_t)(q << (2 * (k % 4)));
                }
            }
    return ORC_OK;
}

/* One dequantised INT2 weight of a single expert's [K/4][N] codes / [K/32][N] scales. */
static float orc_weight_int2(const uint8_t* codes, const uint16_t* scales, int64_t N, int64_t k, int64_t n)
{
    const int q = (codes[(k / 4) * N + n] >> (2 * (k % 4))) & 3;
    return (float)orc_int2_decode(q) * orc_bf16_to_f32(scales[(k / 32) * N + n]);
}

float orc_dequant_int2(const uint8_t* codes, const uint16_t* scales, int64_t N, int64_t k, int64_t n)
{
    return orc_weight_int2(codes, scales, N, k, n);
}

/* ---------------------------------------------------------------------- */
/* Router GEMM ("FireEcho Engine", section "Architecture": MoEFFN, the packed */
/* MoE whose dispatch starts from the router's scores; "Speed Optimization   */
/* History" step 1, the router in front of the grouped dispatch):           */
/*   logits[t][e] = sum_{h = 0..H-1} x[t][h] * W_r[e][h]                    */
/* x_bf16 [T][H], w_bf16 [E][H] (expert e's router row), logits [T][E] fp64; */
/* each product of two bf16 values is exact in fp64, and the sum runs in    */
/* the order h = 0, 1, ..., H-1.                                            */
/* ---------------------------------------------------------------------- */
int orc_router_logits(const uint16_t* x_bf16, const uint16_t* w_bf16, int T, int H, int E, double* logits)
{
    if (T < 0 || H <= 0 || E <= 0 || (T > 0 && (!x_bf16 || !w_bf16 || !logits))) return ORC_EINVAL;
    for (int t = 0; t < T; ++t)
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int h = 0; h < H; ++h)
                acc += (double)orc_bf16_to_f32(x_bf16[(int64_t)t * H + h]) *
                       (double)orc_bf16_to_f32(w_bf16[(int64_t)e * H + h]);
            logits[(int64_t)t * E + e] = acc;
        }
    return ORC_OK;
}

/* ---------------------------------------------------------------------- */
/* Grouping: histogram, exclusive scan, pairs ordered by (expert, pair id). */
/* ---------------------------------------------------------------------- */
int orc_group(const int32_t* idx, int T, int k, int E, int32_t* counts, int32_t* offsets,
              int32_t* sorted_pair, int32_t* pair_row)
{
    if (T < 0 || k < 1 || E <= 0 || !counts || !offsets) return ORC_EINVAL;
    const int64_t P = (int64_t)T * k;
    if (P > 0 && (!idx || !sorted_pair || !pair_row)) return ORC_EINVAL;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t p = 0; p < P; ++p) {
        if (idx[p] < 0 || idx[p] >= E) return ORC_EINVAL;
        counts[idx[p]]++;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int64_t pos = 0;
    for (int e = 0; e < E; ++e)
        for (int64_t p = 0; p < P; ++p)
            if (idx[p] == e) {
                sorted_pair[pos] = (int32_t)p;
                pair_row[p] = (int32_t)pos;
                ++pos;
            }
    return ORC_OK;
}

/* ---------------------------------------------------------------------- */
/* The layer.  Expert weights are passed as one pointer per expert (NULL for */
/* an expert the caller did not materialise; routing to it is an error), so */
/* a test can hand over only the experts a token batch touches.            */
/*   gu_codes[e]  : uint8 [H/2][2I]     gu_scales[e] : bf16 [H/32][2I]       */
/*   dn_codes[e]  : uint8 [I/2][H]      dn_scales[e] : bf16 [I/32][H]        */
/*   x_bf16 [T][H], logits [T][E]; outputs y64 [T][H], y_bf16 [T][H]        */
/*   (either may be NULL), act64 [T*k][I] in pair order p = t*k + j (NULL   */
/*   to skip).                                                              */
/* ---------------------------------------------------------------------- */
static float orc_weight_fmt(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t N, int64_t k, int64_t n)
{
    return fmt ? orc_weight_int2(codes, scales, N, k, n) : orc_weight(codes, scales, N, k, n);
}

/* The layer with a format per expert: fmt[e] = 0 E2M1 (codes [K/2][N]), 1 INT2 */
/* (codes [K/4][N]); fmt NULL: every expert E2M1.  Otherwise as             */
/* orc_moe_forward.                                                         */
int orc_moe_forward_fmt(int E, int H, int I, int T, int k, const uint16_t* x_bf16, const float* logits,
                        const uint8_t* fmt, const uint8_t* const* gu_codes, const uint16_t* const* gu_scales,
                        const uint8_t* const* dn_codes, const uint16_t* const* dn_scales, double* y64,
                        uint16_t* y_bf16, double* act64)
{
    if (E <= 0 || H <= 0 || I <= 0 || H % 32 || I % 32 || T < 0 || k < 1 || k > E) return ORC_EINVAL;
    if (T == 0) return ORC_OK;
    if (!x_bf16 || !logits || !gu_codes || !gu_scales || !dn_codes || !dn_scales) return ORC_EINVAL;
    int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
    float* w = (float*)malloc(sizeof(float) * (size_t)k);
    double* x = (double*)malloc(sizeof(double) * (size_t)H);
    double* gu = (double*)malloc(sizeof(double) * 2 * (size_t)I);
    double* act = (double*)malloc(sizeof(double) * (size_t)I);
    double* o = (double*)malloc(sizeof(double) * (size_t)H);
    double* y = (double*)malloc(sizeof(double) * (size_t)H);
    int rc = ORC_OK;
    if (!idx || !w || !x || !gu || !act || !o || !y) { rc = ORC_ENOMEM; goto done; }
    const int64_t N1 = 2 * (int64_t)I;
    for (int t = 0; t < T; ++t) {
        rc = orc_route(logits + (int64_t)t * E, 1, E, k, idx, w);
        if (rc) goto done;
        for (int h = 0; h < H; ++h) x[h] = orc_bf16_to_f32(x_bf16[(int64_t)t * H + h]);
        for (int h = 0; h < H; ++h) y[h] = 0.0;
        for (int j = 0; j < k; ++j) {
            const int e = idx[j];
            if (!gu_codes[e] || !gu_scales[e] || !dn_codes[e] || !dn_scales[e]) { rc = ORC_EINVAL; goto done; }
            const int f = fmt ? fmt[e] : 0;
            /* gate_up: K = H, N = 2I */
            for (int64_t n = 0; n < N1; ++n) gu[n] = 0.0;
            for (int64_t kk = 0; kk < H; ++kk)
                for (int64_t n = 0; n < N1; ++n)
                    gu[n] += x[kk] * (double)orc_weight_fmt(f, gu_codes[e], gu_scales[e], N1, kk, n);
            for (int i = 0; i < I; ++i) {
                double g = gu[i], u = gu[I + i];
                act[i] = g / (1.0 + exp(-g)) * u;
            }
            if (act64) memcpy(act64 + ((int64_t)t * k + j) * I, act, sizeof(double) * (size_t)I);
            /* down: K = I, N = H */
            for (int h = 0; h < H; ++h) o[h] = 0.0;
            for (int64_t kk = 0; kk < I; ++kk)
                for (int64_t h = 0; h < H; ++h)
                    o[h] += act[kk] * (double)orc_weight_fmt(f, dn_codes[e], dn_scales[e], H, kk, h);
            /* weighted combine, slot order */
            for (int h = 0; h < H; ++h) y[h] += (double)w[j] * o[h];
        }
        for (int h = 0; h < H; ++h) {
            if (y64) y64[(int64_t)t * H + h] = y[h];
            if (y_bf16) y_bf16[(int64_t)t * H + h] = orc_f64_to_bf16_rne(y[h]);
        }
    }
done:
    free(idx); free(w); free(x); free(gu); free(act); free(o); free(y);
    return rc;
}

int orc_moe_forward(int E, int H, int I, int T, int k, const uint16_t* x_bf16, const float* logits,
                    const uint8_t* const* gu_codes, const uint16_t* const* gu_scales,
                    const uint8_t* const* dn_codes, const uint16_t* const* dn_scales, double* y64,
                    uint16_t* y_bf16, double* act64)
{
    return orc_moe_forward_fmt(E, H, I, T, k, x_bf16, logits, NULL, gu_codes, gu_scales, dn_codes, dn_scales, y64,
                               y_bf16, act64);
}

/* ---------------------------------------------------------------------- */
/* Block-scaled FP4 variant of the projections (NVFP4).  An approximation  */
/* of the layer above, not its definition: the tensor cores' FP4 rate      */
/* ("FireEcho Engine", "The Goliath Kernel: Why It's Fast": FP4 operands at */
/* the matmul) takes only scale factors that are E4M3 per 16 elements (or   */
/* powers of two per 32), so the BF16 group scales cannot be fed exactly.  */
/* This is the variant's own definition:                                   */
/*                                                                          */
/*   E4M3 (the scale factors): 1 sign, 4 exponent bits (bias 7), 3 mantissa */
/*   bits; exponent field 0 is subnormal, m/8 * 2^-6; 0x7F and 0xFF are NaN; */
/*   the largest finite value is 448 (0x7E).                                 */
/*                                                                          */
/*   NVFP4 encoding of a row of K values v (K a multiple of 16), every step */
/*   in float32:                                                            */
/*     g   = amax(|v|) / 2688          (2688 = 6 * 448: the row's scale)     */
/*     d6  = 6 * g                                                          */
/*     s_b = E4M3(amax_b / d6) for each block b of 16 (nearest, ties to the */
/*           even mantissa, above 448 -> 448; 0 when d6 = 0)               */
/*     q   = E2M1(v * r_b), r_b = 1 / (s_b * g)  (orc_e2m1_encode; 0 when   */
/*           s_b g = 0): the block's fp32 reciprocal, then one product     */
/*   decoded value: E2M1(q) * s_b * g (exact in fp64).                      */
/*                                                                          */
/*   The layer: x (bf16) is encoded per token row; the gate_up and down     */
/*   weights (the packed E2M1 * bf16 values, exact in float32) per output   */
/*   column along K; gate_up and SwiGLU in fp64 on the decoded values; act  */
/*   is rounded to bf16 (the form in which it crosses to the down           */
/*   projection), encoded per pair row, down in fp64; routing and the       */
/*   slot-order combine as in orc_moe_forward.                              */
/* ---------------------------------------------------------------------- */
double orc_e4m3_decode(int byte)
{
    const int b = byte & 0xFF;
    const int e = (b >> 3) & 0xF, m = b & 7;
    if ((b & 0x7F) == 0x7F) return NAN;
    const double mag = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return (b & 0x80) ? -mag : mag;
}

/* Nearest non-negative finite E4M3 value to t >= 0 by search over all of them, */
/* ties to the even code; t above 448 gives 448.                               */
int orc_e4m3_encode(float t)
{
    if (isnan(t)) return 0x7F;
    if (t >= 448.0f) return 0x7E;
    if (t <= 0.0f) return 0;
    int best = 0;
    double bd = fabs((double)t);
    for (int c = 1; c <= 0x7E; ++c) {
        const double d = fabs((double)t - orc_e4m3_decode(c));
        if (d < bd || (d == bd && (c & 1) == 0)) {
            bd = d;
            best = c;
        }
    }
    return best;
}

static void orc_nvfp4_row(const float* v, int64_t K, uint8_t* codes, uint8_t* sf, float* g_out)
{
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k)
        if (fabsf(v[k]) > amax) amax = fabsf(v[k]);
    const float g = amax / 2688.0f;
    const float d6 = 6.0f * g;
    for (int64_t c = 0; c < K / 2; ++c) codes[c] = 0;
    for (int64_t b = 0; b < K / 16; ++b) {
        float ab = 0.0f;
        for (int64_t kk = 0; kk < 16; ++kk)
            if (fabsf(v[b * 16 + kk]) > ab) ab = fabsf(v[b * 16 + kk]);
        const int sb = (d6 > 0.0f) ? orc_e4m3_encode(ab / d6) : 0;
        sf[b] = (uint8_t)sb;
        const float dq = (float)orc_e4m3_decode(sb) * g;
        const float rq = (dq > 0.0f) ? 1.0f / dq : 0.0f;
        for (int64_t kk = 0; kk < 16; ++kk) {
            const int64_t k = b * 16 + kk;
            const int code = (dq > 0.0f) ? orc_e2m1_encode(v[k] * rq) : 0;
            if (k % 2 == 0) codes[k / 2] = (uint8_t)((codes[k / 2] & 0xF0) | code);
            else            codes[k / 2] = (uint8_t)((codes[k / 2] & 0x0F) | (code << 4));
        }
    }
    *g_out = g;
}

/* NVFP4 encoding of R rows of K values: codes [R][K/2] (low nibble = even k), */
/* scale factors [R][K/16] (E4M3 bytes), row scales g [R].                     */
int orc_nvfp4_quantize(const float* V, int64_t R, int64_t K, uint8_t* codes, uint8_t* sf, float* g)
{
    if (!V || !codes || !sf || !g || R < 0 || K <= 0 || K % 16) return ORC_EINVAL;
    for (int64_t r = 0; r < R; ++r) orc_nvfp4_row(V + r * K, K, codes + r * (K / 2), sf + r * (K / 16), g + r);
    return ORC_OK;
}

/* Decoded value of element k of an encoded row. */
static double orc_nvfp4_value(const uint8_t* codes, const uint8_t* sf, float g, int64_t k)
{
    const int code = (k & 1) ? (codes[k / 2] >> 4) : (codes[k / 2] & 0x0F);
    return orc_e2m1_decode(code) * orc_e4m3_decode(sf[k / 16]) * (double)g;
}

/* One expert matrix's columns [K/2][N] codes, [K/32][N] bf16 scales, encoded */
/* column by column along K: qc [N][K/2], qs [N][K/16], qg [N].               */
static void orc_nvfp4_columns(const uint8_t* codes, const uint16_t* scales, int64_t K, int64_t N, uint8_t* qc,
                              uint8_t* qs, float* qg, float* col)
{
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) col[k] = orc_weight(codes, scales, N, k, n);
        orc_nvfp4_row(col, K, qc + n * (K / 2), qs + n * (K / 16), qg + n);
    }
}

typedef struct {
    uint8_t *gc, *gs, *dc, *ds;
    float *gg, *dg;
} orc_nvfp4_expert;

/* The NVFP4 variant of the layer (arguments as orc_moe_forward, E2M1 experts; */
/* act64 [T*k][I] receives the bf16-rounded act in pair order).                */
int orc_moe_forward_nvfp4(int E, int H, int I, int T, int k, const uint16_t* x_bf16, const float* logits,
                          const uint8_t* const* gu_codes, const uint16_t* const* gu_scales,
                          const uint8_t* const* dn_codes, const uint16_t* const* dn_scales, double* y64,
                          uint16_t* y_bf16, double* act64)
{
    if (E <= 0 || H <= 0 || I <= 0 || H % 32 || I % 32 || T < 0 || k < 1 || k > E) return ORC_EINVAL;
    if (T == 0) return ORC_OK;
    if (!x_bf16 || !logits || !gu_codes || !gu_scales || !dn_codes || !dn_scales) return ORC_EINVAL;
    const int64_t N1 = 2 * (int64_t)I;
    int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
    float* w = (float*)malloc(sizeof(float) * (size_t)k);
    float* xf = (float*)malloc(sizeof(float) * (size_t)H);
    uint8_t* xc = (uint8_t*)malloc((size_t)H / 2);
    uint8_t* xs = (uint8_t*)malloc((size_t)H / 16);
    float* af = (float*)malloc(sizeof(float) * (size_t)I);
    uint8_t* ac = (uint8_t*)malloc((size_t)I / 2);
    uint8_t* as = (uint8_t*)malloc((size_t)I / 16);
    float* col = (float*)malloc(sizeof(float) * (size_t)(H > I ? H : I));
    double* gu = (double*)malloc(sizeof(double) * (size_t)N1);
    double* o = (double*)malloc(sizeof(double) * (size_t)H);
    double* y = (double*)malloc(sizeof(double) * (size_t)H);
    orc_nvfp4_expert* ex = (orc_nvfp4_expert*)calloc((size_t)E, sizeof(orc_nvfp4_expert));
    int rc = ORC_OK;
    if (!idx || !w || !xf || !xc || !xs || !af || !ac || !as || !col || !gu || !o || !y || !ex) {
        rc = ORC_ENOMEM;
        goto done;
    }
    for (int t = 0; t < T; ++t) {
        rc = orc_route(logits + (int64_t)t * E, 1, E, k, idx, w);
        if (rc) goto done;
        float gx;
        for (int h = 0; h < H; ++h) xf[h] = orc_bf16_to_f32(x_bf16[(int64_t)t * H + h]);
        orc_nvfp4_row(xf, H, xc, xs, &gx);
        for (int h = 0; h < H; ++h) y[h] = 0.0;
        for (int j = 0; j < k; ++j) {
            const int e = idx[j];
            if (!gu_codes[e] || !gu_scales[e] || !dn_codes[e] || !dn_scales[e]) { rc = ORC_EINVAL; goto done; }
            orc_nvfp4_expert* q = &ex[e];
            if (!q->gc) {   /* encode this expert's weights once */
                q->gc = (uint8_t*)malloc((size_t)(N1 * H / 2));
                q->gs = (uint8_t*)malloc((size_t)(N1 * H / 16));
                q->gg = (float*)malloc(sizeof(float) * (size_t)N1);
                q->dc = (uint8_t*)malloc((size_t)H * (size_t)I / 2);
                q->ds = (uint8_t*)malloc((size_t)H * (size_t)I / 16);
                q->dg = (float*)malloc(sizeof(float) * (size_t)H);
                if (!q->gc || !q->gs || !q->gg || !q->dc || !q->ds || !q->dg) { rc = ORC_ENOMEM; goto done; }
                orc_nvfp4_columns(gu_codes[e], gu_scales[e], H, N1, q->gc, q->gs, q->gg, col);
                orc_nvfp4_columns(dn_codes[e], dn_scales[e], I, H, q->dc, q->ds, q->dg, col);
            }
            /* gate_up: K = H, N = 2I */
            for (int64_t n = 0; n < N1; ++n) {
                double acc = 0.0;
                for (int64_t kk = 0; kk < H; ++kk)
                    acc += orc_nvfp4_value(xc, xs, gx, kk) *
                           orc_nvfp4_value(q->gc + n * (H / 2), q->gs + n * (H / 16), q->gg[n], kk);
                gu[n] = acc;
            }
            for (int i = 0; i < I; ++i) {
                const double gv = gu[i], uv = gu[I + i];
                af[i] = orc_bf16_to_f32(orc_f64_to_bf16_rne(gv / (1.0 + exp(-gv)) * uv));
            }
            if (act64)
                for (int i = 0; i < I; ++i) act64[((int64_t)t * k + j) * I + i] = (double)af[i];
            float ga;
            orc_nvfp4_row(af, I, ac, as, &ga);
            /* down: K = I, N = H */
            for (int64_t h = 0; h < H; ++h) {
                double acc = 0.0;
                for (int64_t kk = 0; kk < I; ++kk)
                    acc += orc_nvfp4_value(ac, as, ga, kk) *
                           orc_nvfp4_value(q->dc + h * (I / 2), q->ds + h * (I / 16), q->dg[h], kk);
                o[h] = acc;
            }
            /* weighted combine, slot order */
            for (int h = 0; h < H; ++h) y[h] += o[h] * (double)w[j];
        }
        for (int h = 0; h < H; ++h) {
            if (y64) y64[(int64_t)t * H + h] = y[h];
            if (y_bf16) y_bf16[(int64_t)t * H + h] = orc_f64_to_bf16_rne(y[h]);
        }
    }
done:
    if (ex)
        for (int e = 0; e < E; ++e) {
            free(ex[e].gc); free(ex[e].gs); free(ex[e].gg); free(ex[e].dc); free(ex[e].ds); free(ex[e].dg);
        }
    free(ex); free(idx); free(w); free(xf); free(xc); free(xs); free(af); free(ac); free(as); free(col);
    free(gu); free(o); free(y);
    return rc;
}
