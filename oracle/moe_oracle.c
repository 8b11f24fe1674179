/*
 * moe_oracle.c -- plain, slow CPU oracle of the MoE expert-FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path links, loads or calls
 * this file; only the test suite, the smoke check and the benchmark's CPU
 * baseline do. It shares no code with the CUDA library.
 *
 * What the layer computes (its plain definition):
 *
 *   out[t] = sum_{j<k} w[t,j] * FFN_{e[t,j]}(x[t])
 *   FFN_e(x) = W_d[e] * (silu(W_g[e] x) (.) (W_u[e] x)),  silu(g) = g / (1 + exp(-g))
 *
 * Sources:
 *  - InfiniLM PR #500, "T2-1-3 Qwen3-MoE inference optimisation" report,
 *    §2.1 (Qwen3-MoE routing: top-k softmax, no shared expert, no bias) and
 *    §2.2 (bucket the routing indices into per-expert counts and a
 *    permutation; gather the activations by that permutation; three grouped
 *    GEMMs gate/up/down with SwiGLU between them; scale by the routing
 *    weights and scatter back to the tokens).
 *  - FlashInfer PR #7196 analysis ("CuTe DSL W4A16 MoE optimisation and
 *    bit-exact tests"), §1 (moe_finalize: slot 0 is a round-to-nearest fp32
 *    multiply, later slots are round-to-nearest fp32 FMAs in slot order, no
 *    flush-to-zero, signed zero kept) and §2-§3 (W4A16: int4 weights decoded
 *    to bf16 with a per-group scale before the MMA).
 *
 * Precision: dot products accumulate in double, are rounded once to fp32 (the
 * "fp32-accumulated" value), and the layer's bf16 rounding points are kept
 * where the layer has them: act = bf16(silu(g) * u), y = bf16(down output),
 * out = bf16(finalize accumulator). Finalize is emulated exactly in fp32.
 * Build flags: -O2 -ffp-contract=off, no fast-math; FTZ/DAZ are cleared at
 * each entry point that does fp32 arithmetic.
 *
 * Readings of points the sources leave open (each also stated where used):
 *  R1 top-k selects on the fp32 logits (softmax is monotone in them): slot
 *     order is descending logit, equal logits go to the lower expert id,
 *     -0 equals +0 and NaN ranks as -inf.
 *  R2 weights are renormalised over the k selected experts.
 *  R3 rows [0,I) of W_gu[e] are the gate projection and rows [I,2I) the up
 *     projection.
 *  R4 the permutation is stable: within one expert, pairs p = t*k + j keep
 *     ascending p (ascending token).
 *  R5 perm[r] = pair id p; inv_perm[p] = r.
 *  R6 the routing weight is applied in finalize only; y is the unscaled
 *     bf16 down-projection output.
 *  R7 int4: the low nibble of byte b is K index 2b, the high nibble 2b+1,
 *     two's complement in [-8,7]; one bf16 scale per 128 consecutive K
 *     elements of a row; w = bf16(q * scale).
 *  R8 bf16 rounding is round-to-nearest-even; NaN stays NaN.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif
#if defined(__x86_64__) || defined(__i386__)
#include <xmmintrin.h>
#endif

/* ---- scalar helpers ----------------------------------------------------- */

static void no_ftz_daz(void) {
#if defined(__x86_64__) || defined(__i386__)
    /* MXCSR bit 15 = FTZ, bit 6 = DAZ. */
    _mm_setcsr(_mm_getcsr() & ~(0x8000u | 0x0040u));
#endif
}

static float bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round-to-nearest-even fp32 -> bf16 (R8). */
static uint16_t f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* Sign-extended nibble n (0..15) as the int4 value (R7). */
static int int4_value(unsigned n) { return (n & 8u) ? (int)n - 16 : (int)n; }

/* w = bf16(q * scale); the fp32 product is exact (<= 12 significant bits). */
static uint16_t dequant_one(const uint8_t *row_q, const uint16_t *row_s, int kidx) {
    unsigned byte = row_q[kidx >> 1];
    unsigned nib = (kidx & 1) ? (byte >> 4) : (byte & 15u);
    float q = (float)int4_value(nib);
    float s = bf16_to_f32(row_s[kidx / 128]);
    return f32_to_bf16(q * s);
}

/* ---- MXFP8 (OCP Microscaling Formats (MX) v1.0: E4M3 elements, one E8M0
 * scale per 32 consecutive elements) ----------------------------------------
 * E4M3 ("fn" variant): sign, 4-bit exponent with bias 7, 3-bit mantissa; no
 * infinities; 0x7F / 0xFF are NaN; the largest finite magnitude is 448 =
 * 1.75 * 2^8; subnormals are m * 2^-9. E8M0: 2^(code - 127), code 255 NaN.
 */
static double e4m3_value(uint8_t b) {
    int sign = b >> 7, ex = (b >> 3) & 15, m = b & 7;
    double v;
    if (ex == 15 && m == 7) return NAN;
    if (ex == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, ex - 7);
    return sign ? -v : v;
}

static double e8m0_value(uint8_t c) { return c == 255 ? NAN : ldexp(1.0, (int)c - 127); }

/* Round-to-nearest-even conversion to E4M3 with saturation to +-448 (every
 * magnitude >= 448 gives 448; NaN gives 0x7F). */
static uint8_t e4m3_rne_satfinite(float x) {
    if (x != x) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0;
    double a = fabs((double)x);
    if (a >= 448.0) return sign | 0x7E;
    if (a == 0.0) return sign;
    int ex;
    frexp(a, &ex);                       /* a = fr * 2^ex, fr in [0.5, 1) */
    int E = ex - 1;                      /* a = (2 fr) * 2^E, 2 fr in [1, 2) */
    double units;                        /* a in units of the spacing at a */
    int field;
    if (E < -6) {                        /* subnormal range: spacing 2^-9 */
        units = ldexp(a, 9);
        field = 0;
    } else {
        units = ldexp(a, 3 - E);         /* in [8, 16): 8 + mantissa */
        field = E + 7;
    }
    double r = nearbyint(units);         /* round half to even (default mode) */
    int q = (int)r;
    if (field == 0) {
        if (q >= 8) return sign | (1 << 3);          /* rounds up to 2^-6 */
        return sign | (uint8_t)q;
    }
    if (q >= 16) { q = 8; ++field; }                 /* mantissa carry */
    if (field > 15 || (field == 15 && q - 8 == 7)) return sign | 0x7E;
    return sign | (uint8_t)((field << 3) | (q - 8));
}

/* MX quantisation of a row of K bf16 values (K a multiple of 32), OCP MX
 * v1.0 §6.3: per block of 32, shared exponent e = floor(log2(max |x|)) - 8
 * (8 = the largest E4M3 exponent), clamped to [-127, 127] (0 for an
 * all-zero block gives code 0), then each element x / 2^e converted to E4M3
 * with round-to-nearest-even and saturation. The division by 2^e is exact
 * in fp32 for these operands, so it is done in fp32. */
void oracle_mx_quantize(const uint16_t *x, int rows, int K, uint8_t *q, uint8_t *scales) {
    no_ftz_daz();
    for (int r = 0; r < rows; ++r) {
        for (int b = 0; b < K / 32; ++b) {
            const uint16_t *xb = x + (size_t)r * K + (size_t)b * 32;
            float amax = 0.0f;
            for (int i = 0; i < 32; ++i) {
                float v = fabsf(bf16_to_f32(xb[i]));
                if (v > amax) amax = v;
            }
            int e;
            if (amax == 0.0f) {
                e = -127;
            } else {
                int ex;
                frexp((double)amax, &ex);
                e = (ex - 1) - 8;
                if (e < -127) e = -127;
                if (e > 127) e = 127;
            }
            scales[(size_t)r * (K / 32) + b] = (uint8_t)(e + 127);
            float inv = (float)ldexp(1.0, -e);
            for (int i = 0; i < 32; ++i)
                q[(size_t)r * K + (size_t)b * 32 + i] = e4m3_rne_satfinite(bf16_to_f32(xb[i]) * inv);
        }
    }
}

/* ---- MXFP4 weights (OCP MX v1.0: E2M1 elements, one E8M0 scale per 32) ------
 * E2M1: sign bit 3, 2-bit exponent field (bits 2-1, bias 1), 1-bit mantissa
 * (bit 0); field 0 is subnormal (m * 2^-1), otherwise (1 + m/2) * 2^(field-1);
 * no infinities or NaN. Two elements per byte, the even K index in the low
 * nibble (the int4 layout's packing). */
static double e2m1_value(unsigned code) {
    int sign = (code >> 3) & 1, ex = (code >> 1) & 3, m = code & 1;
    double v = ex == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, ex - 1);
    return sign ? -v : v;
}

static double mx4_value(const uint8_t *row_q, const uint8_t *row_s, int k) {
    uint8_t b = row_q[k / 2];
    return e2m1_value((k & 1) ? (b >> 4) : (b & 15)) * e8m0_value(row_s[k / 32]);
}

void oracle_mx4_dequantize(const uint8_t *q, const uint8_t *scales, int rows, int K, double *out) {
    for (int r = 0; r < rows; ++r)
        for (int k = 0; k < K; ++k)
            out[(size_t)r * K + k] = mx4_value(q + (size_t)r * (K / 2), scales + (size_t)r * (K / 32), k);
}

/* Decoded value of element k of an MX row: E4M3 element times its block's E8M0 scale. */
static double mx_value(const uint8_t *row_q, const uint8_t *row_s, int k) {
    return e4m3_value(row_q[k]) * e8m0_value(row_s[k / 32]);
}

void oracle_mx_dequantize(const uint8_t *q, const uint8_t *scales, int rows, int K, double *out) {
    for (int r = 0; r < rows; ++r)
        for (int k = 0; k < K; ++k)
            out[(size_t)r * K + k] = mx_value(q + (size_t)r * K, scales + (size_t)r * (K / 32), k);
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* ---- step 1: routing ------------------------------------------------------
 * Keep the k experts with the largest softmax probabilities (R1), then
 * renormalise their probabilities to sum to one (R2). InfiniLM PR #500 §2.1,
 * §2.4 (op::topksoftmax); the renormalisation is Qwen3's norm_topk_prob.
 *
 * Softmax is strictly increasing in the logit, so the k most probable experts
 * are the k largest fp32 logits; the selection compares the logits as given,
 * never a rounded probability (two distinct logits can round to the same
 * probability in any finite precision). Equal logits go to the lower expert
 * id; -0 equals +0, as in IEEE comparison; a NaN logit ranks as -inf.
 * The weights are exp(l_j - l_0) / sum_{i<k} exp(l_i - l_0) in double, l_0 the
 * largest logit: the full-softmax denominator cancels in the renormalisation.
 * Returns 0, or -1 on bad sizes.
 */

/* The value a logit ranks with: NaN as -inf, -0 as +0. */
static double rank_value(float l) {
    if (l != l) return -INFINITY;
    if (l == 0.0f) return 0.0;
    return (double)l;
}

/* Does expert a come before expert b (larger logit, then lower id)? */
static int ranks_before(const float *l, int a, int b) {
    double va = rank_value(l[a]), vb = rank_value(l[b]);
    if (va != vb) return va > vb;
    return a < b;
}

int oracle_route(const float *logits, int T, int E, int k, int32_t *ids, float *w) {
    if (T < 0 || E < 1 || k < 1 || k > E) return -1;
    int bad = 0;
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        const float *l = logits + (size_t)t * E;
        int32_t *id = ids + (size_t)t * k;
        char *taken = (char *)calloc((size_t)E, 1);
        double *p = (double *)malloc(sizeof(double) * (size_t)k);
        if (!taken || !p) { bad = 1; free(taken); free(p); continue; }
        /* selection: k passes, each takes the first expert in rank order */
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e)
                if (!taken[e] && (best < 0 || ranks_before(l, e, best))) best = e;
            taken[best] = 1;
            id[j] = best;
        }
        /* renormalised softmax over the selected logits, summed in slot order */
        double l0 = rank_value(l[id[0]]), s = 0.0;
        for (int j = 0; j < k; ++j) {
            p[j] = exp(rank_value(l[id[j]]) - l0);
            s += p[j];
        }
        for (int j = 0; j < k; ++j) w[(size_t)t * k + j] = (float)(p[j] / s);
        free(taken);
        free(p);
    }
    return bad ? -1 : 0;
}

/* ---- step 2: bucketing ----------------------------------------------------
 * Counting sort of the flat pair list p = t*k + j by expert id, stable in p
 * (R4, R5). InfiniLM PR #500 §2.2 step 1. Returns 0, or -1 if an id is out of
 * range (outputs are then undefined).
 */
int oracle_permute(const int32_t *ids, int P, int E, int32_t *counts, int32_t *offsets,
                   int32_t *perm, int32_t *inv_perm) {
    if (P < 0 || E < 1) return -1;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int p = 0; p < P; ++p) {
        if (ids[p] < 0 || ids[p] >= E) return -1;
        counts[ids[p]]++;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t *fill = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    if (!fill) return -1;
    for (int e = 0; e < E; ++e) fill[e] = offsets[e];
    for (int p = 0; p < P; ++p) {
        int r = fill[ids[p]]++;
        perm[r] = p;
        inv_perm[p] = r;
    }
    free(fill);
    return 0;
}

/* ---- step 3: gather -------------------------------------------------------
 * hidden_perm[r] = hidden[perm[r] / k]. InfiniLM PR #500 §2.2 step 2.
 */
void oracle_gather(const uint16_t *hidden, const int32_t *perm, int P, int H, int k,
                   uint16_t *hidden_perm) {
    for (int r = 0; r < P; ++r)
        memcpy(hidden_perm + (size_t)r * H, hidden + (size_t)(perm[r] / k) * H, sizeof(uint16_t) * (size_t)H);
}

/* ---- step 7: W4A16 weight decoding -----------------------------------------
 * out[r][c] = bf16(q[r][c] * scale[r][c/128]) (R7). FlashInfer PR #7196
 * analysis §2 (W4A16: 4-bit weights, 16-bit activations) and §3 (exact
 * reference covering bf16 weight decoding).
 */
void oracle_dequant_int4(const uint8_t *q, const uint16_t *scales, int rows, int K, uint16_t *out) {
    no_ftz_daz();
    for (int r = 0; r < rows; ++r)
        for (int c = 0; c < K; ++c)
            out[(size_t)r * K + c] = dequant_one(q + (size_t)r * (K / 2), scales + (size_t)r * (K / 128), c);
}

/* ---- steps 4-5: one expert's FFN on one activation row ---------------------
 * act[i] = bf16(silu(g_i) * u_i),  g = W_g x, u = W_u x  (R3), InfiniLM PR
 * #500 §2.2 (gate/up grouped GEMM, then SwiGLU);
 * y[h] = bf16(sum_i act[i] * W_d[h][i]) (R6), the down grouped GEMM.
 * Weights are bf16 (fmt 0), int4 + bf16 scales (fmt 1, decoded per element)
 * MXFP8 (fmt 2: E4M3 + one E8M0 scale per 32 K, decoded per element; the
 * activation row x, and act before the down projection, are MX-quantised
 * first, since the block-scaled MMA takes both operands in MX form) or MXFP4
 * (fmt 3: E2M1 + one E8M0 scale per 32 K, with activations MX-quantised to
 * E4M3 as for fmt 2: FP4 weights times FP8 activations).
 */
static double weight_at(int fmt, const void *w, const void *s, int K, int row, int col) {
    if (fmt == 0) return (double)bf16_to_f32(((const uint16_t *)w)[(size_t)row * K + col]);
    if (fmt == 1)
        return (double)bf16_to_f32(dequant_one((const uint8_t *)w + (size_t)row * (K / 2),
                                               (const uint16_t *)s + (size_t)row * (K / 128), col));
    if (fmt == 3)
        return mx4_value((const uint8_t *)w + (size_t)row * (K / 2), (const uint8_t *)s + (size_t)row * (K / 32), col);
    return mx_value((const uint8_t *)w + (size_t)row * K, (const uint8_t *)s + (size_t)row * (K / 32), col);
}

/* The activation row as the MMA sees it: bf16 values, or for fmt 2 and 3 the
 * decoded MXFP8 quantisation of the row. xv has K entries. */
static void activation_values(int fmt, const uint16_t *x, int K, double *xv) {
    if (fmt < 2) {
        for (int k = 0; k < K; ++k) xv[k] = (double)bf16_to_f32(x[k]);
        return;
    }
    uint8_t *q = (uint8_t *)malloc((size_t)K);
    uint8_t *sc = (uint8_t *)malloc((size_t)K / 32);
    oracle_mx_quantize(x, 1, K, q, sc);
    for (int k = 0; k < K; ++k) xv[k] = mx_value(q, sc, k);
    free(q);
    free(sc);
}

void oracle_expert_gate_up(int fmt, const uint16_t *x, const void *w_gu, const void *w_gu_s, int H, int I,
                           uint16_t *act) {
    no_ftz_daz();
    double *xv = (double *)malloc(sizeof(double) * (size_t)H);
    activation_values(fmt, x, H, xv);
    for (int i = 0; i < I; ++i) {
        double g = 0.0, u = 0.0;
        for (int h = 0; h < H; ++h) {
            g += xv[h] * weight_at(fmt, w_gu, w_gu_s, H, i, h);
            u += xv[h] * weight_at(fmt, w_gu, w_gu_s, H, I + i, h);
        }
        float gf = (float)g, uf = (float)u;
        double silu = (double)gf / (1.0 + exp(-(double)gf));
        act[i] = f32_to_bf16((float)(silu * (double)uf));
    }
    free(xv);
}

void oracle_expert_down(int fmt, const uint16_t *act, const void *w_d, const void *w_d_s, int H, int I,
                        uint16_t *y) {
    no_ftz_daz();
    double *av = (double *)malloc(sizeof(double) * (size_t)I);
    activation_values(fmt, act, I, av);
    for (int h = 0; h < H; ++h) {
        double acc = 0.0;
        for (int i = 0; i < I; ++i) acc += av[i] * weight_at(fmt, w_d, w_d_s, I, h, i);
        y[h] = f32_to_bf16((float)acc);
    }
    free(av);
}

void oracle_expert_ffn(int fmt, const uint16_t *x, const void *w_gu, const void *w_gu_s,
                       const void *w_d, const void *w_d_s, int H, int I,
                       uint16_t *act, uint16_t *y) {
    oracle_expert_gate_up(fmt, x, w_gu, w_gu_s, H, I, act);
    oracle_expert_down(fmt, act, w_d, w_d_s, H, I, y);
}

/* ---- step 6: finalize / unpermute ------------------------------------------
 * out[t][h] = bf16(acc), acc = v_0 * w_0 (fp32 multiply), then
 * acc = fma(v_j, w_j, acc) for j = 1..k-1 in slot order, round to nearest,
 * no FTZ, v_j = y[inv_perm[t*k+j]][h]. FlashInfer PR #7196 analysis §1
 * (moe_finalize.py: _mul_rn for slot 0, _fma_rn without .ftz afterwards).
 */
static float combine_slots(const float *v, const float *w, int k) {
    float acc = v[0] * w[0];  /* one fp32 multiply; -ffp-contract=off keeps it unfused */
    for (int j = 1; j < k; ++j) acc = fmaf(v[j], w[j], acc);
    return acc;
}

void oracle_finalize(const uint16_t *y, const float *w, const int32_t *inv_perm, int T, int H, int k,
                     uint16_t *out) {
    no_ftz_daz();
#pragma omp parallel
    {
        no_ftz_daz();
        float *v = (float *)malloc(sizeof(float) * (size_t)(k > 0 ? k : 1));
#pragma omp for schedule(static)
        for (int t = 0; t < T; ++t) {
            for (int h = 0; h < H; ++h) {
                for (int j = 0; j < k; ++j)
                    v[j] = bf16_to_f32(y[(size_t)inv_perm[(size_t)t * k + j] * H + h]);
                out[(size_t)t * H + h] = f32_to_bf16(combine_slots(v, w + (size_t)t * k, k));
            }
        }
        free(v);
    }
}

/* ---- the whole layer --------------------------------------------------------
 * route -> permute -> gather -> per-expert FFN over its rows -> finalize,
 * the order of InfiniLM PR #500 §2.2. Intermediates are returned so that each
 * step of the GPU path can be compared with its own stage. fmt 0: bf16
 * weights [E,2I,H] and [E,H,I]; fmt 1: int4 [E,2I,H/2], [E,H,I/2] with bf16
 * scales [E,2I,H/128], [E,H,I/128].
 */
/* Every permuted row r through its expert's FFN: row r of expert e's segment
 * [offsets[e], offsets[e+1]) is token perm[r] / K through expert e; rows are
 * independent. */
/* Bytes of one expert's weight matrix [rows, K] and of its scales in format fmt. */
static size_t weight_bytes(int fmt, int rows, int K) {
    return fmt == 0 ? (size_t)rows * K * 2 : fmt == 2 ? (size_t)rows * K : (size_t)rows * (K / 2);
}
static size_t scale_bytes(int fmt, int rows, int K) {
    return fmt == 1 ? (size_t)rows * (K / 128) * 2 : fmt >= 2 ? (size_t)rows * (K / 32) : 0;
}

static void ffn_rows(int fmt, const uint16_t *hidden, const void *w_gu, const void *w_gu_s, const void *w_d,
                     const void *w_d_s, int H, int I, int K, int P, const int32_t *ids, const int32_t *perm,
                     uint16_t *act, uint16_t *y) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < P; ++r) {
        int p = perm[r], t = p / K, e = ids[p];
        const char *wgu_e = (const char *)w_gu + (size_t)e * weight_bytes(fmt, 2 * I, H);
        const char *wd_e = (const char *)w_d + (size_t)e * weight_bytes(fmt, H, I);
        const char *sgu_e = fmt ? (const char *)w_gu_s + (size_t)e * scale_bytes(fmt, 2 * I, H) : NULL;
        const char *sd_e = fmt ? (const char *)w_d_s + (size_t)e * scale_bytes(fmt, H, I) : NULL;
        oracle_expert_ffn(fmt, hidden + (size_t)t * H, wgu_e, sgu_e, wd_e, sd_e, H, I,
                          act + (size_t)r * I, y + (size_t)r * H);
    }
}

int oracle_forward(int fmt, const uint16_t *hidden, const float *logits,
                   const void *w_gu, const void *w_gu_s, const void *w_d, const void *w_d_s,
                   int T, int H, int I, int E, int k,
                   int32_t *ids, float *w, int32_t *counts, int32_t *offsets,
                   int32_t *perm, int32_t *inv_perm, uint16_t *act, uint16_t *y, uint16_t *out) {
    if (T < 0 || H < 1 || I < 1 || k < 1 || k > E) return -1;
    if ((fmt == 1 && (H % 128 || I % 128)) || (fmt >= 2 && (H % 32 || I % 32)) || fmt < 0 || fmt > 3) return -1;
    int P = T * k;
    if (oracle_route(logits, T, E, k, ids, w)) return -1;
    if (oracle_permute(ids, P, E, counts, offsets, perm, inv_perm)) return -1;
    ffn_rows(fmt, hidden, w_gu, w_gu_s, w_d, w_d_s, H, I, k, P, ids, perm, act, y);
    oracle_finalize(y, w, inv_perm, T, H, k, out);
    return 0;
}

/* ---- shared experts -----------------------------------------------------------
 * GC-MoE abstract (MoE layers with shared experts beside the routed ones):
 *   out[t] = sum_{j<k} w_j FFN_{e_j}(x_t) + sum_{s<S} FFN_{E+s}(x_t)
 * The S shared experts are experts E..E+S-1 of the weight arrays; every
 * token takes them as extra slots k..k+S-1 with weight 1, after its routed
 * slots, and the layer proceeds over E+S experts and k+S slots, so the
 * finalize sum adds them after the routed slots (fma with weight 1 is an
 * add rounded once). ids, w are [T, k+S]; counts, offsets are over E+S.
 */
int oracle_forward_shared(int fmt, const uint16_t *hidden, const float *logits,
                          const void *w_gu, const void *w_gu_s, const void *w_d, const void *w_d_s,
                          int T, int H, int I, int E, int k, int S,
                          int32_t *ids, float *w, int32_t *counts, int32_t *offsets,
                          int32_t *perm, int32_t *inv_perm, uint16_t *act, uint16_t *y, uint16_t *out) {
    if (S < 0) return -1;
    if (S == 0) return oracle_forward(fmt, hidden, logits, w_gu, w_gu_s, w_d, w_d_s, T, H, I, E, k,
                                      ids, w, counts, offsets, perm, inv_perm, act, y, out);
    if (T < 0 || H < 1 || I < 1 || k < 1 || k > E) return -1;
    if ((fmt == 1 && (H % 128 || I % 128)) || (fmt >= 2 && (H % 32 || I % 32)) || fmt < 0 || fmt > 3) return -1;
    int K = k + S, P = T * K;
    int32_t *ids_k = (int32_t *)malloc(sizeof(int32_t) * (size_t)(T > 0 ? T : 1) * k);
    float *w_k = (float *)malloc(sizeof(float) * (size_t)(T > 0 ? T : 1) * k);
    if (!ids_k || !w_k) { free(ids_k); free(w_k); return -1; }
    int rc = oracle_route(logits, T, E, k, ids_k, w_k);
    for (int t = 0; rc == 0 && t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            ids[(size_t)t * K + j] = ids_k[(size_t)t * k + j];
            w[(size_t)t * K + j] = w_k[(size_t)t * k + j];
        }
        for (int s2 = 0; s2 < S; ++s2) {
            ids[(size_t)t * K + k + s2] = E + s2;
            w[(size_t)t * K + k + s2] = 1.0f;
        }
    }
    free(ids_k);
    free(w_k);
    if (rc) return -1;
    if (oracle_permute(ids, P, E + S, counts, offsets, perm, inv_perm)) return -1;
    ffn_rows(fmt, hidden, w_gu, w_gu_s, w_d, w_d_s, H, I, K, P, ids, perm, act, y);
    oracle_finalize(y, w, inv_perm, T, H, K, out);
    return 0;
}

/* The same layer for a subset of tokens only (used where the full layer is
 * too slow for the oracle): routes the listed tokens, evaluates the FFN of
 * each of their k pairs in slot order, and combines in slot order exactly as
 * finalize does. out_rows[n] receives token tokens[n]; ids_out/w_out are
 * [n_tokens, k].
 */
int oracle_forward_tokens(int fmt, const uint16_t *hidden, const float *logits,
                          const void *w_gu, const void *w_gu_s, const void *w_d, const void *w_d_s,
                          int T, int H, int I, int E, int k, const int32_t *tokens, int n_tokens,
                          int32_t *ids_out, float *w_out, uint16_t *out_rows) {
    if (T < 0 || H < 1 || I < 1 || k < 1 || k > E || n_tokens < 0) return -1;
    if ((fmt == 1 && (H % 128 || I % 128)) || (fmt >= 2 && (H % 32 || I % 32)) || fmt < 0 || fmt > 3) return -1;
    for (int n = 0; n < n_tokens; ++n) {
        if (tokens[n] < 0 || tokens[n] >= T) return -1;
        if (oracle_route(logits + (size_t)tokens[n] * E, 1, E, k, ids_out + (size_t)n * k, w_out + (size_t)n * k))
            return -1;
    }
    int npairs = n_tokens * k;
    uint16_t *ybuf = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(npairs > 0 ? npairs : 1) * H);
    if (!ybuf) return -1;
    int bad = 0;
#pragma omp parallel
    {
        uint16_t *abuf = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)I);
        if (!abuf) bad = 1;
#pragma omp for schedule(dynamic, 1)
        for (int q = 0; q < npairs; ++q) {
            if (!abuf) continue;
            int n = q / k;
            int e = ids_out[q];
            const char *wgu_e = (const char *)w_gu + (size_t)e * weight_bytes(fmt, 2 * I, H);
            const char *wd_e = (const char *)w_d + (size_t)e * weight_bytes(fmt, H, I);
            const char *sgu_e = fmt ? (const char *)w_gu_s + (size_t)e * scale_bytes(fmt, 2 * I, H) : NULL;
            const char *sd_e = fmt ? (const char *)w_d_s + (size_t)e * scale_bytes(fmt, H, I) : NULL;
            oracle_expert_ffn(fmt, hidden + (size_t)tokens[n] * H, wgu_e, sgu_e, wd_e, sd_e, H, I,
                              abuf, ybuf + (size_t)q * H);
        }
        free(abuf);
    }
    if (!bad) {
        /* the pairs of token n sit at rows n*k + j, so an identity inverse
           permutation over ybuf gives the slot-ordered combine */
        int32_t *ident = (int32_t *)malloc(sizeof(int32_t) * (size_t)(npairs > 0 ? npairs : 1));
        if (!ident) { free(ybuf); return -1; }
        for (int q = 0; q < npairs; ++q) ident[q] = q;
        oracle_finalize(ybuf, w_out, ident, n_tokens, H, k, out_rows);
        free(ident);
    }
    free(ybuf);
    return bad ? -1 : 0;
}
