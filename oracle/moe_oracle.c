/*
 * CPU oracle for the 4-bit routed-expert MoE layer of Step-5-Preview.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow reference that the
 * CUDA library is checked against.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load it.  It shares no code, header,
 * table or constant with the CUDA library, and the library never calls it.
 *
 * Sources (web pages, by title and section):
 *   [Int4]  "Step-5-Preview-Int4-g128": Recipe (RTN + clip search over 17 ratios
 *           in [0.60, 1.00], search in bf16 = storage precision of the scale);
 *           Tensor layout (experts fused as [352, out, in]).
 *   [NVFP4] "Step-5-Preview-NVFP4-Local": Modifications item 2 (E2M1 pairs
 *           U8 [352, R, K/2], weight_scale_2 F32 [352], BF16 activations);
 *           Format (one E4M3 byte per 16 weights, [E, R, C]; dequant =
 *           E2M1 value x E4M3 block scale x weight_scale_2; nibble order
 *           "low nibble first" stated there for the CSF codes).
 *   [Spark] "Step-5-Preview-Spark": At a glance (hidden 4096; a sigmoid
 *           router keeps 8 of 352 routed experts; one shared expert).
 *   [Art]   "Step 5 Preview: 92 narrow layers, and a sparse indexer that scores
 *           blocks of 8": The shape (each token goes to 8 routed SwiGLU experts
 *           and to a shared one, all of width 1536).
 *   [CSF]   "Step-5-Preview-NVFP4-Local", Format (the compressed scale format:
 *           each slab of 16 rows holds their 16 bases and then their 4-bit
 *           codes, the lower nibble of a byte first; exceptions are
 *           (row*C + col) | byte << 24, expert by expert in increasing
 *           position; starts [E+1]; a row's base, in 0..240, is the start of
 *           the 16-value window holding the largest share of its bytes) and
 *           Size.
 *
 * Readings where the pages are silent:
 *   - int4: divisor 7 with clamp [-8, 7]; ratios r_i = (24 + i) / 40, i = 0..16;
 *     candidate scale bf16_rne((r_i * amax) / 7) in fp32; rounding error
 *     sum (q*s - w)^2 accumulated in fp32 in index order; ties keep the larger
 *     ratio; offset-binary nibbles u = q + 8, element 8c+j in bits 4j..4j+3
 *     of word c.
 *   - NVFP4: global g = amax / (6 * 448) per expert matrix (fp32);
 *     block scale sb = e4m3_rne_sat(amax_b / (6 * g)); code =
 *     e2m1_rne_sat(w / (e4m3(sb) * g)); even element in the low nibble.
 *   - Router: l = sum_h x*Wr (fp32, index order) + bias; s = 1/(1+exp(-l))
 *     (fp32); top-k by s, ties to the lower expert id, listed by descending s;
 *     weights s / sum(selected s) (fp32).
 *   - Layer: no routed scaling factor, no shared-expert gate, SwiGLU limit off.
 *   - NVFP4 W4A4 (layers 3-87, quant_algo NVFP4 with an input_scale): the
 *     activation entering a projection is quantised like a weight row, per
 *     16 elements, with the expert's input_scale as its global scale (a static
 *     value, so large blocks saturate at 448 x 6); gate and up read the same
 *     activation, quantised once with the gate's input_scale; the down
 *     projection's input is h rounded to bf16 (the activations between the
 *     projections are bf16), then quantised with the down input_scale.
 *   - CSF: the 4-bit code stored at an exception's position is 0 (the
 *     decoder replaces that byte, so any code would do; 0 is the plainest);
 *     the rows of a slab follow one another, each C/2 bytes.
 *
 * Floating point: quantiser decisions are taken in fp32 (the precision the
 * CUDA library's own quantiser uses, so codes agree bit for bit); dequantised
 * weights are exact in fp32; the layer forward accumulates in fp64.
 *
 * Parity pins: every function here is pinned by tests against facts the pages
 * or mathematics fix (exhaustive code tables, library conversions, the pages'
 * error table, closed forms, brute force).  The absolute layer output has no
 * printed example on the pages; it is pinned only through those invariants and
 * the brute-force dense mixture.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* bf16 <-> fp32                                                             */
/* ------------------------------------------------------------------------ */

float oracle_bf16_to_f32(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* IEEE binary16 -> fp32 (exact): 1 sign, 5 exponent (bias 15), 10 mantissa bits. */
float oracle_f16_to_f32(uint16_t h) {
    int s = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
    float v;
    if (e == 0) v = ldexpf((float)m, -24);                         /* subnormal: m 2^-24 */
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexpf(1.0f + (float)m / 1024.0f, e - 15);
    return s ? -v : v;
}

/* The layer's input activations are bf16 by default; fp16 when set ("Step-5-
 * Preview-Spark", Quality: the release runs activations in fp16).  Only the
 * readers of the input x follow this; intermediates are given as bf16.  The
 * BF16 shared expert computes in bf16, so it reads x rounded to bf16. */
static int g_x_f16 = 0;
void oracle_set_x_f16(int on) { g_x_f16 = on; }

/* Thread control for timing, no part of the arithmetic: every parallel loop
 * here gives each item (a row, an expert, a group) to one thread and no loop
 * reduces across threads, so results do not depend on the count.  n > 0 sets
 * the OpenMP thread count of later calls, n <= 0 restores one thread per host
 * core; returns the count in effect. */
int oracle_set_threads(int n) {
#ifdef _OPENMP
    omp_set_num_threads(n > 0 ? n : omp_get_num_procs());
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}
static float x_to_f32(uint16_t v);

/* Round-to-nearest-even to bf16 (finite inputs). */
uint16_t oracle_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u) {            /* inf / nan: truncate */
        return (uint16_t)((u >> 16) | ((u & 0xffffu) ? 0x40u : 0u));
    }
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

static float x_to_f32(uint16_t v) { return g_x_f16 ? oracle_f16_to_f32(v) : oracle_bf16_to_f32(v); }

/* ------------------------------------------------------------------------ */
/* E2M1 and E4M3 (the two NVFP4 element types)                               */
/* ------------------------------------------------------------------------ */

/* E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit; no inf/nan.
 * Magnitudes for codes 0..7: 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
float oracle_e2m1_decode(uint8_t code) {
    int s = (code >> 3) & 1;
    int e = (code >> 1) & 3;
    int m = code & 1;
    float mag;
    if (e == 0) mag = 0.5f * (float)m;                         /* subnormal */
    else        mag = ldexpf(1.0f + 0.5f * (float)m, e - 1);
    return s ? -mag : mag;
}

/* Nearest E2M1 code, ties to the code with an even (zero) mantissa bit,
 * saturating at 6.  Negative inputs keep the sign bit even when the magnitude
 * rounds to zero (IEEE behaviour). */
uint8_t oracle_e2m1_encode(float v) {
    uint8_t sign = 0;
    float a = v;
    if (v < 0.0f) { sign = 8; a = -v; }
    if (a >= 6.0f) return (uint8_t)(sign | 7);       /* saturate at the largest magnitude */
    uint8_t best = 0;
    float best_d = INFINITY;
    for (uint8_t c = 0; c < 8; c++) {
        float d = fabsf(oracle_e2m1_decode(c) - a);
        if (d < best_d || (d == best_d && (c & 1) == 0)) { best = c; best_d = d; }
    }
    return (uint8_t)(sign | best);
}

/* E4M3 "FN": 1 sign, 4 exponent (bias 7), 3 mantissa bits, subnormals,
 * S.1111.111 is NaN, no infinity; largest finite 448. */
float oracle_e4m3_decode(uint8_t b) {
    int s = (b >> 7) & 1;
    int e = (b >> 3) & 15;
    int m = b & 7;
    float mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) mag = ldexpf((float)m, -9);                    /* m/8 * 2^(1-7) */
    else        mag = ldexpf(1.0f + (float)m / 8.0f, e - 7);
    return s ? -mag : mag;
}

/* Nearest non-negative E4M3 byte for v >= 0, ties to an even mantissa,
 * saturating at 448.  Codes 0x00..0x7E decode to strictly increasing values,
 * so a binary search finds the bracketing pair. */
uint8_t oracle_e4m3_encode_nonneg(float v) {
    if (!(v > 0.0f)) return 0;
    if (v >= 448.0f) return 0x7E;
    int lo = 0, hi = 0x7E;                       /* decode(lo) <= v < decode(hi) */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (oracle_e4m3_decode((uint8_t)mid) <= v) lo = mid; else hi = mid;
    }
    float dl = v - oracle_e4m3_decode((uint8_t)lo);
    float dh = oracle_e4m3_decode((uint8_t)hi) - v;
    if (dl < dh) return (uint8_t)lo;
    if (dh < dl) return (uint8_t)hi;
    return (uint8_t)(((lo & 1) == 0) ? lo : hi);
}

/* ------------------------------------------------------------------------ */
/* int4 symmetric g128 with clip search  [Int4] Recipe                       */
/* ------------------------------------------------------------------------ */

#define I4_GROUP 128
#define I4_NRATIO 17

/* Clip ratio i of the search, i = 0..16: (24 + i) / 40, evenly spaced from 0.60 to 1.00. */
static float clip_ratio(int i) { return (float)(24 + i) / 40.0f; }

static int32_t rne_clamp_q(float w, float s) {
    /* Division in double is exact enough that rint() sees the true
     * rounding of w/s (w and s carry 8 significant bits each). */
    double q = rint((double)w / (double)s);
    if (q < -8.0) q = -8.0;
    if (q > 7.0) q = 7.0;
    return (int32_t)q;
}

/* One group of n <= 128 bf16 weights -> scale (bf16 bits) and codes q.
 * Candidates are ratios first_ratio..16; first_ratio = 16 is the plain
 * max-abs scale (the page's "max-abs scale" row), 0 the full clip search. */
static void quant_int4_group(const uint16_t* w, int n, int first_ratio,
                             uint16_t* scale_out, int8_t* q_out, int* ratio_out) {
    float wf[I4_GROUP];
    float amax = 0.0f;
    for (int i = 0; i < n; i++) {
        wf[i] = oracle_bf16_to_f32(w[i]);
        float a = fabsf(wf[i]);
        if (a > amax) amax = a;
    }
    if (amax == 0.0f) {
        *scale_out = 0;
        for (int i = 0; i < n; i++) q_out[i] = 0;
        if (ratio_out) *ratio_out = I4_NRATIO - 1;
        return;
    }
    float best_err = INFINITY;
    uint16_t best_s = 0;
    int best_i = I4_NRATIO - 1;
    /* Larger ratios first; a later candidate must be strictly better. */
    for (int i = I4_NRATIO - 1; i >= first_ratio; i--) {
        float t = clip_ratio(i) * amax;
        float sf = t / 7.0f;
        uint16_t sb = oracle_f32_to_bf16(sf);
        float s = oracle_bf16_to_f32(sb);
        if (s == 0.0f) continue;
        float err = 0.0f;
        for (int j = 0; j < n; j++) {
            int32_t q = rne_clamp_q(wf[j], s);
            float d = (float)q * s - wf[j];
            err = err + d * d;
        }
        if (err < best_err) { best_err = err; best_s = sb; best_i = i; }
    }
    float s = oracle_bf16_to_f32(best_s);
    for (int j = 0; j < n; j++) q_out[j] = (int8_t)(s == 0.0f ? 0 : rne_clamp_q(wf[j], s));
    *scale_out = best_s;
    if (ratio_out) *ratio_out = best_i;
}

/* Quantise a bf16 matrix [rows, cols] (cols % 128 == 0).
 * packed: int32 [rows, cols/8]; scales: bf16 bits [rows, cols/128];
 * q (optional): int8 [rows, cols]; ratio_idx (optional): int32 [rows, cols/128].
 * first_ratio: 0 for the clip search of the recipe, 16 for max-abs only. */
void oracle_quant_int4_g128(const uint16_t* w, int64_t rows, int64_t cols,
                            int32_t* packed, uint16_t* scales, int8_t* q,
                            int32_t* ratio_idx, int first_ratio) {
    int64_t ng = cols / I4_GROUP;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        int8_t qg[I4_GROUP];
        for (int64_t g = 0; g < ng; g++) {
            int ri;
            quant_int4_group(w + r * cols + g * I4_GROUP, I4_GROUP, first_ratio,
                             &scales[r * ng + g], qg, &ri);
            if (ratio_idx) ratio_idx[r * ng + g] = ri;
            for (int c = 0; c < I4_GROUP / 8; c++) {
                uint32_t word = 0;
                for (int j = 0; j < 8; j++) {
                    uint32_t u = (uint32_t)(qg[c * 8 + j] + 8) & 0xFu;
                    word |= u << (4 * j);
                }
                packed[r * (cols / 8) + g * (I4_GROUP / 8) + c] = (int32_t)word;
            }
            if (q) memcpy(q + r * cols + g * I4_GROUP, qg, I4_GROUP);
        }
    }
}

/* Exact dequantisation: fp32(q) * fp32(s). */
void oracle_dequant_int4_g128(const int32_t* packed, const uint16_t* scales,
                              int64_t rows, int64_t cols, float* out) {
    int64_t ng = cols / I4_GROUP;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t c = 0; c < cols; c++) {
            uint32_t word = (uint32_t)packed[r * (cols / 8) + c / 8];
            int32_t q = (int32_t)((word >> (4 * (c % 8))) & 0xFu) - 8;
            float s = oracle_bf16_to_f32(scales[r * ng + c / I4_GROUP]);
            out[r * cols + c] = (float)q * s;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* NVFP4 (W4A16)  [NVFP4] Modifications item 2, Format                       */
/* ------------------------------------------------------------------------ */

#define FP4_BLOCK 16

/* Quantise one expert matrix [rows, cols] (cols % 16 == 0).
 * packed: uint8 [rows, cols/2]; scales: uint8 E4M3 [rows, cols/16];
 * *global: fp32 weight_scale_2. */
void oracle_quant_nvfp4(const uint16_t* w, int64_t rows, int64_t cols,
                        uint8_t* packed, uint8_t* scales, float* global) {
    float amax = 0.0f;
    for (int64_t i = 0; i < rows * cols; i++) {
        float a = fabsf(oracle_bf16_to_f32(w[i]));
        if (a > amax) amax = a;
    }
    float g = amax / (6.0f * 448.0f);
    *global = g;
    int64_t nb = cols / FP4_BLOCK;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t b = 0; b < nb; b++) {
            const uint16_t* wb = w + r * cols + b * FP4_BLOCK;
            float wf[FP4_BLOCK];
            float amax_b = 0.0f;
            for (int j = 0; j < FP4_BLOCK; j++) {
                wf[j] = oracle_bf16_to_f32(wb[j]);
                float a = fabsf(wf[j]);
                if (a > amax_b) amax_b = a;
            }
            uint8_t sb = 0;
            if (g > 0.0f) sb = oracle_e4m3_encode_nonneg(amax_b / (6.0f * g));
            scales[r * nb + b] = sb;
            float eff = oracle_e4m3_decode(sb) * g;
            uint8_t codes[FP4_BLOCK];
            for (int j = 0; j < FP4_BLOCK; j++)
                codes[j] = (eff > 0.0f) ? oracle_e2m1_encode(wf[j] / eff) : 0;
            for (int j = 0; j < FP4_BLOCK / 2; j++)
                packed[r * (cols / 2) + b * (FP4_BLOCK / 2) + j] =
                    (uint8_t)(codes[2 * j] | (codes[2 * j + 1] << 4));
        }
    }
}

/* Exact dequantisation in fp32: (E2M1 value x E4M3 scale) x global.  The
 * first product is exact (at most 5 significant bits); one rounding follows. */
void oracle_dequant_nvfp4(const uint8_t* packed, const uint8_t* scales, float global,
                          int64_t rows, int64_t cols, float* out) {
    int64_t nb = cols / FP4_BLOCK;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t c = 0; c < cols; c++) {
            uint8_t byte = packed[r * (cols / 2) + c / 2];
            uint8_t code = (c % 2 == 0) ? (byte & 0xF) : (byte >> 4);
            float sb = oracle_e4m3_decode(scales[r * nb + c / FP4_BLOCK]);
            out[r * cols + c] = (oracle_e2m1_decode(code) * sb) * global;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Expert banks (fused [E, out, in], [Int4] Tensor layout / [NVFP4] Format)  */
/* ------------------------------------------------------------------------ */

typedef struct {
    int32_t fmt;            /* 0 int4 g128, 1 nvfp4, 2 bf16 */
    int32_t E, out, in;
    const void* packed;     /* int4: int32 [E,out,in/8]; nvfp4: u8 [E,out,in/2]; bf16: u16 [E,out,in] */
    const void* scales;     /* int4: bf16 bits [E,out,in/128]; nvfp4: u8 [E,out,in/16]; bf16: NULL */
    const float* global_scale; /* nvfp4: [E]; else NULL */
} oracle_bank;

/* Dequantise expert e of a bank into fp32 [out, in]. */
void oracle_dequant_expert(const oracle_bank* b, int e, float* w) {
    int64_t rows = b->out, cols = b->in;
    if (b->fmt == 0) {
        oracle_dequant_int4_g128((const int32_t*)b->packed + (int64_t)e * rows * (cols / 8),
                                 (const uint16_t*)b->scales + (int64_t)e * rows * (cols / I4_GROUP),
                                 rows, cols, w);
    } else if (b->fmt == 1) {
        oracle_dequant_nvfp4((const uint8_t*)b->packed + (int64_t)e * rows * (cols / 2),
                             (const uint8_t*)b->scales + (int64_t)e * rows * (cols / FP4_BLOCK),
                             b->global_scale[e], rows, cols, w);
    } else {
        const uint16_t* src = (const uint16_t*)b->packed + (int64_t)e * rows * cols;
        for (int64_t i = 0; i < rows * cols; i++) w[i] = oracle_bf16_to_f32(src[i]);
    }
}

/* ------------------------------------------------------------------------ */
/* Router  [Spark] At a glance: sigmoid router, top-8                        */
/* ------------------------------------------------------------------------ */

/* x: bf16 bits [T,H]; Wr: fp32 [E,H]; bias: fp32 [E] or NULL.
 * ids: int32 [T,k]; w: fp32 [T,k]; scores (optional): fp32 [T,E] sigmoids. */
void oracle_route(const uint16_t* x, int64_t T, int64_t H, const float* Wr,
                  const float* bias, int64_t E, int k, int32_t* ids, float* w,
                  float* scores) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < T; t++) {
        float* s = (float*)malloc(sizeof(float) * E);
        char* taken = (char*)calloc(E, 1);
        for (int64_t e = 0; e < E; e++) {
            float l = 0.0f;
            for (int64_t h = 0; h < H; h++)
                l = l + x_to_f32(x[t * H + h]) * Wr[e * H + h];
            if (bias) l = l + bias[e];
            s[e] = 1.0f / (1.0f + expf(-l));
            if (scores) scores[t * E + e] = s[e];
        }
        float sum = 0.0f;
        for (int j = 0; j < k; j++) {
            int64_t best = -1;
            for (int64_t e = 0; e < E; e++) {
                if (taken[e]) continue;
                if (best < 0 || s[e] > s[best]) best = e;   /* strict: lower id wins ties */
            }
            taken[best] = 1;
            ids[t * k + j] = (int32_t)best;
            w[t * k + j] = s[best];
            sum = sum + s[best];
        }
        for (int j = 0; j < k; j++) w[t * k + j] = w[t * k + j] / sum;
        free(s);
        free(taken);
    }
}

/* ------------------------------------------------------------------------ */
/* Token -> expert bucketing                                                 */
/* ------------------------------------------------------------------------ */

/* Stable counting sort of the R = T*k slots (slot = t*k + j) by expert id.
 * offsets: [E+1]; row_slot[r] = slot at permuted row r; slot_row = inverse.
 * Returns 0, or -1 if an id is out of range. */
int oracle_permute(const int32_t* ids, int64_t T, int k, int64_t E,
                   int32_t* offsets, int32_t* row_slot, int32_t* slot_row) {
    int64_t R = T * k;
    int64_t* count = (int64_t*)calloc(E, sizeof(int64_t));
    for (int64_t s = 0; s < R; s++) {
        if (ids[s] < 0 || ids[s] >= E) { free(count); return -1; }
        count[ids[s]]++;
    }
    offsets[0] = 0;
    for (int64_t e = 0; e < E; e++) offsets[e + 1] = offsets[e] + (int32_t)count[e];
    memset(count, 0, sizeof(int64_t) * E);
    for (int64_t s = 0; s < R; s++) {
        int64_t e = ids[s];
        int64_t r = offsets[e] + count[e]++;
        row_slot[r] = (int32_t)s;
        slot_row[s] = (int32_t)r;
    }
    free(count);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Layer forward  [Art] The shape: 8 routed SwiGLU experts + 1 shared        */
/* ------------------------------------------------------------------------ */

static double silu(double v) { return v / (1.0 + exp(-v)); }

/* y[i,:] for tokens tok[i], i < n:
 *   y = FFN_shared(x) + sum_j w[t,j] * FFN_{ids[t,j]}(x),
 *   FFN(x) = Wd (silu(Wg x) * (Wu x)),
 * with fp32-exact dequantised weights and fp64 accumulation.  Experts are
 * visited one at a time (each dequantised once); each expert serves the
 * (token, slot) pairs that selected it.  sh_* may be NULL (no shared expert).
 * Returns 0, or -1 on an out-of-range id. */
int oracle_moe_forward(const uint16_t* x, int64_t T, int64_t H, int64_t F, int k,
                       const int32_t* ids, const float* topk_w,
                       const oracle_bank* gate, const oracle_bank* up,
                       const oracle_bank* down, const oracle_bank* sh_gate,
                       const oracle_bank* sh_up, const oracle_bank* sh_down,
                       const int32_t* tok, int64_t n, double* y) {
    int64_t E = gate->E;
    for (int64_t i = 0; i < n; i++)
        for (int64_t j = 0; j < k; j++) {
            int32_t e = ids[tok[i] * k + j];
            if (e < 0 || e >= E) return -1;
        }
    double* xd = (double*)malloc(sizeof(double) * n * H);
    for (int64_t i = 0; i < n; i++)
        for (int64_t h = 0; h < H; h++)
            xd[i * H + h] = (double)x_to_f32(x[tok[i] * H + h]);
    /* the BF16 shared expert computes in bf16: with fp16 inputs it reads x rounded to bf16 */
    double* xs = (double*)malloc(sizeof(double) * n * H);
    for (int64_t i = 0; i < n * H; i++)
        xs[i] = g_x_f16 ? (double)oracle_bf16_to_f32(oracle_f32_to_bf16((float)xd[i])) : xd[i];
    memset(y, 0, sizeof(double) * n * H);

    float* wg = (float*)malloc(sizeof(float) * F * H);
    float* wu = (float*)malloc(sizeof(float) * F * H);
    float* wd = (float*)malloc(sizeof(float) * H * F);
    double* hbuf = (double*)malloc(sizeof(double) * F);
    int64_t* who = (int64_t*)malloc(sizeof(int64_t) * n * k);

    int64_t nexp = E + (sh_gate ? 1 : 0);
    for (int64_t e = 0; e < nexp; e++) {
        int shared = (e == E);
        int64_t m = 0;                           /* (token index i, weight slot) pairs */
        if (shared) {
            for (int64_t i = 0; i < n; i++) who[m++] = -1 - i;  /* negative: shared, weight 1 */
        } else {
            for (int64_t i = 0; i < n; i++)
                for (int64_t j = 0; j < k; j++)
                    if (ids[tok[i] * k + j] == e) who[m++] = i * k + j;
        }
        if (m == 0) continue;
        oracle_dequant_expert(shared ? sh_gate : gate, shared ? 0 : (int)e, wg);
        oracle_dequant_expert(shared ? sh_up : up, shared ? 0 : (int)e, wu);
        oracle_dequant_expert(shared ? sh_down : down, shared ? 0 : (int)e, wd);
        for (int64_t p = 0; p < m; p++) {
            int64_t i, slot;
            double wt;
            if (who[p] < 0) { i = -1 - who[p]; slot = -1; wt = 1.0; }
            else { i = who[p] / k; slot = who[p] % k; wt = (double)topk_w[tok[i] * k + slot]; }
            const double* xi = (shared ? xs : xd) + i * H;
            #pragma omp parallel for schedule(static)
            for (int64_t f = 0; f < F; f++) {
                double g = 0.0, u = 0.0;
                for (int64_t h = 0; h < H; h++) {
                    g += (double)wg[f * H + h] * xi[h];
                    u += (double)wu[f * H + h] * xi[h];
                }
                hbuf[f] = silu(g) * u;
            }
            #pragma omp parallel for schedule(static)
            for (int64_t h = 0; h < H; h++) {
                double acc = 0.0;
                for (int64_t f = 0; f < F; f++) acc += (double)wd[h * F + f] * hbuf[f];
                y[i * H + h] += wt * acc;
            }
        }
    }
    free(xd); free(xs); free(wg); free(wu); free(wd); free(hbuf); free(who);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Per-step definitions (one per library call), fp64 accumulation           */
/* ------------------------------------------------------------------------ */

/* Gate/up + SwiGLU over bucketed rows: for expert e and row r in
 * [offsets[e], offsets[e+1]), token t = row_slot[r] / k:
 *   h[r, f] = silu(x[t] . Wg[e,f,:]) * (x[t] . Wu[e,f,:]).
 * Rows listed in `rows` (n of them) are computed; h is [n, F]. */
void oracle_grouped_swiglu(const uint16_t* x, int64_t H, int64_t F, int k,
                           const int32_t* offsets, const int32_t* row_slot,
                           const oracle_bank* gate, const oracle_bank* up,
                           const int32_t* rows, int64_t n, double* h) {
    int64_t E = gate->E;
    float* wg = (float*)malloc(sizeof(float) * F * H);
    float* wu = (float*)malloc(sizeof(float) * F * H);
    for (int64_t e = 0; e < E; e++) {
        int any = 0;
        for (int64_t i = 0; i < n; i++)
            if (rows[i] >= offsets[e] && rows[i] < offsets[e + 1]) any = 1;
        if (!any) continue;
        oracle_dequant_expert(gate, (int)e, wg);
        oracle_dequant_expert(up, (int)e, wu);
        for (int64_t i = 0; i < n; i++) {
            int32_t r = rows[i];
            if (r < offsets[e] || r >= offsets[e + 1]) continue;
            int64_t t = row_slot[r] / k;
            #pragma omp parallel for schedule(static)
            for (int64_t f = 0; f < F; f++) {
                double g = 0.0, u = 0.0;
                for (int64_t hh = 0; hh < H; hh++) {
                    double xv = (double)x_to_f32(x[t * H + hh]);
                    g += (double)wg[f * H + hh] * xv;
                    u += (double)wu[f * H + hh] * xv;
                }
                h[i * F + f] = silu(g) * u;
            }
        }
    }
    free(wg);
    free(wu);
}

/* Down projection with the routing weight: for row r of expert e,
 *   y[r, :] = w[row_slot[r]] * (Wd[e] h_in[r])     (w = 1 if topk_w is NULL).
 * h_in: bf16 bits [R, F]; rows listed in `rows`; y is [n, H]. */
void oracle_grouped_down(const uint16_t* h_in, int64_t F, int64_t H,
                         const int32_t* offsets, const int32_t* row_slot,
                         const float* topk_w, const oracle_bank* down,
                         const int32_t* rows, int64_t n, double* y) {
    int64_t E = down->E;
    float* wd = (float*)malloc(sizeof(float) * H * F);
    for (int64_t e = 0; e < E; e++) {
        int any = 0;
        for (int64_t i = 0; i < n; i++)
            if (rows[i] >= offsets[e] && rows[i] < offsets[e + 1]) any = 1;
        if (!any) continue;
        oracle_dequant_expert(down, (int)e, wd);
        for (int64_t i = 0; i < n; i++) {
            int32_t r = rows[i];
            if (r < offsets[e] || r >= offsets[e + 1]) continue;
            double wt = topk_w ? (double)topk_w[row_slot[r]] : 1.0;
            #pragma omp parallel for schedule(static)
            for (int64_t hh = 0; hh < H; hh++) {
                double acc = 0.0;
                for (int64_t f = 0; f < F; f++)
                    acc += (double)wd[hh * F + f] * (double)oracle_bf16_to_f32(h_in[(int64_t)r * F + f]);
                y[i * H + hh] = wt * acc;
            }
        }
    }
    free(wd);
}

/* Combine: y[t] = shared[t] + sum_j y_perm[slot_row[t*k + j]] (fp64).
 * y_perm: bf16 bits [T*k, H]; shared: bf16 bits [T, H] or NULL.
 * A slot whose row is negative was dropped by the bucketing (its expert id
 * was out of range) and contributes nothing. */
void oracle_combine(const uint16_t* y_perm, const int32_t* slot_row, int64_t T, int k,
                    int64_t H, const uint16_t* shared, double* y) {
    for (int64_t t = 0; t < T; t++)
        for (int64_t hh = 0; hh < H; hh++) {
            double acc = shared ? (double)oracle_bf16_to_f32(shared[t * H + hh]) : 0.0;
            for (int j = 0; j < k; j++) {
                int32_t r = slot_row[t * k + j];
                if (r < 0) continue;
                acc += (double)oracle_bf16_to_f32(y_perm[(int64_t)r * H + hh]);
            }
            y[t * H + hh] = acc;
        }
}


/* ------------------------------------------------------------------------ */
/* Compressed scale format (CSF)  [CSF] Format                               */
/* ------------------------------------------------------------------------ */

/* Base of one row of n scale bytes: the smallest b in 0..240 that puts the
 * largest number of the row's bytes inside [b, b + 15]. */
static int csf_row_base(const uint8_t* row, int64_t n) {
    int64_t hist[256];
    memset(hist, 0, sizeof(hist));
    for (int64_t i = 0; i < n; i++) hist[row[i]]++;
    int best = 0;
    int64_t best_cnt = -1;
    for (int b = 0; b <= 240; b++) {
        int64_t cnt = 0;
        for (int v = b; v < b + 16; v++) cnt += hist[v];
        if (cnt > best_cnt) { best_cnt = cnt; best = b; }      /* strict: the lowest base wins ties */
    }
    return best;
}

/* Encode scales u8 [E, R, C] (R % 16 == 0, C even).
 * fixed: u8 [E, R/16, 16 * (1 + C/2)]: per slab of 16 rows, the 16 row bases,
 *        then the rows' codes in row order, C/2 bytes each, column 2j in the
 *        low nibble of byte j and column 2j + 1 in its high nibble;
 * starts: int64 [E + 1], expert e's entries are exceptions[starts[e] .. starts[e+1]);
 * exceptions: uint32 [n] (may be NULL to count only), (row * C + col) | byte << 24
 *        for every byte outside its row's window, in (expert, row, col) order.
 * Returns n, the number of exceptions. */
int64_t oracle_csf_encode(const uint8_t* scales, int64_t E, int64_t R, int64_t C,
                          uint8_t* fixed, int64_t* starts, uint32_t* exceptions) {
    int64_t slab = 16 * (1 + C / 2);
    int64_t n = 0;
    for (int64_t e = 0; e < E; e++) {
        starts[e] = n;
        for (int64_t r = 0; r < R; r++) {
            const uint8_t* row = scales + (e * R + r) * C;
            int base = csf_row_base(row, C);
            uint8_t* sl = fixed + (e * (R / 16) + r / 16) * slab;
            sl[r % 16] = (uint8_t)base;
            uint8_t* codes = sl + 16 + (r % 16) * (C / 2);
            for (int64_t j = 0; j < C / 2; j++) codes[j] = 0;
            for (int64_t c = 0; c < C; c++) {
                int v = row[c];
                int code = 0;
                if (v >= base && v <= base + 15) {
                    code = v - base;
                } else {
                    if (exceptions) exceptions[n] = (uint32_t)(r * C + c) | ((uint32_t)v << 24);
                    n++;
                }
                codes[c / 2] |= (uint8_t)(code << (4 * (c % 2)));
            }
        }
    }
    starts[E] = n;
    return n;
}

/* Decode back to scales u8 [E, R, C]: base + code, then each exception of
 * expert e replaces the byte at its position. */
void oracle_csf_decode(const uint8_t* fixed, const uint32_t* exceptions, const int64_t* starts,
                       int64_t E, int64_t R, int64_t C, uint8_t* scales) {
    int64_t slab = 16 * (1 + C / 2);
    for (int64_t e = 0; e < E; e++) {
        for (int64_t r = 0; r < R; r++) {
            const uint8_t* sl = fixed + (e * (R / 16) + r / 16) * slab;
            int base = sl[r % 16];
            const uint8_t* codes = sl + 16 + (r % 16) * (C / 2);
            for (int64_t c = 0; c < C; c++) {
                int code = (codes[c / 2] >> (4 * (c % 2))) & 0xF;
                scales[(e * R + r) * C + c] = (uint8_t)(base + code);
            }
        }
        for (int64_t i = starts[e]; i < starts[e + 1]; i++) {
            uint32_t x = exceptions[i];
            int64_t pos = (int64_t)(x & 0xFFFFFFu);
            scales[e * R * C + pos] = (uint8_t)(x >> 24);
        }
    }
}


/* ------------------------------------------------------------------------ */
/* NVFP4 W4A4  [NVFP4] Modifications items 2-3 (quant_algo NVFP4 with an     */
/* input_scale for layers 3-87; group size 16)                              */
/* ------------------------------------------------------------------------ */

/* Quantise one activation row of n bf16 values (n % 16 == 0) with global g:
 * per block sb = e4m3_rne_sat(amax_b / (6 g)), codes e2m1_rne_sat(x / (e4m3(sb) g));
 * returns the dequantised values e2m1 x e4m3 x g in xq (fp32, one rounding),
 * and (optionally) the packed codes [n/2] and block scales [n/16]. */
static void act_quant_row(const float* x, int64_t n, float g, float* xq, uint8_t* packed, uint8_t* scales) {
    for (int64_t b = 0; b < n / FP4_BLOCK; b++) {
        const float* xb = x + b * FP4_BLOCK;
        float amax_b = 0.0f;
        for (int j = 0; j < FP4_BLOCK; j++) {
            float a = fabsf(xb[j]);
            if (a > amax_b) amax_b = a;
        }
        uint8_t sb = 0;
        if (g > 0.0f) sb = oracle_e4m3_encode_nonneg(amax_b / (6.0f * g));
        float eff = oracle_e4m3_decode(sb) * g;
        if (scales) scales[b] = sb;
        for (int j = 0; j < FP4_BLOCK; j++) {
            uint8_t code = (eff > 0.0f) ? oracle_e2m1_encode(xb[j] / eff) : 0;
            xq[b * FP4_BLOCK + j] = (oracle_e2m1_decode(code) * oracle_e4m3_decode(sb)) * g;
            if (packed) {
                int64_t c = b * FP4_BLOCK + j;
                if (c % 2 == 0) packed[c / 2] = code;
                else packed[c / 2] = (uint8_t)(packed[c / 2] | (code << 4));
            }
        }
    }
}

/* Activation quantiser: bf16 rows [rows, cols], row r with global g[r]
 * -> packed u8 [rows, cols/2] (even element in the low nibble), scales u8
 * E4M3 [rows, cols/16], and the dequantised values fp32 [rows, cols]
 * (any output may be NULL). */
void oracle_act_quant_nvfp4(const uint16_t* x, int64_t rows, int64_t cols, const float* g,
                            uint8_t* packed, uint8_t* scales, float* xq) {
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        float* xf = (float*)malloc(sizeof(float) * cols);
        float* q = (float*)malloc(sizeof(float) * cols);
        for (int64_t c = 0; c < cols; c++) xf[c] = oracle_bf16_to_f32(x[r * cols + c]);
        act_quant_row(xf, cols, g[r], q, packed ? packed + r * (cols / 2) : NULL,
                      scales ? scales + r * (cols / FP4_BLOCK) : NULL);
        if (xq) memcpy(xq + r * cols, q, sizeof(float) * cols);
        free(xf);
        free(q);
    }
}

/* W4A4 gate/up + SwiGLU over bucketed rows: for row r of expert e (token
 * t = row_slot[r] / k), xq = x[t] quantised with in_scale[e], then
 * h[r] = silu(Wg[e] xq) * (Wu[e] xq) in fp64.  h is [n, F]. */
void oracle_grouped_swiglu_w4a4(const uint16_t* x, int64_t H, int64_t F, int k,
                                const int32_t* offsets, const int32_t* row_slot,
                                const oracle_bank* gate, const oracle_bank* up, const float* in_scale,
                                const int32_t* rows, int64_t n, double* h) {
    int64_t E = gate->E;
    float* wg = (float*)malloc(sizeof(float) * F * H);
    float* wu = (float*)malloc(sizeof(float) * F * H);
    float* xf = (float*)malloc(sizeof(float) * H);
    float* xq = (float*)malloc(sizeof(float) * H);
    for (int64_t e = 0; e < E; e++) {
        int any = 0;
        for (int64_t i = 0; i < n; i++)
            if (rows[i] >= offsets[e] && rows[i] < offsets[e + 1]) any = 1;
        if (!any) continue;
        oracle_dequant_expert(gate, (int)e, wg);
        oracle_dequant_expert(up, (int)e, wu);
        for (int64_t i = 0; i < n; i++) {
            int32_t r = rows[i];
            if (r < offsets[e] || r >= offsets[e + 1]) continue;
            int64_t t = row_slot[r] / k;
            for (int64_t hh = 0; hh < H; hh++) xf[hh] = x_to_f32(x[t * H + hh]);
            act_quant_row(xf, H, in_scale[e], xq, NULL, NULL);
            #pragma omp parallel for schedule(static)
            for (int64_t f = 0; f < F; f++) {
                double g = 0.0, u = 0.0;
                for (int64_t hh = 0; hh < H; hh++) {
                    g += (double)wg[f * H + hh] * (double)xq[hh];
                    u += (double)wu[f * H + hh] * (double)xq[hh];
                }
                h[i * F + f] = silu(g) * u;
            }
        }
    }
    free(wg); free(wu); free(xf); free(xq);
}

/* W4A4 down projection: for row r of expert e, hq = h_in[r] (bf16) quantised
 * with in_scale[e]; y[r] = w[row_slot[r]] * (Wd[e] hq) (w = 1 if topk_w is NULL). */
void oracle_grouped_down_w4a4(const uint16_t* h_in, int64_t F, int64_t H,
                              const int32_t* offsets, const int32_t* row_slot,
                              const float* topk_w, const oracle_bank* down, const float* in_scale,
                              const int32_t* rows, int64_t n, double* y) {
    int64_t E = down->E;
    float* wd = (float*)malloc(sizeof(float) * H * F);
    float* hf = (float*)malloc(sizeof(float) * F);
    float* hq = (float*)malloc(sizeof(float) * F);
    for (int64_t e = 0; e < E; e++) {
        int any = 0;
        for (int64_t i = 0; i < n; i++)
            if (rows[i] >= offsets[e] && rows[i] < offsets[e + 1]) any = 1;
        if (!any) continue;
        oracle_dequant_expert(down, (int)e, wd);
        for (int64_t i = 0; i < n; i++) {
            int32_t r = rows[i];
            if (r < offsets[e] || r >= offsets[e + 1]) continue;
            double wt = topk_w ? (double)topk_w[row_slot[r]] : 1.0;
            for (int64_t f = 0; f < F; f++) hf[f] = oracle_bf16_to_f32(h_in[(int64_t)r * F + f]);
            act_quant_row(hf, F, in_scale[e], hq, NULL, NULL);
            #pragma omp parallel for schedule(static)
            for (int64_t hh = 0; hh < H; hh++) {
                double acc = 0.0;
                for (int64_t f = 0; f < F; f++) acc += (double)wd[hh * F + f] * (double)hq[f];
                y[i * H + hh] = wt * acc;
            }
        }
    }
    free(wd); free(hf); free(hq);
}

/* W4A4 layer forward for the listed tokens: as oracle_moe_forward, with each
 * routed expert's input quantised (in_gu[e] for gate/up, in_dn[e] for down,
 * the down input being h rounded to bf16).  The shared expert is BF16 and
 * reads x unquantised.  Returns 0, or -1 on an out-of-range id. */
int oracle_moe_forward_w4a4(const uint16_t* x, int64_t T, int64_t H, int64_t F, int k,
                            const int32_t* ids, const float* topk_w,
                            const oracle_bank* gate, const oracle_bank* up, const oracle_bank* down,
                            const float* in_gu, const float* in_dn,
                            const oracle_bank* sh_gate, const oracle_bank* sh_up, const oracle_bank* sh_down,
                            const int32_t* tok, int64_t n, double* y) {
    int64_t E = gate->E;
    for (int64_t i = 0; i < n; i++)
        for (int64_t j = 0; j < k; j++) {
            int32_t e = ids[tok[i] * k + j];
            if (e < 0 || e >= E) return -1;
        }
    /* routed part through the per-step definitions, one (token, slot) row at a time */
    memset(y, 0, sizeof(double) * n * H);
    double* hrow = (double*)malloc(sizeof(double) * F);
    uint16_t* hb = (uint16_t*)malloc(sizeof(uint16_t) * F);
    double* yrow = (double*)malloc(sizeof(double) * H);
    for (int64_t i = 0; i < n; i++) {
        for (int64_t j = 0; j < k; j++) {
            int32_t e = ids[tok[i] * k + j];
            /* a one-row problem: expert e owns row 0, which holds slot tok[i]*k + j of token tok[i] */
            int32_t* off = (int32_t*)calloc(E + 1, sizeof(int32_t));
            for (int64_t q = e + 1; q <= E; q++) off[q] = 1;
            int32_t slot = (int32_t)(tok[i] * k + j);
            int32_t row0 = 0;
            oracle_grouped_swiglu_w4a4(x, H, F, k, off, &slot, gate, up, in_gu, &row0, 1, hrow);
            for (int64_t f = 0; f < F; f++) hb[f] = oracle_f32_to_bf16((float)hrow[f]);
            oracle_grouped_down_w4a4(hb, F, H, off, &slot, topk_w, down, in_dn, &row0, 1, yrow);
            for (int64_t hh = 0; hh < H; hh++) y[i * H + hh] += yrow[hh];
            free(off);
        }
    }
    if (sh_gate) {                           /* shared expert: BF16 weights, x unquantised, weight 1 */
        float* wg = (float*)malloc(sizeof(float) * F * H);
        float* wu = (float*)malloc(sizeof(float) * F * H);
        float* wd = (float*)malloc(sizeof(float) * H * F);
        oracle_dequant_expert(sh_gate, 0, wg);
        oracle_dequant_expert(sh_up, 0, wu);
        oracle_dequant_expert(sh_down, 0, wd);
        for (int64_t i = 0; i < n; i++) {
            const uint16_t* xt = x + (int64_t)tok[i] * H;
            #pragma omp parallel for schedule(static)
            for (int64_t f = 0; f < F; f++) {
                double g = 0.0, u = 0.0;
                for (int64_t hh = 0; hh < H; hh++) {
                    float xf32 = x_to_f32(xt[hh]);
                    /* the BF16 shared expert: x rounded to bf16 when x is fp16 */
                    double xv = g_x_f16 ? (double)oracle_bf16_to_f32(oracle_f32_to_bf16(xf32)) : (double)xf32;
                    g += (double)wg[f * H + hh] * xv;
                    u += (double)wu[f * H + hh] * xv;
                }
                hrow[f] = silu(g) * u;
            }
            #pragma omp parallel for schedule(static)
            for (int64_t hh = 0; hh < H; hh++) {
                double acc = 0.0;
                for (int64_t f = 0; f < F; f++) acc += (double)wd[hh * F + f] * hrow[f];
                y[i * H + hh] += acc;
            }
        }
        free(wg); free(wu); free(wd);
    }
    free(hrow); free(hb); free(yrow);
    return 0;
}
