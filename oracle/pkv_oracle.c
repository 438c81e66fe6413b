/*
 * pkv_oracle.c -- plain, slow, fp64 CPU oracle for the paged-KV decode path.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the reference the CUDA library is
 * checked against.  Only the test suite, the package smoke check and the
 * CPU-baseline leg of the benchmark may load it; the product path never does.
 * It shares no code, header, helper or constant with the CUDA library.
 *
 * What it computes (each function below names its source passage):
 *   - RoPE on the new token's q and k, then the k/v write into the physical
 *     slot of a block-structured cache (orc_kv_append);
 *   - single-query attention softmax(q K^T * scale) V over the tokens a
 *     sequence's block table lists (orc_paged_decode), written out as the
 *     plain two-pass definition: no online softmax, no split, no blocking;
 *   - two self-check variants of the same definition: attention over a
 *     contiguous K/V array (orc_contiguous_decode) and full-prefix causal
 *     attention over a whole sequence (orc_causal_prefill);
 *   - the same append and decode over an 8-bit floating-point cache
 *     (orc_kv_append_e4m3, orc_paged_decode_e4m3): each cached element is an
 *     E4M3 code times a per-tensor scale.
 *
 * Sources:
 *   [BOOK]    "Inference From Scratch" (book intro), "What you will build" and
 *             the chapter table: ch. 4 KV cache, ch. 8 online softmax / flash
 *             attention, ch. 10 "Paged attention, block tables", ch. 11 prefix
 *             caching with block reuse.
 *   [PROJ]    "The Project: Serve Your Own LLM", milestones table M2 (choose
 *             n_kv_heads: MHA/GQA/MQA), M13b (paged greedy tokens equal the
 *             full-recompute reference), M13c (block pool smaller than the
 *             worst case).
 *   [LIFS]    "LLM Inference from Scratch", Architecture overview: Llama-style
 *             decoder with RoPE and causal attention; M1 KV cache with
 *             prefill/decode equivalence.
 *   [WARP]    "warpllama", Milestones: static KV cache + single-token decode,
 *             fused RoPE kernel.
 *   [EFF]     "Efficient LLM Inference", "KV Caching: Verify Reuse, Positions
 *             and Windows" (chunked computation equals a full-prefix pass);
 *             "Quantization: From Rounding Errors to Model-quality Limits"
 *             (values rounded to a small set of levels with a scale) and
 *             "Verify Exact Execution and Approximate Quality Separately".
 *   [OFP8]    The E4M3 format itself is not on the pages; it is the public
 *             OCP 8-bit floating point format: 1 sign bit, 4 exponent bits
 *             (bias 7), 3 mantissa bits, no infinities, S.1111.111 = NaN,
 *             largest finite value 448, subnormals m * 2^-9.
 *
 * Readings where the pages are silent (all stated once here):
 *   - RoPE pairs element i with element i + d/2 ("rotate half", the Llama
 *     convention), frequency theta^(-2i/d), no frequency rescaling; q and k
 *     are rotated, v never is.  The rotated values are rounded once to the
 *     tensor's storage type (bf16: round to nearest, ties to even).
 *   - Cache layout [num_blocks][num_kv_heads][block_size][head_dim]; token t
 *     of a sequence lives in physical block block_tables[b][t / block_size]
 *     at row t % block_size.  A slot s names block s / block_size, row
 *     s % block_size.  A negative slot means "do not write this token".
 *   - Query head h reads kv head h / (Hq / Hkv) (contiguous groups).
 *   - A context of length 0 produces an all-zero output row.
 *   - Sliding window W > 0 ([EFF] "KV Caching: Verify Reuse, Positions and
 *     Windows"): the query at the last position of a context of L tokens
 *     attends to its last min(W, L) tokens, L - W .. L - 1 (itself
 *     included); W = 0 means no window.
 *   - 8-bit cache: one scale per tensor (k_scale, v_scale); the stored code
 *     of a value x is x / scale (fp64) rounded to binary32, then to the
 *     nearest E4M3 value, ties to even, saturating to +-448.  The binary32
 *     step is the precision the GPU takes that decision in.  V pages of this
 *     cache are stored transposed, [num_blocks][num_kv_heads][head_dim]
 *     [block_size]; K pages keep the [block_size][head_dim] row layout.
 *
 * Floating point: every input is converted exactly to double; all sums and
 * exponentials are in double.  Build with plain -O2 (no fast-math).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_F32 0
#define ORC_BF16 1
#define ORC_E4M3 2

#define ORC_OK 0
#define ORC_EARG (-1)
#define ORC_EBLOCK (-2)
#define ORC_ECTX (-3)
#define ORC_ESLOT (-4)
#define ORC_ENOMEM (-5)

/* ---- storage types ---------------------------------------------------- */

/* bf16 is the upper half of an IEEE binary32: widening is exact. */
static double bf16_to_double(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16 value (8 significant bits, binary32's
 * exponent range), ties to even, in ONE rounding step: the value is scaled
 * by the bf16 spacing at its binade (a power of two, so exact), rounded to
 * an integer with nearbyint (ties-to-even in the default rounding mode) and
 * scaled back.  Going through float first would round twice. */
static uint16_t double_to_bf16(double x) {
    if (isnan(x)) return (uint16_t)0x7FC0;
    uint16_t sign = signbit(x) ? (uint16_t)0x8000 : (uint16_t)0;
    double a = fabs(x);
    if (a == 0.0) return sign;
    if (isinf(a)) return (uint16_t)(sign | 0x7F80);
    int e;
    (void)frexp(a, &e);           /* a in [2^(e-1), 2^e) */
    int spacing_exp = (e - 1) - 7; /* 7 stored mantissa bits */
    if (spacing_exp < -133) spacing_exp = -133; /* subnormal spacing 2^-133 */
    double r = nearbyint(ldexp(a, -spacing_exp));
    r = ldexp(r, spacing_exp);
    if (r >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80); /* overflow */
    float f = (float)r; /* exact: r has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | (uint16_t)(u >> 16));
}

static double load_elem(const void* base, int dtype, int64_t i) {
    if (dtype == ORC_F32) return (double)((const float*)base)[i];
    return bf16_to_double(((const uint16_t*)base)[i]);
}

static void store_elem(void* base, int dtype, int64_t i, double v) {
    if (dtype == ORC_F32)
        ((float*)base)[i] = (float)v; /* C conversion: round to nearest even */
    else
        ((uint16_t*)base)[i] = double_to_bf16(v);
}

int orc_round_bf16(const double* x, uint16_t* out, int64_t n) {
    if (n < 0 || (n > 0 && (!x || !out))) return ORC_EARG;
    for (int64_t i = 0; i < n; ++i) out[i] = double_to_bf16(x[i]);
    return ORC_OK;
}

int orc_bf16_to_double(const uint16_t* x, double* out, int64_t n) {
    if (n < 0 || (n > 0 && (!x || !out))) return ORC_EARG;
    for (int64_t i = 0; i < n; ++i) out[i] = bf16_to_double(x[i]);
    return ORC_OK;
}

/* ---- E4M3 ([OFP8]; [EFF] quantization) ---------------------------------- */

/* The value a code stands for, straight from the format's definition. */
static double e4m3_to_double(uint8_t c) {
    int neg = c >> 7, E = (c >> 3) & 15, m = c & 7;
    double v;
    if (E == 15 && m == 7) return NAN;
    if (E == 0)
        v = ldexp((double)m, -9);           /* subnormal: m * 2^-9 */
    else
        v = ldexp(1.0 + m / 8.0, E - 7);   /* normal: 1.m * 2^(E-7) */
    return neg ? -v : v;
}

/* Nearest E4M3 value of x, ties to even, saturating: like double_to_bf16,
 * scale by the spacing of the representable values in x's binade (2^-9 for
 * everything below 2^-5, where subnormals and the first normal binade share
 * that spacing), round to an integer, scale back; anything that rounds
 * above 448 (the largest finite value) becomes 448.  NaN maps to S.1111.111. */
static uint8_t double_to_e4m3(double x) {
    if (isnan(x)) return (uint8_t)0x7F;
    uint8_t sign = signbit(x) ? (uint8_t)0x80 : (uint8_t)0;
    double a = fabs(x);
    double r = 448.0;
    if (!isinf(a)) {
        int e = 0;
        if (a > 0.0) (void)frexp(a, &e); /* a in [2^(e-1), 2^e) */
        int spacing_exp = (e - 1) - 3;   /* 3 stored mantissa bits */
        if (spacing_exp < -9) spacing_exp = -9;
        r = ldexp(nearbyint(ldexp(a, -spacing_exp)), spacing_exp);
        if (r > 448.0) r = 448.0;
    }
    if (r < ldexp(1.0, -6)) return (uint8_t)(sign | (uint8_t)ldexp(r, 9)); /* 0 .. 7 */
    int er;
    double f = frexp(r, &er);                 /* r = f * 2^er, f in [0.5, 1) */
    int E = er - 1 + 7;                       /* biased exponent, 1 .. 15 */
    int m = (int)((2.0 * f - 1.0) * 8.0);     /* exact: r has 4 significant bits */
    return (uint8_t)(sign | (uint8_t)(E << 3) | (uint8_t)m);
}

/* The stored code of x under `scale`: x / scale rounded to binary32, then to
 * E4M3 (the binary32 value is exact in double, so the second rounding is the
 * correctly rounded E4M3 value of that binary32 number). */
static uint8_t quantize_e4m3(double x, double scale) {
    return double_to_e4m3((double)(float)(x / scale));
}

int orc_e4m3_to_double(const uint8_t* c, double* out, int64_t n) {
    if (n < 0 || (n > 0 && (!c || !out))) return ORC_EARG;
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_to_double(c[i]);
    return ORC_OK;
}

int orc_round_e4m3(const double* x, uint8_t* out, int64_t n) {
    if (n < 0 || (n > 0 && (!x || !out))) return ORC_EARG;
    for (int64_t i = 0; i < n; ++i) out[i] = double_to_e4m3(x[i]);
    return ORC_OK;
}

/* ---- RoPE ([LIFS] Architecture overview; [WARP] Milestones) ------------- */

/* Rotate one head vector x[0..d) in place for integer position pos:
 * for i < d/2 the pair (x[i], x[i + d/2]) turns by the angle
 * pos * theta^(-2i/d). */
static void rope_rotate(double* x, int64_t d, int64_t pos, double theta) {
    int64_t half = d / 2;
    for (int64_t i = 0; i < half; ++i) {
        double freq = pow(theta, -(2.0 * (double)i) / (double)d);
        double angle = (double)pos * freq;
        double c = cos(angle), s = sin(angle);
        double x0 = x[i], x1 = x[i + half];
        x[i] = x0 * c - x1 * s;
        x[i + half] = x1 * c + x0 * s;
    }
}

/* x: [n][d] doubles, each row rotated for its own position. */
int orc_rope(double* x, int64_t n, int64_t d, const int64_t* positions, double theta) {
    if (n < 0 || d <= 0 || (d % 2) != 0 || (n > 0 && (!x || !positions))) return ORC_EARG;
    for (int64_t r = 0; r < n; ++r) rope_rotate(x + r * d, d, positions[r], theta);
    return ORC_OK;
}

/* ---- KV append ([WARP] static KV cache + single-token decode; [BOOK]
 *      ch. 10 block tables; [PROJ] M13c block pool) ----------------------
 *
 * For every token t:
 *   q[t, h, :]  <- round(rope(q[t, h, :], positions[t]))          (all h < Hq)
 *   if slot = slot_mapping[t] >= 0:
 *     k_cache[slot / bs, h, slot % bs, :] <- round(rope(k_new[t, h, :]))
 *     v_cache[slot / bs, h, slot % bs, :] <- v_new[t, h, :]        (h < Hkv)
 * q, k_new, v_new, k_cache and v_cache all have storage type `dtype`.
 * Every slot is validated before anything is written. */
/* q[t, h, :] <- round(rope(q[t, h, :], pos)) for every query head h. */
static void rotate_q_token(void* q, int dtype, int64_t t, int64_t Hq, int64_t d, int64_t pos,
                           double theta, double* row) {
    for (int64_t h = 0; h < Hq; ++h) {
        int64_t base = (t * Hq + h) * d;
        for (int64_t i = 0; i < d; ++i) row[i] = load_elem(q, dtype, base + i);
        rope_rotate(row, d, pos, theta);
        for (int64_t i = 0; i < d; ++i) store_elem(q, dtype, base + i, row[i]);
    }
}

int orc_kv_append(int dtype, void* q, const void* k_new, const void* v_new,
                  const int64_t* positions, const int64_t* slot_mapping,
                  void* k_cache, void* v_cache,
                  int64_t T, int64_t Hq, int64_t Hkv, int64_t d,
                  int64_t num_blocks, int64_t bs, double theta) {
    if (dtype != ORC_F32 && dtype != ORC_BF16) return ORC_EARG;
    if (T < 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || (d % 2) != 0 || num_blocks <= 0 || bs <= 0)
        return ORC_EARG;
    if (T == 0) return ORC_OK;
    if (!q || !k_new || !v_new || !positions || !slot_mapping || !k_cache || !v_cache)
        return ORC_EARG;
    for (int64_t t = 0; t < T; ++t)
        if (slot_mapping[t] >= num_blocks * bs) return ORC_ESLOT;

    double* row = (double*)malloc((size_t)d * sizeof(double));
    if (!row) return ORC_ENOMEM;
    for (int64_t t = 0; t < T; ++t) {
        int64_t pos = positions[t];
        rotate_q_token(q, dtype, t, Hq, d, pos, theta, row);
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        int64_t blk = slot / bs, off = slot % bs;
        for (int64_t h = 0; h < Hkv; ++h) {
            int64_t src = (t * Hkv + h) * d;
            int64_t dst = ((blk * Hkv + h) * bs + off) * d;
            for (int64_t i = 0; i < d; ++i) row[i] = load_elem(k_new, dtype, src + i);
            rope_rotate(row, d, pos, theta);
            for (int64_t i = 0; i < d; ++i) store_elem(k_cache, dtype, dst + i, row[i]);
            /* v is copied unchanged, so its bits must survive exactly */
            if (dtype == ORC_F32)
                memcpy((float*)v_cache + dst, (const float*)v_new + src, (size_t)d * 4);
            else
                memcpy((uint16_t*)v_cache + dst, (const uint16_t*)v_new + src, (size_t)d * 2);
        }
    }
    free(row);
    return ORC_OK;
}

/* The same append into an E4M3 cache ([EFF] quantization; [OFP8]):
 *   q[t, h, :] <- round(rope(q[t, h, :]))  in q's storage type `dtype`
 *   if slot >= 0, for h < Hkv and i < d:
 *     k_cache[blk, h, off, i] <- code(rope(k_new[t, h, :])[i] / k_scale)
 *     v_cache[blk, h, i, off] <- code(v_new[t, h, i] / v_scale)    (transposed)
 * where code() is quantize_e4m3 (binary32, then nearest E4M3, saturating). */
int orc_kv_append_e4m3(int dtype, void* q, const void* k_new, const void* v_new,
                       const int64_t* positions, const int64_t* slot_mapping,
                       uint8_t* k_cache, uint8_t* v_cache,
                       int64_t T, int64_t Hq, int64_t Hkv, int64_t d,
                       int64_t num_blocks, int64_t bs, double theta,
                       double k_scale, double v_scale) {
    if (dtype != ORC_F32 && dtype != ORC_BF16) return ORC_EARG;
    if (T < 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || (d % 2) != 0 || num_blocks <= 0 || bs <= 0)
        return ORC_EARG;
    if (!(k_scale > 0.0) || !(v_scale > 0.0) || isinf(k_scale) || isinf(v_scale)) return ORC_EARG;
    if (T == 0) return ORC_OK;
    if (!q || !k_new || !v_new || !positions || !slot_mapping || !k_cache || !v_cache)
        return ORC_EARG;
    for (int64_t t = 0; t < T; ++t)
        if (slot_mapping[t] >= num_blocks * bs) return ORC_ESLOT;

    double* row = (double*)malloc((size_t)d * sizeof(double));
    if (!row) return ORC_ENOMEM;
    for (int64_t t = 0; t < T; ++t) {
        int64_t pos = positions[t];
        rotate_q_token(q, dtype, t, Hq, d, pos, theta, row);
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        int64_t blk = slot / bs, r = slot % bs; /* block, row within the page */
        for (int64_t h = 0; h < Hkv; ++h) {
            int64_t src = (t * Hkv + h) * d;
            int64_t page = (blk * Hkv + h) * bs * d;
            for (int64_t i = 0; i < d; ++i) row[i] = load_elem(k_new, dtype, src + i);
            rope_rotate(row, d, pos, theta);
            for (int64_t i = 0; i < d; ++i) k_cache[page + r * d + i] = quantize_e4m3(row[i], k_scale);
            for (int64_t i = 0; i < d; ++i)
                v_cache[page + i * bs + r] = quantize_e4m3(load_elem(v_new, dtype, src + i), v_scale);
        }
    }
    free(row);
    return ORC_OK;
}

/* ---- paged decode ([BOOK] ch. 8 and ch. 10; [PROJ] M2, M13b) -----------
 *
 * For sequence b with L = context_lens[b] and query head h (kv head
 * kvh = h / (Hq / Hkv)), over the tokens t0 <= t < L where t0 = 0, or
 * max(0, L - window) with a sliding window:
 *   K[t] = k_cache[block_tables[b][t / bs], kvh, t % bs, :]
 *   s_t  = scale * sum_i q[b, h, i] * K[t][i]
 *   M    = max_t s_t ;   w_t = exp(s_t - M)
 *   out[b, h, :] = sum_t w_t V[t] / sum_t w_t          (zeros when L == 0)
 */
typedef struct {
    int q_dtype, kv_dtype;
    const void *q, *k_cache, *v_cache;
    const int32_t *block_tables, *context_lens;
    int64_t B, Hq, Hkv, d, num_blocks, bs, MB;
    double scale;
    double k_scale, v_scale; /* E4M3 cache only */
    int64_t window;          /* 0: none */
    const int64_t* pairs; /* optional list of (b, h) pairs */
    int64_t npairs;
    double* out;
    int nthreads, tid;
    int status;
} decode_job;

/* Element i of cached token `row` (block blk, kv head kvh).  K pages are
 * [bs][d]; V pages are [bs][d] too, except in the E4M3 cache ([d][bs]). */
static double k_elem(const decode_job* J, int64_t blk, int64_t kvh, int64_t row, int64_t i) {
    int64_t idx = ((blk * J->Hkv + kvh) * J->bs + row) * J->d + i;
    if (J->kv_dtype == ORC_E4M3)
        return e4m3_to_double(((const uint8_t*)J->k_cache)[idx]) * J->k_scale;
    return load_elem(J->k_cache, J->kv_dtype, idx);
}

static double v_elem(const decode_job* J, int64_t blk, int64_t kvh, int64_t row, int64_t i) {
    if (J->kv_dtype == ORC_E4M3) {
        int64_t idx = ((blk * J->Hkv + kvh) * J->d + i) * J->bs + row;
        return e4m3_to_double(((const uint8_t*)J->v_cache)[idx]) * J->v_scale;
    }
    return load_elem(J->v_cache, J->kv_dtype, ((blk * J->Hkv + kvh) * J->bs + row) * J->d + i);
}

static int decode_one(const decode_job* J, int64_t b, int64_t h, double* s) {
    const int64_t G = J->Hq / J->Hkv, d = J->d;
    const int64_t kvh = h / G;
    const int64_t L = J->context_lens[b];
    double* o = J->out + (b * J->Hq + h) * d;
    for (int64_t i = 0; i < d; ++i) o[i] = 0.0;
    if (L == 0) return ORC_OK;

    const int64_t qbase = (b * J->Hq + h) * d;
    const int64_t t0 = (J->window > 0 && L > J->window) ? L - J->window : 0;
    double M = -INFINITY;
    for (int64_t t = t0; t < L; ++t) {
        int64_t blk = J->block_tables[b * J->MB + t / J->bs];
        if (blk < 0 || blk >= J->num_blocks) return ORC_EBLOCK;
        double acc = 0.0;
        for (int64_t i = 0; i < d; ++i)
            acc += load_elem(J->q, J->q_dtype, qbase + i) * k_elem(J, blk, kvh, t % J->bs, i);
        s[t] = J->scale * acc;
        if (s[t] > M) M = s[t];
    }
    double den = 0.0;
    for (int64_t t = t0; t < L; ++t) {
        double w = exp(s[t] - M);
        den += w;
        int64_t blk = J->block_tables[b * J->MB + t / J->bs];
        for (int64_t i = 0; i < d; ++i) o[i] += w * v_elem(J, blk, kvh, t % J->bs, i);
    }
    for (int64_t i = 0; i < d; ++i) o[i] /= den;
    return ORC_OK;
}

static void* decode_worker(void* arg) {
    decode_job* J = (decode_job*)arg;
    int64_t maxL = J->MB * J->bs;
    double* s = (double*)malloc((size_t)(maxL > 0 ? maxL : 1) * sizeof(double));
    if (!s) { J->status = ORC_ENOMEM; return NULL; }
    int64_t total = J->pairs ? J->npairs : J->B * J->Hq;
    for (int64_t k = J->tid; k < total; k += J->nthreads) {
        int64_t b, h;
        if (J->pairs) { b = J->pairs[2 * k]; h = J->pairs[2 * k + 1]; }
        else { b = k / J->Hq; h = k % J->Hq; }
        int st = decode_one(J, b, h, s);
        if (st != ORC_OK) { J->status = st; break; }
    }
    free(s);
    return NULL;
}

static int run_decode(int q_dtype, int kv_dtype, const void* q,
                      const void* k_cache, const void* v_cache,
                      const int32_t* block_tables, const int32_t* context_lens,
                      int64_t B, int64_t Hq, int64_t Hkv, int64_t d,
                      int64_t num_blocks, int64_t bs, int64_t MB, double scale,
                      double k_scale, double v_scale, int64_t window,
                      const int64_t* pairs, int64_t npairs, int nthreads, double* out) {
    if (window < 0) return ORC_EARG;
    if (B < 0 || Hq <= 0 || Hkv <= 0 || (Hq % Hkv) != 0 || d <= 0 || bs <= 0 || MB < 0 ||
        num_blocks <= 0 || npairs < 0)
        return ORC_EARG;
    if (B == 0) return ORC_OK;
    if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out) return ORC_EARG;
    for (int64_t b = 0; b < B; ++b)
        if (context_lens[b] < 0 || (int64_t)context_lens[b] > MB * bs) return ORC_ECTX;
    if (pairs)
        for (int64_t k = 0; k < npairs; ++k)
            if (pairs[2 * k] < 0 || pairs[2 * k] >= B || pairs[2 * k + 1] < 0 || pairs[2 * k + 1] >= Hq)
                return ORC_EARG;
    if (nthreads < 1) nthreads = 1;

    decode_job* jobs = (decode_job*)calloc((size_t)nthreads, sizeof(decode_job));
    pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !th) { free(jobs); free(th); return ORC_ENOMEM; }
    for (int i = 0; i < nthreads; ++i) {
        decode_job J = {q_dtype, kv_dtype, q, k_cache, v_cache, block_tables, context_lens,
                        B, Hq, Hkv, d, num_blocks, bs, MB, scale, k_scale, v_scale, window,
                        pairs, npairs, out, nthreads, i, ORC_OK};
        jobs[i] = J;
    }
    for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, decode_worker, &jobs[i]);
    decode_worker(&jobs[0]);
    for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
    int st = ORC_OK;
    for (int i = 0; i < nthreads; ++i)
        if (jobs[i].status != ORC_OK) st = jobs[i].status;
    free(jobs);
    free(th);
    return st;
}

int orc_paged_decode(int q_dtype, int kv_dtype, const void* q,
                     const void* k_cache, const void* v_cache,
                     const int32_t* block_tables, const int32_t* context_lens,
                     int64_t B, int64_t Hq, int64_t Hkv, int64_t d,
                     int64_t num_blocks, int64_t bs, int64_t MB, double scale, int64_t window,
                     const int64_t* pairs, int64_t npairs, int nthreads, double* out) {
    if ((q_dtype != ORC_F32 && q_dtype != ORC_BF16) || (kv_dtype != ORC_F32 && kv_dtype != ORC_BF16))
        return ORC_EARG;
    return run_decode(q_dtype, kv_dtype, q, k_cache, v_cache, block_tables, context_lens, B, Hq,
                      Hkv, d, num_blocks, bs, MB, scale, 1.0, 1.0, window, pairs, npairs,
                      nthreads, out);
}

/* The decode over an E4M3 cache: the same definition with
 * K[t][i] = value(k code) * k_scale and V[t][i] = value(v code) * v_scale
 * (V pages transposed, see k_elem / v_elem). */
int orc_paged_decode_e4m3(int q_dtype, const void* q,
                          const uint8_t* k_cache, const uint8_t* v_cache,
                          const int32_t* block_tables, const int32_t* context_lens,
                          int64_t B, int64_t Hq, int64_t Hkv, int64_t d,
                          int64_t num_blocks, int64_t bs, int64_t MB, double scale,
                          double k_scale, double v_scale, int64_t window,
                          const int64_t* pairs, int64_t npairs, int nthreads, double* out) {
    if (q_dtype != ORC_F32 && q_dtype != ORC_BF16) return ORC_EARG;
    if (!(k_scale > 0.0) || !(v_scale > 0.0) || isinf(k_scale) || isinf(v_scale)) return ORC_EARG;
    return run_decode(q_dtype, ORC_E4M3, q, k_cache, v_cache, block_tables, context_lens, B, Hq,
                      Hkv, d, num_blocks, bs, MB, scale, k_scale, v_scale, window, pairs, npairs,
                      nthreads, out);
}

/* ---- self-check variants (same definition, no paging) ------------------ */

/* Attention of q [Hq][d] over a contiguous K, V [L][Hkv][d]; out [Hq][d].
 * ([BOOK] ch. 4 KV cache: the unpaged cache the paged one must reproduce.) */
int orc_contiguous_decode(const double* q, const double* K, const double* V,
                          int64_t L, int64_t Hq, int64_t Hkv, int64_t d, double scale,
                          double* out) {
    if (L < 0 || Hq <= 0 || Hkv <= 0 || (Hq % Hkv) != 0 || d <= 0) return ORC_EARG;
    if (!q || !out || (L > 0 && (!K || !V))) return ORC_EARG;
    const int64_t G = Hq / Hkv;
    double* s = (double*)malloc((size_t)(L > 0 ? L : 1) * sizeof(double));
    if (!s) return ORC_ENOMEM;
    for (int64_t h = 0; h < Hq; ++h) {
        const int64_t kvh = h / G;
        double* o = out + h * d;
        for (int64_t i = 0; i < d; ++i) o[i] = 0.0;
        if (L == 0) continue;
        double M = -INFINITY;
        for (int64_t t = 0; t < L; ++t) {
            double acc = 0.0;
            for (int64_t i = 0; i < d; ++i) acc += q[h * d + i] * K[(t * Hkv + kvh) * d + i];
            s[t] = scale * acc;
            if (s[t] > M) M = s[t];
        }
        double den = 0.0;
        for (int64_t t = 0; t < L; ++t) {
            double w = exp(s[t] - M);
            den += w;
            for (int64_t i = 0; i < d; ++i) o[i] += w * V[(t * Hkv + kvh) * d + i];
        }
        for (int64_t i = 0; i < d; ++i) o[i] /= den;
    }
    free(s);
    return ORC_OK;
}

/* Full-prefix causal attention: query row r attends to tokens 0..r.
 * Q [L][Hq][d], K, V [L][Hkv][d], out [L][Hq][d].  Its last row is what one
 * decode step over the cached prefix must return ([LIFS] M1 prefill/decode
 * equivalence; [EFF] chunked equals full-prefix). */
int orc_causal_prefill(const double* Q, const double* K, const double* V,
                       int64_t L, int64_t Hq, int64_t Hkv, int64_t d, double scale,
                       double* out) {
    if (L < 0 || Hq <= 0 || Hkv <= 0 || (Hq % Hkv) != 0 || d <= 0) return ORC_EARG;
    if (L == 0) return ORC_OK;
    if (!Q || !K || !V || !out) return ORC_EARG;
    const int64_t G = Hq / Hkv;
    double* s = (double*)malloc((size_t)L * sizeof(double));
    if (!s) return ORC_ENOMEM;
    for (int64_t r = 0; r < L; ++r) {
        for (int64_t h = 0; h < Hq; ++h) {
            const int64_t kvh = h / G;
            double* o = out + (r * Hq + h) * d;
            double M = -INFINITY;
            for (int64_t t = 0; t <= r; ++t) {
                double acc = 0.0;
                for (int64_t i = 0; i < d; ++i)
                    acc += Q[(r * Hq + h) * d + i] * K[(t * Hkv + kvh) * d + i];
                s[t] = scale * acc;
                if (s[t] > M) M = s[t];
            }
            for (int64_t i = 0; i < d; ++i) o[i] = 0.0;
            double den = 0.0;
            for (int64_t t = 0; t <= r; ++t) {
                double w = exp(s[t] - M);
                den += w;
                for (int64_t i = 0; i < d; ++i) o[i] += w * V[(t * Hkv + kvh) * d + i];
            }
            for (int64_t i = 0; i < d; ++i) o[i] /= den;
        }
    }
    free(s);
    return ORC_OK;
}
