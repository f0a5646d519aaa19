/*
 * oracle.c -- plain, slow, obviously correct CPU definition of the DSA / SWA
 * decode layer-step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link,
 * load or execute this file: only the test-suite, the smoke check and the CPU
 * baseline leg of the benchmark do.  It shares no code, header, table or
 * constant with the CUDA library.
 *
 * Sources (page title, then section):
 *   [EXPL]  "Naive-N0.5-Flash: no full-attention layers, and a runtime built
 *           by AI" (ai.thesatyajit.com explainer)
 *             - property table (index heads 16, fp8_e4m3 indexer, top 2,048,
 *               window 128, 64 Q heads, head dim 192, v dim 128, GQA4 / GQA8)
 *             - "What 'no full-attention layers' means" (SWA mask
 *               query_offset - key_offset < window; DSA argsort top-k)
 *             - "Inside a DSA layer: the lightning indexer" (relu(q k^T) per
 *               index head, combined by a learned per-head weight; sink column)
 *             - "How much of this did AI actually build?" (stable-tie argsort)
 *
 * Every floating-point quantity is computed in double; the indexer dot
 * product of two e4m3 vectors is exact in double (each product has at most 8
 * significant bits and a 128-term sum spans fewer than 53 bits), and the
 * score is rounded to float once, last.
 *
 * Pins (tests/test_oracle_pins.py): e4m3 and bf16 decoding against torch's
 * own conversions; the exact dot against rational arithmetic; a hand-worked
 * indexer example (tests/golden); the ReLU-free special case against a numpy
 * matrix-vector product; power-of-two scale folding; top-k against Python's
 * sorted() and against a second, selection-based implementation; attention
 * against torch scaled_dot_product_attention (no sink), the closed-form sink
 * identity, the single-key closed form, GQA == MHA with repeated heads, and
 * dense / full-window equivalences.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Threads: the loops over key positions (indexer) and over heads (attention)
 * may run on several host threads.  Every output element is computed by one
 * thread with the same loop order as on one thread, so the results do not
 * depend on the thread count. */
void oracle_set_threads(int n) {
#ifdef _OPENMP
    omp_set_num_threads(n > 0 ? n : 1);
#else
    (void)n;
#endif
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---------------------------------------------------------------- formats */

/* OCP FP8 E4M3 ("e4m3fn"): 1 sign bit, 4 exponent bits (bias 7), 3 mantissa
 * bits; exponent field 0 is subnormal; no infinities; S.1111.111 is NaN;
 * largest finite magnitude 1.75 * 2^8 = 448.  [EXPL, property table:
 * the indexer runs in fp8_e4m3] */
double oracle_e4m3_to_double(uint8_t b) {
    int sign = (b >> 7) & 1;
    int e = (b >> 3) & 0xF;
    int m = b & 0x7;
    double mag;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        mag = ldexp((double)m, -9);            /* (m / 8) * 2^(1 - 7) */
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* bfloat16 is the upper half of an IEEE-754 binary32 word. */
double oracle_bf16_to_double(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ----------------------------------------------------------- indexer (a1) */

/* Exact e4m3 dot product of two length-d code vectors. */
double oracle_fp8_dot(const uint8_t *a, const uint8_t *b, int d) {
    double acc = 0.0;
    for (int i = 0; i < d; ++i)
        acc += oracle_e4m3_to_double(a[i]) * oracle_e4m3_to_double(b[i]);
    return acc;
}

/* Lightning-indexer scores for one sequence.
 *   I[t][s] = sum_h w[t][h] * max(0, qs[t][h] * ks[s] * <q8[t][h], k8[s]>)
 * for s <= q_pos[t]; entries s > q_pos[t] (not visible to query t) are set to
 * -infinity.  [EXPL, "Inside a DSA layer": relu(q @ k^T) per index head,
 * combined across heads by a learned weight into one score per key]
 *
 * q8      [T][H][D] e4m3 codes      q_scale [T][H]     w [T][H]
 * k8      [L][D]    e4m3 codes      k_scale [L]
 * q_pos   [T]                        scores  [T][L] (float, written)
 */
void oracle_indexer_scores(const uint8_t *q8, const float *q_scale,
                           const float *w, const uint8_t *k8,
                           const float *k_scale, const int32_t *q_pos,
                           int T, int H, int D, int64_t L, float *scores) {
    for (int t = 0; t < T; ++t) {
#pragma omp parallel for schedule(static)
        for (int64_t s = 0; s < L; ++s) {
            if (s > q_pos[t]) {
                scores[(int64_t)t * L + s] = -INFINITY;
                continue;
            }
            double sum = 0.0;
            for (int h = 0; h < H; ++h) {
                double dot = oracle_fp8_dot(q8 + ((int64_t)t * H + h) * D,
                                            k8 + s * D, D);
                double x = (double)q_scale[t * H + h] * (double)k_scale[s] * dot;
                if (x < 0.0) x = 0.0;
                sum += (double)w[t * H + h] * x;
            }
            scores[(int64_t)t * L + s] = (float)sum;
        }
    }
}

/* ------------------------------------------------------------- top-k (a2) */

/* Order used by the selection: larger score first; equal scores are broken
 * toward the lower position (the stable-tie argsort of [EXPL, "What 'no
 * full-attention layers' means" and "How much of this did AI actually
 * build?"]).  -0.0 and +0.0 compare equal because the comparison is on the
 * float values. */
typedef struct { float v; int32_t pos; } oracle_item;

static int oracle_item_cmp(const void *pa, const void *pb) {
    const oracle_item *a = (const oracle_item *)pa, *b = (const oracle_item *)pb;
    if (a->v > b->v) return -1;
    if (a->v < b->v) return 1;
    return (a->pos < b->pos) ? -1 : (a->pos > b->pos);
}

/* Full stable sort of the n visible scores; writes the first min(k, n)
 * positions (in sort order) to idx[0..k), pads the rest with -1 and returns
 * the count.  Scores must not be NaN. */
int oracle_topk(const float *scores, int64_t n, int k, int32_t *idx) {
    oracle_item *it = (oracle_item *)malloc(sizeof(oracle_item) * (size_t)(n > 0 ? n : 1));
    for (int64_t i = 0; i < n; ++i) { it[i].v = scores[i]; it[i].pos = (int32_t)i; }
    qsort(it, (size_t)n, sizeof(oracle_item), oracle_item_cmp);
    int cnt = (int)(n < k ? n : k);
    for (int i = 0; i < k; ++i) idx[i] = i < cnt ? it[i].pos : -1;
    free(it);
    return cnt;
}

/* Second, independent top-k used only to cross-check oracle_topk: find the
 * k-th largest value by quickselect on a copy of the values, then take every
 * position whose value is larger and the lowest-positioned ties, in position
 * order. */
static float oracle_kth_largest(float *a, int64_t n, int64_t k) {
    int64_t lo = 0, hi = n - 1, want = k - 1;   /* index in descending order */
    while (lo < hi) {
        float piv = a[lo + (hi - lo) / 2];
        int64_t i = lo, j = hi;
        while (i <= j) {
            while (a[i] > piv) ++i;
            while (a[j] < piv) --j;
            if (i <= j) { float t = a[i]; a[i] = a[j]; a[j] = t; ++i; --j; }
        }
        if (want <= j) hi = j;
        else if (want >= i) lo = i;
        else return a[want];
    }
    return a[want];
}

int oracle_topk_select(const float *scores, int64_t n, int k, int32_t *idx) {
    int cnt = (int)(n < k ? n : k);
    if (cnt == 0) { for (int i = 0; i < k; ++i) idx[i] = -1; return 0; }
    float *tmp = (float *)malloc(sizeof(float) * (size_t)n);
    memcpy(tmp, scores, sizeof(float) * (size_t)n);
    float thr = oracle_kth_largest(tmp, n, cnt);
    free(tmp);
    int64_t above = 0;
    for (int64_t i = 0; i < n; ++i) above += scores[i] > thr;
    int64_t ties = cnt - above, o = 0;
    for (int64_t i = 0; i < n; ++i) {
        if (scores[i] > thr) idx[o++] = (int32_t)i;
        else if (scores[i] == thr && ties > 0) { idx[o++] = (int32_t)i; --ties; }
    }
    for (int i = cnt; i < k; ++i) idx[i] = -1;
    return cnt;
}

/* --------------------------------------------------- attention (a3 / a5) */

/* Softmax attention of one query token over a set of key positions, grouped
 * query attention with contiguous head groups (head h reads KV head
 * h / (H / G)), and an optional per-head sink logit that enters the softmax
 * denominator only (it carries no value row).  [EXPL, property table: 64 Q
 * heads, head dim 192, v dim 128, GQA4 / GQA8; "Inside a DSA layer": the
 * sink column]
 *
 *   s_i  = sm_scale * sum_d Q[h][d] * K[idx_i][h/(H/G)][d]
 *   m    = max(max_i s_i, sink_h)
 *   o[h] = sum_i e^(s_i - m) V[idx_i][.] / (sum_i e^(s_i - m) + e^(sink_h - m))
 *   lse[h] = m + log(sum_i e^(s_i - m) + e^(sink_h - m))
 *
 * Q [H][Dk] bf16 bits; K [L][G][Dk], V [L][G][Dv] bf16 bits; idx [n];
 * sink [H] or NULL (no sink); out [H][Dv]; lse [H] or NULL.
 * An empty set with no sink gives o = 0 and lse = -inf.
 */
void oracle_gqa_attention(const uint16_t *Q, const uint16_t *K,
                          const uint16_t *V, int64_t L, int H, int G, int Dk,
                          int Dv, const int32_t *idx, int n, const float *sink,
                          double sm_scale, double *out, double *lse) {
    (void)L;
    int hpg = H / G;
#pragma omp parallel for schedule(static)
    for (int h = 0; h < H; ++h) {
        double *s = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
        int g = h / hpg;
        double m = -INFINITY;
        for (int i = 0; i < n; ++i) {
            const uint16_t *kr = K + ((int64_t)idx[i] * G + g) * Dk;
            double dot = 0.0;
            for (int d = 0; d < Dk; ++d)
                dot += oracle_bf16_to_double(Q[(int64_t)h * Dk + d]) *
                       oracle_bf16_to_double(kr[d]);
            s[i] = sm_scale * dot;
            if (s[i] > m) m = s[i];
        }
        double sk = sink ? (double)sink[h] : -INFINITY;
        if (sk > m) m = sk;
        double den = 0.0;
        for (int d = 0; d < Dv; ++d) out[(int64_t)h * Dv + d] = 0.0;
        if (m == -INFINITY) {               /* nothing to attend to */
            if (lse) lse[h] = -INFINITY;
            free(s);
            continue;
        }
        for (int i = 0; i < n; ++i) {
            double p = exp(s[i] - m);
            den += p;
            const uint16_t *vr = V + ((int64_t)idx[i] * G + g) * Dv;
            for (int d = 0; d < Dv; ++d)
                out[(int64_t)h * Dv + d] += p * oracle_bf16_to_double(vr[d]);
        }
        if (sink) den += exp(sk - m);
        for (int d = 0; d < Dv; ++d) out[(int64_t)h * Dv + d] /= den;
        if (lse) lse[h] = m + log(den);
        free(s);
    }
}

/* Sliding-window index set of the query at 0-based position p: the keys with
 * p - key < window, i.e. {max(0, p - window + 1), ..., p}.  [EXPL, "What 'no
 * full-attention layers' means": the SWA path masks every key with
 * query_offset - key_offset >= sliding_window]  Returns the count. */
int oracle_swa_indices(int64_t p, int window, int32_t *idx) {
    int64_t lo = p - window + 1;
    if (lo < 0) lo = 0;
    int n = 0;
    for (int64_t j = lo; j <= p; ++j) idx[n++] = (int32_t)j;
    return n;
}

/* ------------------------------------------- index-K / index-Q producer (f1) */

/* The indexer's key path before the cache: "normalises the key, applies RoPE,
 * rounds both to fp8_e4m3" [EXPL, "Inside a DSA layer: the lightning
 * indexer"; its figure: LayerNorm, partial RoPE, FP8 quantization], with the
 * partial rotary layout of the inherited attention block ("partial RoPE on a
 * third of each head", a rope base of 10,000,000 on the sparse layers [EXPL,
 * same section]).  The readings this follows where the page is silent:
 *   - LayerNorm over the 128 dims with a learned weight and bias;
 *   - RoPE on the first `rot` dims in the rotate-half arrangement: dim i and
 *     dim i + rot/2 (i < rot/2) form a pair turned by the angle
 *     pos * base^(-2i / rot); the other dims pass unchanged;
 *   - e4m3 per token: scale = amax / 448 (1 for an all-zero token), value /
 *     scale rounded to the nearest e4m3 value, ties to the even code,
 *     saturating at +-448.
 * Real arithmetic in double.  The quantisation decision is taken in fp32, as
 * the kernel takes it: the rotated value is rounded to float, the scale is
 * float(amax) / 448 in float, and the code is chosen for float(v / scale). */

/* LayerNorm of x[0..D): (x - mean) / sqrt(var + eps) * w + b, var the
 * population variance. */
void oracle_layernorm(const double *x, int D, const float *w, const float *b, double eps, double *y) {
    double mean = 0.0;
    for (int i = 0; i < D; ++i) mean += x[i];
    mean /= D;
    double var = 0.0;
    for (int i = 0; i < D; ++i) var += (x[i] - mean) * (x[i] - mean);
    var /= D;
    double inv = 1.0 / sqrt(var + eps);
    for (int i = 0; i < D; ++i) y[i] = (x[i] - mean) * inv * (double)w[i] + (double)b[i];
}

/* Partial rotary embedding of x[0..D) at position pos, in place. */
void oracle_rope_partial(double *x, int D, int rot, int64_t pos, double base) {
    (void)D;
    int h = rot / 2;
    for (int i = 0; i < h; ++i) {
        double inv_freq = pow(base, -2.0 * (double)i / (double)rot);
        double ang = (double)pos * inv_freq;
        double c = cos(ang), s = sin(ang);
        double a = x[i], b = x[i + h];
        x[i] = a * c - b * s;
        x[i + h] = b * c + a * s;
    }
}

/* The e4m3 code nearest to v (ties to the even code), saturating at +-448;
 * the sign of v (also of a zero) is kept.  From the format definition: the
 * candidates are the 127 non-negative finite codes 0x00..0x7E. */
uint8_t oracle_e4m3_encode(float v) {
    int neg = signbit(v) ? 1 : 0;
    double a = fabs((double)v);
    if (a >= 448.0) return (uint8_t)(0x7E | (neg << 7));
    int best = 0;
    double bestd = INFINITY;
    for (int c = 0; c <= 0x7E; ++c) {
        double d = fabs(oracle_e4m3_to_double((uint8_t)c) - a);
        if (d < bestd || (d == bestd && (c & 1) == 0)) {
            bestd = d;
            best = c;
        }
    }
    return (uint8_t)(best | (neg << 7));
}

/* Per-token quantisation of n real values (rounded to float first). */
static float oracle_quantize_token(const double *y, int n, uint8_t *codes) {
    float amax = 0.0f;
    for (int i = 0; i < n; ++i) {
        float f = fabsf((float)y[i]);
        if (f > amax) amax = f;
    }
    float scale = amax > 0.0f ? amax / 448.0f : 1.0f;
    for (int i = 0; i < n; ++i) codes[i] = oracle_e4m3_encode((float)y[i] / scale);
    return scale;
}

/* One token's index key: bf16 k[D] -> LayerNorm -> partial RoPE at pos ->
 * e4m3 codes[D] and the token's scale.  y_out (optional) gets the real
 * values before quantisation. */
float oracle_index_k_produce(const uint16_t *k, const float *ln_w, const float *ln_b, double eps, int D, int rot,
                             double base, int64_t pos, uint8_t *codes, double *y_out) {
    double x[512], y[512];
    for (int i = 0; i < D; ++i) x[i] = oracle_bf16_to_double(k[i]);
    oracle_layernorm(x, D, ln_w, ln_b, eps, y);
    oracle_rope_partial(y, D, rot, pos, base);
    if (y_out)
        for (int i = 0; i < D; ++i) y_out[i] = y[i];
    return oracle_quantize_token(y, D, codes);
}

/* One token's index query: bf16 q[H][D] -> partial RoPE at pos on every head
 * -> e4m3 codes[H][D] with one scale for the whole token (returned). */
float oracle_index_q_produce(const uint16_t *q, int H, int D, int rot, double base, int64_t pos, uint8_t *codes,
                             double *y_out) {
    double *y = (double *)malloc(sizeof(double) * (size_t)H * D);
    for (int h = 0; h < H; ++h) {
        for (int i = 0; i < D; ++i) y[h * D + i] = oracle_bf16_to_double(q[h * D + i]);
        oracle_rope_partial(y + h * D, D, rot, pos, base);
    }
    if (y_out)
        for (int i = 0; i < H * D; ++i) y_out[i] = y[i];
    float s = oracle_quantize_token(y, H * D, codes);
    free(y);
    return s;
}

/* --------------------------------------- indexer warm-up KL target (f4) */

/* The indexer warm-up trains only the indexer, "aligned to a full-attention
 * reference by a KL objective" [EXPL, "Inside a DSA layer: the lightning
 * indexer"; BLOG, "What's genuinely new": the layers being converted keep
 * full attention and supervise the indexer through a KL-divergence loss].
 * Reading (the pages give no formula): for a query token at position p,
 * over its visible keys s = 0..p,
 *   target  P[s] = (1/H) sum_h softmax_s(sm_scale * Q[h] . K[s][h / (H/G)])
 *           (each head's dense attention distribution over the keys, no
 *           sink, averaged over the H heads),
 *   indexer R[s] = softmax_s(I[s]) of the indexer scores,
 *   loss    KL(P || R) = sum_s P[s] (log P[s] - log R[s]).
 * Q [H][Dk] bf16; K [L][G][Dk] bf16 (rows 0..p are the visible keys);
 * I [p + 1] indexer scores.  Writes P[0..p] and returns the KL. */
double oracle_indexer_kl(const uint16_t *Q, const uint16_t *K, int H, int G, int Dk, const float *I, int64_t p,
                         double sm_scale, double *P) {
    int64_t n = p + 1;
    int hpg = H / G;
    double *s = (double *)malloc(sizeof(double) * (size_t)n);
    for (int64_t j = 0; j < n; ++j) P[j] = 0.0;
    for (int h = 0; h < H; ++h) {
        int g = h / hpg;
        double m = -INFINITY;
        for (int64_t j = 0; j < n; ++j) {
            const uint16_t *kr = K + (j * G + g) * Dk;
            double dot = 0.0;
            for (int d = 0; d < Dk; ++d)
                dot += oracle_bf16_to_double(Q[(int64_t)h * Dk + d]) * oracle_bf16_to_double(kr[d]);
            s[j] = sm_scale * dot;
            if (s[j] > m) m = s[j];
        }
        double den = 0.0;
        for (int64_t j = 0; j < n; ++j) den += exp(s[j] - m);
        for (int64_t j = 0; j < n; ++j) P[j] += exp(s[j] - m) / den / H;
    }
    free(s);
    double mi = -INFINITY;
    for (int64_t j = 0; j < n; ++j)
        if ((double)I[j] > mi) mi = (double)I[j];
    double li = 0.0;
    for (int64_t j = 0; j < n; ++j) li += exp((double)I[j] - mi);
    double lse_i = mi + log(li);
    double kl = 0.0;
    for (int64_t j = 0; j < n; ++j)
        if (P[j] > 0.0) kl += P[j] * (log(P[j]) - ((double)I[j] - lse_i));
    return kl;
}
