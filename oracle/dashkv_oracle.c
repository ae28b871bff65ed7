/*
 * dashkv_oracle.c -- plain, slow CPU statement of the decode-step
 * hash-score -> top-k select -> exact sparse attention path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file.  Only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or constant with the
 * CUDA library: the hyperplane generator below is written from the published
 * definition of splitmix64 (Steele, Lea & Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014), not taken from the GPU side.
 *
 * The method, as the pages describe it:
 *   - keys are stored as compact codes and queries stay in full precision
 *     (DASH-KV page, sections "DASH-KV的核心创新：非对称深度哈希" and
 *     "技术架构：动态混合精度机制");
 *   - the codes are locality-sensitive hashes, a light scorer ranks every
 *     cached key and only the Top-K survive
 *     (DASH-KV page, section "从平方到线性：复杂度降低的数学原理");
 *   - scores are taken directly from the compact key codes, never from a
 *     reconstructed dense key (Spherical KV page, section 2.1 ADA,
 *     "no reconstruction invariant");
 *   - an indexer scores the history, real attention runs on the top-k only,
 *     and a sliding window keeps recent tokens exact (DeepSeek DSA->CSA/HCA
 *     page, section "从 DSA 说起" and the SWA paragraph of the CSA section);
 *   - the first tokens (attention sinks) are kept as well (DySCO page, Q3 on
 *     StreamingLLM).
 *
 * Exact definitions used here (each step is written out directly):
 *   R[j][i] in {+1,-1}, j < bits, i < d  (seeded Rademacher hyperplanes)
 *   encode:  bit_j(k) = [ sum_i R[j][i] * k[i] >= 0 ]     (tie at 0 gives 1)
 *            bit j lives in 64-bit word j/64 at position j%64.
 *   score:   qp_{h,j} = sum_i R[j][i] * q_h[i]            (full precision)
 *            s_t = sum_{h in group} sum_j qp_{h,j} * (2*bit_j(k_t) - 1)
 *            query head h belongs to KV head h / G, G = Hq / Hkv.
 *   select:  top-k of s over all N cached tokens, order (s desc, t asc),
 *            united with sinks [0, S) and window [N-W, N); output ascending.
 *   attend:  out_h = sum_{t in sel} softmax_t(q_h . K_t / sqrt(d)) V_t,
 *            lse_h = log sum_{t in sel} exp(q_h . K_t / sqrt(d)).
 *
 * Arithmetic: everything in double.  Inputs are passed as double arrays
 * (bf16 values widen exactly).  For inputs on the 1/64 grid with magnitude
 * <= 4, every encode and score sum is an exact multiple of 1/64 far inside
 * double's exact range, so those results are exact.
 *
 * KV layouts (shared convention with the library's public header, restated):
 *   dense : K/V  [B][Hkv][n_cap][d],        codes [B][Hkv][n_cap][W64]
 *   paged : K/V  [P][page][Hkv][d],         codes [P][Hkv][page][W64]
 *           logical token t of sequence b lives in physical page
 *           page_table[b*max_pages + t/page], slot t%page.
 *   page == 0 selects the dense layout.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- threads */

void dko_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int dko_get_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* -------------------------------------------------------------- splitmix64 */

/* The n-th output (n >= 1) of a splitmix64 stream started at `seed`:
 * the state advances by the golden-ratio increment, then the mix function
 * (two xor-shift-multiply rounds and a final xor-shift) is applied. */
uint64_t dko_splitmix64_nth(uint64_t seed, uint64_t n) {
    uint64_t z = seed + n * 0x9E3779B97F4A7C15ULL;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* Rademacher hyperplanes: R[j][i] = -1 when the top bit of output number
 * (j*d + i + 1) of the stream is set, +1 otherwise. */
void dko_hyperplanes(uint64_t seed, int bits, int d, int8_t *R) {
    for (int j = 0; j < bits; ++j)
        for (int i = 0; i < d; ++i) {
            uint64_t z = dko_splitmix64_nth(seed, (uint64_t)j * (uint64_t)d + (uint64_t)i + 1u);
            R[(size_t)j * d + i] = (z >> 63) ? (int8_t)-1 : (int8_t)1;
        }
}

/* ---------------------------------------------------------------- layouts */

typedef struct {
    int B, Hkv, d, bits;
    int64_t n_cap;            /* dense capacity per sequence */
    const int32_t *page_table;/* paged: [B][max_pages]; NULL for dense */
    int max_pages;
    int page;                 /* tokens per page; 0 = dense */
} dko_layout;

static int64_t row_index(const dko_layout *L, int b, int h, int64_t t) {
    if (L->page == 0)
        return (((int64_t)b * L->Hkv + h) * L->n_cap + t) * L->d;
    int64_t p = L->page_table[(int64_t)b * L->max_pages + t / L->page];
    return ((p * L->page + t % L->page) * L->Hkv + h) * (int64_t)L->d;
}

static int64_t code_index(const dko_layout *L, int b, int h, int64_t t) {
    int w64 = L->bits / 64 > 0 ? L->bits / 64 : 1;
    if (L->page == 0)
        return (((int64_t)b * L->Hkv + h) * L->n_cap + t) * w64;
    int64_t p = L->page_table[(int64_t)b * L->max_pages + t / L->page];
    return ((p * L->Hkv + h) * L->page + t % L->page) * (int64_t)w64;
}

static dko_layout make_layout(int B, int Hkv, int d, int bits, int64_t n_cap,
                              const int32_t *page_table, int max_pages, int page) {
    dko_layout L;
    L.B = B; L.Hkv = Hkv; L.d = d; L.bits = bits; L.n_cap = n_cap;
    L.page_table = page_table; L.max_pages = max_pages; L.page = page;
    return L;
}

/* ----------------------------------------------------------------- encode */

/* Sign bits of one key against all hyperplanes, packed LSB-first into
 * ceil(bits/64) words (bits is a multiple of 32; a 32-bit code uses the low
 * half of one word). */
static void encode_one(const double *k, const int8_t *R, int bits, int d, uint64_t *code) {
    int w64 = bits / 64 > 0 ? bits / 64 : 1;
    for (int w = 0; w < w64; ++w) code[w] = 0;
    for (int j = 0; j < bits; ++j) {
        double dot = 0.0;
        for (int i = 0; i < d; ++i) dot += (double)R[(size_t)j * d + i] * k[i];
        if (dot >= 0.0) code[j / 64] |= (uint64_t)1 << (j % 64);
    }
}

/* Codes of tokens [0, seq_lens[b]) for every (b, kv head). */
void dko_encode(int B, int Hkv, int d, int bits, int64_t n_cap,
                const int32_t *page_table, int max_pages, int page,
                const double *K, const int32_t *seq_lens, const int8_t *R,
                uint64_t *codes) {
    dko_layout L = make_layout(B, Hkv, d, bits, n_cap, page_table, max_pages, page);
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hkv; ++h) {
            int64_t n = seq_lens[b];
#pragma omp parallel for schedule(static)
            for (int64_t t = 0; t < n; ++t)
                encode_one(K + row_index(&L, b, h, t), R, bits, d, codes + code_index(&L, b, h, t));
        }
}

/* One decode step's append: the new key/value of every (b, kv head) goes to
 * position seq_lens[b]; its code is written there; seq_lens[b] grows by 1.
 * k_new, v_new: [B][Hkv][d]. */
void dko_append(int B, int Hkv, int d, int bits, int64_t n_cap,
                const int32_t *page_table, int max_pages, int page,
                double *K, double *V, uint64_t *codes, int32_t *seq_lens,
                const double *k_new, const double *v_new, const int8_t *R) {
    dko_layout L = make_layout(B, Hkv, d, bits, n_cap, page_table, max_pages, page);
    for (int b = 0; b < B; ++b) {
        int64_t t = seq_lens[b];
        for (int h = 0; h < Hkv; ++h) {
            int64_t r = row_index(&L, b, h, t);
            const double *kn = k_new + ((int64_t)b * Hkv + h) * d;
            const double *vn = v_new + ((int64_t)b * Hkv + h) * d;
            for (int i = 0; i < d; ++i) { K[r + i] = kn[i]; V[r + i] = vn[i]; }
            encode_one(K + r, R, bits, d, codes + code_index(&L, b, h, t));
        }
        seq_lens[b] = (int32_t)(t + 1);
    }
}

/* ------------------------------------------------------------------ score */

/* s[b][kvh][t] for t < seq_lens[b], written into scores[B][Hkv][n_cap];
 * entries at t >= seq_lens[b] are left untouched.  Returns the largest
 * sum_j |sum_{h in group} qp_{h,j}| seen, a bound on every |s|. */
double dko_scores(int B, int Hq, int Hkv, int d, int bits, int64_t n_cap,
                  const int32_t *page_table, int max_pages, int page,
                  const double *q, const uint64_t *codes, const int32_t *seq_lens,
                  const int8_t *R, double *scores) {
    dko_layout L = make_layout(B, Hkv, d, bits, n_cap, page_table, max_pages, page);
    int G = Hq / Hkv;
    double bound = 0.0;
    double *qp = (double *)malloc(sizeof(double) * (size_t)G * bits);
    for (int b = 0; b < B; ++b)
        for (int kvh = 0; kvh < Hkv; ++kvh) {
            /* full-precision projection of each query head of the group */
            for (int g = 0; g < G; ++g) {
                const double *qh = q + ((int64_t)b * Hq + (int64_t)kvh * G + g) * d;
                for (int j = 0; j < bits; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < d; ++i) acc += (double)R[(size_t)j * d + i] * qh[i];
                    qp[(size_t)g * bits + j] = acc;
                }
            }
            double bsum = 0.0;
            for (int j = 0; j < bits; ++j) {
                double c = 0.0;
                for (int g = 0; g < G; ++g) c += qp[(size_t)g * bits + j];
                bsum += fabs(c);
            }
            if (bsum > bound) bound = bsum;
            int64_t n = seq_lens[b];
#pragma omp parallel for schedule(static)
            for (int64_t t = 0; t < n; ++t) {
                const uint64_t *code = codes + code_index(&L, b, kvh, t);
                double s = 0.0;
                for (int g = 0; g < G; ++g)
                    for (int j = 0; j < bits; ++j) {
                        int bit = (int)((code[j / 64] >> (j % 64)) & 1u);
                        s += qp[(size_t)g * bits + j] * (double)(2 * bit - 1);
                    }
                scores[((int64_t)b * Hkv + kvh) * n_cap + t] = s + 0.0; /* no -0 */
            }
        }
    free(qp);
    return bound;
}

/* ----------------------------------------------------------------- select */

typedef struct { double s; int64_t t; } scored;

/* order: higher score first, equal scores by lower index */
static int by_score_desc_index_asc(const void *a, const void *b) {
    const scored *x = (const scored *)a, *y = (const scored *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->t > y->t) - (x->t < y->t);
}

/* sel_idx[B][Hkv][cap] (ascending, unused slots = -1), sel_cnt[B][Hkv].
 * Top-k over all N tokens by full sort, then the union with the sinks and
 * the window.  Returns 0, or -1 when cap is too small. */
int dko_select(int B, int Hkv, int64_t n_cap, const int32_t *seq_lens,
               const double *scores, int topk, int sink, int window,
               int32_t *sel_idx, int32_t *sel_cnt, int cap) {
    int rc = 0;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hkv; ++h) {
            int64_t n = seq_lens[b];
            const double *s = scores + ((int64_t)b * Hkv + h) * n_cap;
            scored *all = (scored *)malloc(sizeof(scored) * (size_t)(n > 0 ? n : 1));
            for (int64_t t = 0; t < n; ++t) { all[t].s = s[t]; all[t].t = t; }
            qsort(all, (size_t)n, sizeof(scored), by_score_desc_index_asc);
            int64_t kk = topk < n ? topk : n;
            char *in = (char *)calloc((size_t)(n > 0 ? n : 1), 1);
            for (int64_t r = 0; r < kk; ++r) in[all[r].t] = 1;
            for (int64_t t = 0; t < n && t < sink; ++t) in[t] = 1;
            for (int64_t t = n - window; t < n; ++t) if (t >= 0) in[t] = 1;
            int64_t c = 0;
            int32_t *out = sel_idx + ((int64_t)b * Hkv + h) * cap;
            for (int64_t t = 0; t < n; ++t)
                if (in[t]) {
                    if (c < cap) out[c] = (int32_t)t; else rc = -1;
                    ++c;
                }
            for (int64_t r = c; r < cap; ++r) out[r] = -1;
            sel_cnt[(int64_t)b * Hkv + h] = (int32_t)c;
            free(in);
            free(all);
        }
    return rc;
}

/* ----------------------------------------------------------------- attend */

/* out[B][Hq][d], lse[B][Hq] over the selected rows, in double. */
void dko_attend(int B, int Hq, int Hkv, int d, int64_t n_cap,
                const int32_t *page_table, int max_pages, int page,
                const double *q, const double *K, const double *V,
                const int32_t *sel_idx, const int32_t *sel_cnt, int cap,
                double *out, double *lse) {
    dko_layout L = make_layout(B, Hkv, d, 64, n_cap, page_table, max_pages, page);
    int G = Hq / Hkv;
    double scale = 1.0 / sqrt((double)d);
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b)
        for (int hq = 0; hq < Hq; ++hq) {
            int kvh = hq / G;
            const double *qh = q + ((int64_t)b * Hq + hq) * d;
            const int32_t *idx = sel_idx + ((int64_t)b * Hkv + kvh) * cap;
            int n = sel_cnt[(int64_t)b * Hkv + kvh];
            double *o = out + ((int64_t)b * Hq + hq) * d;
            for (int i = 0; i < d; ++i) o[i] = 0.0;
            if (n <= 0) { lse[(int64_t)b * Hq + hq] = -INFINITY; continue; }
            double *logit = (double *)malloc(sizeof(double) * (size_t)n);
            double m = -INFINITY;
            for (int r = 0; r < n; ++r) {
                const double *k = K + row_index(&L, b, kvh, idx[r]);
                double dot = 0.0;
                for (int i = 0; i < d; ++i) dot += qh[i] * k[i];
                logit[r] = dot * scale;
                if (logit[r] > m) m = logit[r];
            }
            double denom = 0.0;
            for (int r = 0; r < n; ++r) denom += exp(logit[r] - m);
            for (int r = 0; r < n; ++r) {
                double p = exp(logit[r] - m) / denom;
                const double *v = V + row_index(&L, b, kvh, idx[r]);
                for (int i = 0; i < d; ++i) o[i] += p * v[i];
            }
            lse[(int64_t)b * Hq + hq] = m + log(denom);
            free(logit);
        }
}

/* ------------------------------------------------------- block summaries */
/*
 * CSA-style two-level index (DeepSeek DSA->CSA/HCA page, CSA section: every m
 * history tokens are compressed into one summary entry and the top-k is taken
 * over the summaries; section on the compressed KV cache versus the state
 * cache: tokens of a block that is not yet complete -- the page's example has
 * 2 of m = 4 -- wait in the state cache until the block fills up).
 *
 * The pages' compressor is learned; none is available here.  The summary of
 * block i (tokens [i*m, (i+1)*m)) is therefore the hash code of the block's
 * summed key: the sign of a projection of the block's mean key is the sign of
 * the projection of its sum.  Only complete blocks, i < floor(N / m), have a
 * summary.  Attention stays exact: it runs over every token of the selected
 * blocks, the sinks, the window and the incomplete tail (the state cache).
 *
 * block codes: dense [B][Hkv][nb_cap][W64], canonical bit order.
 */
void dko_encode_blocks(int B, int Hkv, int d, int bits, int64_t n_cap,
                       const int32_t *page_table, int max_pages, int page,
                       const double *K, const int32_t *seq_lens, int block,
                       const int8_t *R, int64_t nb_cap, uint64_t *block_codes) {
    dko_layout L = make_layout(B, Hkv, d, bits, n_cap, page_table, max_pages, page);
    int w64 = bits / 64 > 0 ? bits / 64 : 1;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hkv; ++h) {
            int64_t nb = seq_lens[b] / block;
#pragma omp parallel for schedule(static)
            for (int64_t i = 0; i < nb; ++i) {
                double *ksum = (double *)calloc((size_t)d, sizeof(double));
                for (int64_t t = i * block; t < (i + 1) * block; ++t) {
                    const double *k = K + row_index(&L, b, h, t);
                    for (int e = 0; e < d; ++e) ksum[e] += k[e];
                }
                encode_one(ksum, R, bits, d, block_codes + (((int64_t)b * Hkv + h) * nb_cap + i) * w64);
                free(ksum);
            }
        }
}

/* Token selection from block scores.  block_scores: [B][Hkv][nb_cap], valid
 * for blocks i < floor(seq_lens[b] / block).  Per (b, kv head): the
 * topk_blocks best complete blocks (score desc, block index asc; all of them
 * when fewer exist), every token of each, united with the sinks [0, S), the
 * window [N-W, N) and the tail [m*floor(N/m), N).  Output as dko_select:
 * ascending ids, -1 padded to cap.  Returns 0, or -1 when cap is too small. */
int dko_select_blocks(int B, int Hkv, int64_t nb_cap, const int32_t *seq_lens, int block,
                      const double *block_scores, int topk_blocks, int sink, int window,
                      int32_t *sel_idx, int32_t *sel_cnt, int cap) {
    int rc = 0;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hkv; ++h) {
            int64_t n = seq_lens[b];
            int64_t nb = n / block;
            const double *s = block_scores + ((int64_t)b * Hkv + h) * nb_cap;
            scored *all = (scored *)malloc(sizeof(scored) * (size_t)(nb > 0 ? nb : 1));
            for (int64_t i = 0; i < nb; ++i) { all[i].s = s[i]; all[i].t = i; }
            qsort(all, (size_t)nb, sizeof(scored), by_score_desc_index_asc);
            int64_t kk = topk_blocks < nb ? topk_blocks : nb;
            char *in = (char *)calloc((size_t)(n > 0 ? n : 1), 1);
            for (int64_t r = 0; r < kk; ++r)
                for (int64_t t = all[r].t * block; t < (all[r].t + 1) * block; ++t) in[t] = 1;
            for (int64_t t = 0; t < n && t < sink; ++t) in[t] = 1;
            for (int64_t t = n - window; t < n; ++t) if (t >= 0) in[t] = 1;
            for (int64_t t = nb * block; t < n; ++t) in[t] = 1;
            int64_t c = 0;
            int32_t *out = sel_idx + ((int64_t)b * Hkv + h) * cap;
            for (int64_t t = 0; t < n; ++t)
                if (in[t]) {
                    if (c < cap) out[c] = (int32_t)t; else rc = -1;
                    ++c;
                }
            for (int64_t r = c; r < cap; ++r) out[r] = -1;
            sel_cnt[(int64_t)b * Hkv + h] = (int32_t)c;
            free(in);
            free(all);
        }
    return rc;
}

/* ---------------------------------------------------------- radius scaling */
/*
 * Radius-scaled scores (Spherical KV page, section 2.1 ADA: the compact key
 * keeps a quantized radius r~ beside its angle code, and the logit is
 * estimated as |q| * r~ * f_b(angle codes); f_b is played here by the
 * asymmetric code score s_t, and |q| is one constant per query, so the
 * ranking only needs s'_t = r~_t * s_t).
 *
 * The page does not fix the quantizer.  Reading used: 8 bits, uniform in the
 * key norm with step 1/4 and midpoint reconstruction,
 *   c_t  = min(255, floor(4 * sqrtf(sum_i k_i^2)))   sum in fp32, i ascending,
 *   r~_t = (c_t + 1/2) / 4.
 * Single precision is part of the definition, so that the integer c_t is
 * decided the same way by any implementation (sqrtf is correctly rounded).
 * On keys of the 1/64 grid the sum is exact.  s'_t is the fp32 product of
 * r~_t and the fp32 score s_t (one rounding: the double product of the two
 * is exact), returned widened to double.
 *
 * radius codes: dense [B][Hkv][n_cap], paged [P][Hkv][page] (the codes'
 * layout without the word axis), uint8.
 */
static int64_t radius_index(const dko_layout *L, int b, int h, int64_t t) {
    if (L->page == 0)
        return ((int64_t)b * L->Hkv + h) * L->n_cap + t;
    int64_t p = L->page_table[(int64_t)b * L->max_pages + t / L->page];
    return (p * L->Hkv + h) * L->page + t % L->page;
}

uint8_t dko_radius_code(const double *k, int d) {
    float s = 0.0f;
    for (int i = 0; i < d; ++i) {
        float x = (float)k[i];
        s += x * x;
    }
    float c = floorf(4.0f * sqrtf(s));
    return c >= 255.0f ? (uint8_t)255 : (uint8_t)c;
}

double dko_radius_value(uint8_t c) { return ((double)c + 0.5) / 4.0; }

/* Radius codes of tokens [0, seq_lens[b]) of every (b, kv head). */
void dko_radius_codes(int B, int Hkv, int d, int64_t n_cap, const int32_t *page_table, int max_pages, int page,
                      const double *K, const int32_t *seq_lens, uint8_t *rc) {
    dko_layout L = make_layout(B, Hkv, d, 64, n_cap, page_table, max_pages, page);
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hkv; ++h)
            for (int64_t t = 0; t < seq_lens[b]; ++t)
                rc[radius_index(&L, b, h, t)] = dko_radius_code(K + row_index(&L, b, h, t), d);
}

/* s'[b][h][t] = fp32(r~_t * s[b][h][t]) for t < seq_lens[b] (scores rows of
 * length n_cap, as dko_scores writes them); other entries untouched. */
void dko_radius_scale(int B, int Hkv, int64_t n_cap, const int32_t *page_table, int max_pages, int page,
                      const int32_t *seq_lens, const uint8_t *rc, const double *scores, double *out) {
    dko_layout L = make_layout(B, Hkv, 1, 64, n_cap, page_table, max_pages, page);
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hkv; ++h)
            for (int64_t t = 0; t < seq_lens[b]; ++t) {
                int64_t i = ((int64_t)b * Hkv + h) * n_cap + t;
                float st = (float)scores[i];  /* the token path's fp32 score */
                float prod = (float)(dko_radius_value(rc[radius_index(&L, b, h, t)]) * (double)st);
                out[i] = (double)prod + 0.0;
            }
}

/* ------------------------------------------------------ precision tiers */
/*
 * Tier-homogeneous pages (Spherical KV page, section 2.2 RDR: every retained
 * state gets a precision tier, protected states keep the highest one, and
 * states are grouped into pages of one tier so that the decode reads a page
 * in one pass guided by its header; DASH-KV page, section
 * "技术架构：动态混合精度机制", paras 2-3: the tokens that matter keep full
 * floating-point precision, the others a cheaper form; DeepSeek DSA->CSA/HCA
 * page: the KV store itself is mixed-precision).
 *
 * Two tiers.  Tier 0: the bf16 rows as stored.  Tier 1: FP8 E4M3 rows (OCP
 * 8-bit floating point, "FN" variant: 1 sign bit, 4 exponent bits with bias
 * 7, 3 mantissa bits, no infinities, S.1111.111 is NaN, largest finite 448)
 * with one power-of-two scale per (token, kv head) row and per tensor (K, V):
 *   s   = the largest integer with amax * 2^s <= 448, capped at 127
 *         (amax = max_i |x_i| over the row; s = 0 for an all-zero row);
 *   c_i = e4m3 code of x_i * 2^s, rounded to nearest, ties to even;
 *   x~_i = value(c_i) * 2^-s.
 * A page's tier is a byte per physical page (its header).  The controller:
 * a page is demoted to tier 1 when every one of its tokens lies in the
 * middle [S, N - W) of its sequence (no sink, no window token), it is still
 * tier 0 and the caller did not protect it.  Attention over a selection reads
 * x~ for rows of tier-1 pages and the bf16 rows otherwise, exactly as before.
 *
 * FP8 arrays: k8 / v8 [P][page][Hkv][d] uint8 (the K / V page layout),
 * exps [P][page][Hkv][2] int8 (s of the K row, then of the V row).
 */
double dko_e4m3_value(uint8_t c) {
    int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    double v = e == 0 ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Nearest e4m3 code of v, ties to the even code; |v| above 448 saturates to
 * +-448 (never reached for scaled rows). */
uint8_t dko_e4m3_encode(double v) {
    uint8_t sign = (v < 0.0 || (v == 0.0 && signbit(v))) ? 0x80 : 0;
    double a = fabs(v);
    if (a >= 448.0) return sign | 0x7E;
    /* quantum of the binade of a: 2^(E-3) for a in [2^E, 2^(E+1)), E >= -6;
     * 2^-9 below 2^-6 (subnormals) */
    int E;
    if (a < ldexp(1.0, -6)) E = -6;
    else {
        frexp(a, &E);  /* a = f * 2^E, f in [0.5, 1) */
        E -= 1;
    }
    double quantum = ldexp(1.0, E - 3);
    double n = a / quantum;            /* exact: power-of-two divisor */
    double r = floor(n);
    double frac = n - r;
    if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
    double q = r * quantum;            /* the rounded magnitude */
    if (q > 448.0) q = 448.0;
    /* the code of q */
    if (q < ldexp(1.0, -6)) return sign | (uint8_t)(q / ldexp(1.0, -9));
    int Eq;
    double f = frexp(q, &Eq);          /* q = f * 2^Eq = (2f) * 2^(Eq-1) */
    int e = Eq - 1 + 7;
    int m = (int)((2.0 * f - 1.0) * 8.0);
    return sign | (uint8_t)((e << 3) | m);
}

int dko_tier_exponent(const double *x, int d) {
    double amax = 0.0;
    for (int i = 0; i < d; ++i)
        if (fabs(x[i]) > amax) amax = fabs(x[i]);
    if (amax == 0.0) return 0;
    /* amax = f * 2^E, f in [0.5, 1); 448 = 0.875 * 2^9 */
    int E;
    double f = frexp(amax, &E);
    int s = (f <= 0.875) ? 9 - E : 8 - E;
    return s > 127 ? 127 : s;
}

/* Scale exponent and codes of one row. */
void dko_tier_quantize_row(const double *x, int d, uint8_t *codes, int8_t *s_out) {
    int s = dko_tier_exponent(x, d);
    for (int i = 0; i < d; ++i) codes[i] = dko_e4m3_encode(ldexp(x[i], s));
    *s_out = (int8_t)s;
}

/* The controller over every (sequence, logical page) of a paged cache:
 * demote the eligible pages (see above), writing their codes and exponents
 * and setting tier[p] = 1.  protect may be NULL.  Returns the number of pages
 * demoted. */
int dko_demote_pages(int B, int Hkv, int d, int page, const int32_t *page_table, int max_pages,
                     const double *K, const double *V, const int32_t *seq_lens, int S, int W,
                     const uint8_t *protect, uint8_t *tier, uint8_t *k8, uint8_t *v8, int8_t *exps) {
    int demoted = 0;
    for (int b = 0; b < B; ++b) {
        int64_t n = seq_lens[b];
        for (int p = 0; p < max_pages; ++p) {
            int64_t lo = (int64_t)p * page, hi = lo + page;  /* tokens [lo, hi) */
            if (lo < S || hi > n - W) continue;
            int32_t phys = page_table[(int64_t)b * max_pages + p];
            if (phys < 0 || tier[phys] != 0 || (protect && protect[phys])) continue;
            for (int slot = 0; slot < page; ++slot)
                for (int h = 0; h < Hkv; ++h) {
                    int64_t row = ((int64_t)phys * page + slot) * Hkv + h;
                    dko_tier_quantize_row(K + row * d, d, k8 + row * d, exps + row * 2);
                    dko_tier_quantize_row(V + row * d, d, v8 + row * d, exps + row * 2 + 1);
                }
            tier[phys] = 1;
            ++demoted;
        }
    }
    return demoted;
}
