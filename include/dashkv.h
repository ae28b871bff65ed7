/*
 * dashkv.h -- C ABI of the decode-step hash-score -> top-k -> exact sparse
 * attention library for NVIDIA B200 (sm_100a).
 *
 * One decode step over a long KV cache runs in four stages:
 *
 *   1. hash_encode  every cached key k (head dim d) becomes `bits` sign bits
 *                   against seeded Rademacher (+1/-1) hyperplanes R:
 *                   bit_j = [ sum_i R[j][i] k[i] >= 0 ]  (a tie at 0 gives 1).
 *                   DASH-KV page, section "从平方到线性：复杂度降低的数学原理"
 *                   (locality-sensitive hashing of the keys) and section
 *                   "技术架构：动态混合精度机制" (a light key-side encoder).
 *   2. asym_score   the query stays in full precision; it is projected onto
 *                   the same hyperplanes and scored against the packed key
 *                   codes, s_t = sum_j qp_j (2 bit_tj - 1); with grouped
 *                   query attention the scores of the query heads that share
 *                   a KV head are summed.  DASH-KV page, section
 *                   "DASH-KV的核心创新：非对称深度哈希" (asymmetric encoding);
 *                   Spherical KV page, section 2.1 ADA (logits straight from
 *                   compact codes, no dense key is rebuilt).
 *   3. select       the top-k scores per (sequence, KV head), ties to the
 *                   lower index, united with the first S (sink) and last W
 *                   (window) tokens.  DeepSeek DSA->CSA/HCA page, section
 *                   "从 DSA 说起" (indexer then top-k) and the SWA paragraph
 *                   of its CSA section; DySCO page, Q3 (attention sinks).
 *   4. attention    softmax(q K^T / sqrt(d)) V over the selected tokens only,
 *                   fp32 accumulation, one output per query head.
 *                   DeepSeek DSA->CSA/HCA page, section "从 DSA 说起"
 *                   (real attention on the top-k only).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Pointers marked "device" are CUDA device pointers; the caller owns and
 *    allocates every buffer.  The library allocates no device memory.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream) and never synchronises the host, except
 *    dashkv_get_error().
 *  - Arguments are validated on the host before anything is launched; an
 *    invalid call returns a status and launches nothing.  Problems only the
 *    device can see (a page id outside [0, num_pages), a sequence length
 *    beyond the cache capacity) set a per-device error word that
 *    dashkv_get_error() reads and clears; the affected tokens are skipped.
 *  - Layouts (B sequences, Hkv KV heads, Hq = G * Hkv query heads,
 *    W = max(1, bits / 64) 64-bit code words per key):
 *      keys / values, dense : bf16 [B][Hkv][n_cap][d]
 *      keys / values, paged : bf16 [num_pages][page_size][Hkv][d]
 *      codes, dense         : u64  [B][Hkv][n_cap][W]
 *      codes, paged         : u64  [num_pages][Hkv][page_size][W]
 *      token t of sequence b lives in physical page
 *      page_table[b * max_pages + t / page_size], slot t % page_size.
 *      Code bits: hyperplane j is bit j % 8 of code byte j / 8 (T = bits/8
 *      bytes, little-endian, i.e. word j / 64 bit j % 64 before the rotation
 *      below; a 32-bit code occupies the low half of its word, high half 0).
 *      Storage rotation: token t's T code bytes are stored rotated by t mod T
 *      (stored byte p holds code byte (p + t mod T) mod T), the order in which
 *      the scorer's lanes consume them.  (Paged: page_size is a multiple of 32,
 *      so the slot index gives the same t mod T.)
 *      queries q : bf16 [B][Hq][d]; query head h reads KV head h / G.
 *  - seq_lens (device int32 [B]) holds each sequence's cached length; the
 *    current decode step's own key is expected to be appended first, so the
 *    recent window includes it.
 */
#ifndef DASHKV_H
#define DASHKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum dashkv_status {
    DASHKV_OK = 0,
    DASHKV_ERR_INVALID_ARG = 1,  /* null pointer, bad shape or size                  */
    DASHKV_ERR_UNSUPPORTED = 2,  /* d, bits, G or page_size outside the supported set */
    DASHKV_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required       */
    DASHKV_ERR_CAPACITY = 4,     /* device error word: a sequence outgrew its cache   */
    DASHKV_ERR_CUDA = 5,         /* a CUDA runtime call failed (launch, sync, copy)   */
    DASHKV_ERR_DEVICE = 6,       /* device error word: bad page id in page_table      */
    DASHKV_ERR_NO_DEVICE = 7,    /* no usable CUDA device                             */
    DASHKV_ERR_TIMEOUT = 8       /* device error word: a bounded wait in a kernel gave
                                    up (a bulk copy did not land); results invalid    */
} dashkv_status;

/* Selection path.  By default dashkv_select runs one kernel with one
 * thread-block cluster per (sequence, kv head): its CTAs (one per SM, up to 16
 * per cluster) stream the codes, build a histogram of the scores and exchange
 * histograms and boundary tokens through distributed shared memory and
 * hardware cluster barriers; dashkv_decode_step runs its own clustered kernel
 * (append, selection and attention in one launch: its CTAs keep candidates
 * at or above a sampled threshold in shared memory and attend over what they
 * kept).  Without cluster launch support, or with this flag, the selection runs
 * two ordinary kernels instead (and dashkv_decode_step the three separate
 * calls).  All give identical selections. */
#define DASHKV_FLAG_TWO_KERNEL_SELECT 1

/* Problem description.  Supported: head_dim in {64, 128}; bits in
 * {32, 64, 128}; num_q_heads = G * num_kv_heads with G in {1, 2, 4, 8};
 * topk >= 1; sink, window >= 0; page_size 0 (dense) or a multiple of 32 up
 * to 1024. */
typedef struct dashkv_config {
    int32_t batch;          /* B  */
    int32_t num_q_heads;    /* Hq */
    int32_t num_kv_heads;   /* Hkv */
    int32_t head_dim;       /* d  */
    int32_t bits;           /* hash bits per key (b) */
    int32_t topk;           /* k  */
    int32_t sink;           /* S: first tokens always kept */
    int32_t window;         /* W: last tokens always kept  */
    int32_t page_size;      /* 0 = dense layout            */
    int32_t flags;          /* DASHKV_FLAG_* bits; 0 = defaults */
    uint64_t seed;          /* hyperplane seed             */
} dashkv_config;

/* The KV cache the calls read (and dashkv_append_keys writes). */
typedef struct dashkv_kv_view {
    void *k;                      /* device bf16 keys   (layout above)               */
    void *v;                      /* device bf16 values (layout above)               */
    uint64_t *codes;              /* device key codes   (layout above)               */
    int64_t n_cap;                /* dense: token capacity per (b, kv head)          */
    const int32_t *page_table;    /* device [B][max_pages]; NULL = dense layout      */
    int32_t max_pages;            /* paged: row length of page_table                 */
    int32_t num_pages;            /* paged: physical pages held by k, v and codes    */
} dashkv_kv_view;

typedef struct dashkv_ctx dashkv_ctx;

/* Validate `cfg` and build a context holding it and the hyperplanes R
 * (host memory only; R[j][i] is -1 when the top bit of splitmix64 output
 * number j*d+i+1 from `seed` is set, else +1).  *out receives the context;
 * release it with dashkv_destroy().  Binds to the CUDA device current at
 * this call (queried for its SM count). */
dashkv_status dashkv_create(const dashkv_config *cfg, dashkv_ctx **out);
void dashkv_destroy(dashkv_ctx *ctx);

/* Bytes of device workspace dashkv_select / dashkv_sparse_decode need for
 * caches of at most `max_tokens` tokens per sequence (dense: n_cap; paged:
 * max_pages * page_size).  The workspace must be zero-filled once before its
 * first use; every call that returns DASHKV_OK leaves it ready for the next
 * one.  Select and decode may share one workspace; calls that use the same
 * workspace must not overlap on the GPU. */
size_t dashkv_workspace_size(const dashkv_ctx *ctx, int64_t max_tokens);

/* Stage 1 for a whole cache: write the codes of tokens [0, seq_lens[b]) of
 * every (b, kv head) into kv->codes.  Reads kv->k.  seq_lens: device int32 [B]. */
dashkv_status dashkv_encode_keys(dashkv_ctx *ctx, const dashkv_kv_view *kv,
                                 const int32_t *seq_lens, void *stream);

/* One decode step's cache append: k_new / v_new (device bf16 [B][Hkv][d])
 * are written at position seq_lens[b] of every (b, kv head), their codes
 * into kv->codes, then seq_lens[b] is incremented on the device. */
dashkv_status dashkv_append_keys(dashkv_ctx *ctx, const dashkv_kv_view *kv,
                                 const void *k_new, const void *v_new,
                                 int32_t *seq_lens, void *stream);

/* Stages 2 and 3.  q: device bf16 [B][Hq][d].  Writes, per (b, kv head),
 * the ascending, duplicate-free selected token ids into
 * sel_idx (device int32 [B][Hkv][topk + sink + window], unused tail = -1)
 * and their number into sel_cnt (device int32 [B][Hkv]).
 * scores (optional, may be NULL): device fp32 [B][Hkv][max_tokens]
 * receives s_t for t < seq_lens[b] (other entries untouched).
 * Reads kv->codes (and kv->page_table), never kv->k / kv->v. */
dashkv_status dashkv_select(dashkv_ctx *ctx, const dashkv_kv_view *kv, const void *q,
                            const int32_t *seq_lens, int32_t *sel_idx, int32_t *sel_cnt,
                            float *scores, void *workspace, size_t workspace_bytes,
                            void *stream);

/* Allocation-free variant of dashkv_select.  The pages have no counterpart
 * of this call: it is an interface convenience, not part of the method.
 * For callers that may not allocate device memory at all -- e.g. code that
 * runs while a CUDA graph is being captured (cudaMalloc cannot be captured)
 * or a host runtime that owns every device allocation -- it uses, instead of
 * a caller workspace, one scratch array compiled into this library: 24 MiB
 * (25165824 bytes) per device, the limit.  Inputs whose
 * dashkv_workspace_size(ctx, capacity) exceeds it are rejected with
 * DASHKV_ERR_WORKSPACE before anything is launched.  It allocates nothing.
 * The device current at the call must be the context's (else
 * DASHKV_ERR_INVALID_ARG).  The first call on a device looks the scratch up
 * (cudaGetSymbolAddress) and zero-fills it with a synchronising memset: that
 * first call must come before any stream capture (during capture it returns
 * DASHKV_ERR_INVALID_ARG).  A later call whose problem shape lays the scratch
 * out differently from the previous successful call's, or that follows a
 * failed call, first clears the selection's counter words with
 * cudaMemsetAsync on `stream` (stream-ordered, so it may be captured).  All
 * calls on a device share the one scratch and it keeps the last call's
 * contents: calls that overlap on the GPU (other streams, other threads)
 * race and must be serialised by the caller.  Arguments and results are
 * those of dashkv_select. */
dashkv_status dashkv_select_static(dashkv_ctx *ctx, const dashkv_kv_view *kv, const void *q,
                                   const int32_t *seq_lens, int32_t *sel_idx, int32_t *sel_cnt,
                                   float *scores, void *stream);

/* Stage 4.  Exact softmax attention of every query head over the rows its
 * KV head selected: out (device fp32 [B][Hq][d]); lse (optional, device
 * fp32 [B][Hq]) receives log sum_t exp(q.K_t / sqrt(d)) (-inf when nothing
 * is selected, out = 0 then).  sel_idx / sel_cnt as dashkv_select writes
 * them; ids must be < seq_lens[b].  seq_lens (optional, device int32 [B]):
 * NULL attends over exactly the rows of sel_idx.  When given, sel_idx /
 * sel_cnt must be dashkv_select's output for these lengths: the sinks and the
 * window (which every selection contains, at the two ends of the list) are
 * then read from the token range directly by extra CTAs that need nothing
 * from the selection and may run while it is still being computed. */
dashkv_status dashkv_sparse_decode(dashkv_ctx *ctx, const dashkv_kv_view *kv, const void *q,
                                   const int32_t *seq_lens, const int32_t *sel_idx,
                                   const int32_t *sel_cnt, float *out, float *lse, void *workspace,
                                   size_t workspace_bytes, void *stream);

/* The whole decode step in one launch: dashkv_append_keys, dashkv_select and
 * dashkv_sparse_decode (given the lengths) fused into one kernel of one
 * thread-block cluster per (sequence, kv head), with the same results as those
 * three calls made in that order: k_new / v_new (device bf16 [B][Hkv][d]) are
 * written at position seq_lens[b] of every (b, kv head) with their codes, the
 * selection (over the cache including them) goes to sel_idx / sel_cnt, the
 * attention output to out (and lse when not NULL), and seq_lens[b] is
 * incremented on the device.  Pages above: DASH-KV page (hashing, asymmetric
 * scoring), DeepSeek DSA->CSA/HCA page "从 DSA 说起" (indexer, top-k, attention
 * on the top-k), the SWA paragraph of its CSA section and the DySCO page, Q3
 * (window and sinks).  The workspace is dashkv_select's (zero-filled once;
 * every successful call leaves it ready for the next).  Without the clustered
 * path (see DASHKV_FLAG_TWO_KERNEL_SELECT) the three calls run one after the
 * other. */
dashkv_status dashkv_decode_step(dashkv_ctx *ctx, const dashkv_kv_view *kv, const void *q, const void *k_new,
                                 const void *v_new, int32_t *seq_lens, int32_t *sel_idx, int32_t *sel_cnt,
                                 float *out, float *lse, void *workspace, size_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------------
 * Block summaries: a CSA-style two-level index.
 *
 * DeepSeek DSA->CSA/HCA page, section CSA: every m history tokens are
 * compressed into one summary entry and the top-k is taken over the
 * summaries, while a sliding window keeps the recent tokens exact; section on
 * the compressed KV cache versus the state cache: the tokens of a block that
 * is not yet complete wait in the state cache until m have arrived.
 *
 * Without the pages' learned compressor, the summary of block i (tokens
 * [i m, (i + 1) m) of a sequence) is the code of the block's summed key,
 * bit_j = [ sum_i R[j][i] (sum_t k_t)[i] >= 0 ], stored like a token code.
 * Only complete blocks, i < seq_lens[b] / m, have one.  Selection scores the
 * summaries with the query exactly as dashkv_select scores keys, takes the
 * top kb = topk / m blocks (ties to the lower block), and lists every token of
 * those blocks united with the sinks and the window; the window must cover
 * the incomplete tail (window >= m - 1).  dashkv_sparse_decode then attends
 * exactly over that list.  The scan reads one code per m tokens.
 * ------------------------------------------------------------------------ */
typedef struct dashkv_block_view {
    uint64_t *codes;   /* device u64 [B][Hkv][nb_cap][W]: summary of block i at
                          index i, stored (rotated by i mod T) like token codes */
    int64_t nb_cap;    /* blocks per (b, kv head); 1 <= nb_cap <= token capacity */
    int32_t block;     /* m, tokens per block: a power of two in [1, 1024]      */
    int32_t reserved;  /* must be 0                                              */
} dashkv_block_view;

/* Summaries of every complete block [0, seq_lens[b] / m) of every (b, kv
 * head) from kv->k (dense or paged), written to blk->codes.  Blocks beyond
 * nb_cap set the capacity error word and are skipped. */
dashkv_status dashkv_encode_blocks(dashkv_ctx *ctx, const dashkv_kv_view *kv, const dashkv_block_view *blk,
                                   const int32_t *seq_lens, void *stream);

/* Decode-step update, to be called after dashkv_append_keys with the lengths
 * it incremented: for every sequence whose length is now a multiple of m, the
 * summary of the block that the append completed (seq_lens[b] / m - 1) is
 * encoded from kv->k.  Other sequences are left alone (their new token waits
 * in the tail).  Idempotent. */
dashkv_status dashkv_append_blocks(dashkv_ctx *ctx, const dashkv_kv_view *kv, const dashkv_block_view *blk,
                                   const int32_t *seq_lens, void *stream);

/* Stages 2 and 3 over the summaries.  Writes sel_idx / sel_cnt exactly as
 * dashkv_select does (ascending, duplicate-free, rows of topk + sink + window,
 * -1 after the count; sinks first, window last), for the token set
 *   { tokens of the top topk / m complete blocks } U [0, S) U [N - W, N).
 * block_scores (optional): device fp32 [B][Hkv][nb_cap] receives the summary
 * scores of blocks i < seq_lens[b] / m.  Requires topk >= m and window >= m-1
 * (else DASHKV_ERR_UNSUPPORTED).  The workspace is dashkv_select's (same size
 * for the token capacity); reads blk->codes, kv only for its capacity. */
dashkv_status dashkv_select_blocks(dashkv_ctx *ctx, const dashkv_kv_view *kv, const dashkv_block_view *blk,
                                   const void *q, const int32_t *seq_lens, int32_t *sel_idx, int32_t *sel_cnt,
                                   float *block_scores, void *workspace, size_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------------
 * Radius-scaled scores.
 *
 * Spherical KV page, section 2.1 ADA: a compact key keeps a quantized radius
 * r~ beside its angle code, and the logit is estimated as |q| r~ f_b(codes).
 * Here the selection may rank s'_t = r~_t s_t (s_t the score of
 * dashkv_select; |q| is one constant per query).  The radius code of a key is
 *   c = min(255, floor(4 sqrt(sum_i k_i^2)))   (fp32, i ascending, every
 *                                               operation rounded once),
 *   r~ = (c + 1/2) / 4,
 * stored as one byte per token and kv head: dense [B][Hkv][n_cap], paged
 * [num_pages][Hkv][page_size] (the codes' layout without the word axis).
 * s' is the fp32 product of r~ and the fp32 score (one rounding).
 * ------------------------------------------------------------------------ */

/* Radius codes of tokens [0, seq_lens[b]) of every (b, kv head) from kv->k,
 * written to `radius` (device, layout above). */
dashkv_status dashkv_encode_radius(dashkv_ctx *ctx, const dashkv_kv_view *kv, const int32_t *seq_lens,
                                   uint8_t *radius, void *stream);

/* Decode-step update, after dashkv_append_keys with the lengths it
 * incremented: the radius code of token seq_lens[b] - 1 of every kv head. */
dashkv_status dashkv_append_radius(dashkv_ctx *ctx, const dashkv_kv_view *kv, const int32_t *seq_lens,
                                   uint8_t *radius, void *stream);

/* dashkv_select on the radius-scaled scores: same arguments and outputs
 * (scores, when given, receives s'), plus the radius codes.  Runs the fused
 * selection only: DASHKV_ERR_UNSUPPORTED without cluster launch support or
 * with DASHKV_FLAG_TWO_KERNEL_SELECT. */
dashkv_status dashkv_select_radius(dashkv_ctx *ctx, const dashkv_kv_view *kv, const uint8_t *radius, const void *q,
                                   const int32_t *seq_lens, int32_t *sel_idx, int32_t *sel_cnt, float *scores,
                                   void *workspace, size_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------------
 * Precision tiers of pages (paged caches only).
 *
 * Spherical KV page, section 2.2 RDR: every retained state gets a precision
 * tier, protected states keep the highest one, and states are grouped into
 * pages of a single tier so that the decode reads each page in one pass
 * guided by its header.  DASH-KV page, section "技术架构：动态混合精度机制",
 * paras 2-3: the tokens that matter keep full floating-point precision, the
 * others a cheaper form.
 *
 * Tier 0: the bf16 rows of kv->k / kv->v.  Tier 1: FP8 E4M3 (OCP "FN"
 * encoding) rows with one power-of-two scale per (token, kv head) row and
 * tensor: s = the largest integer with max_i |x_i| * 2^s <= 448, capped at
 * 127 (0 for a zero row); code_i = E4M3(x_i * 2^s), nearest, ties to even;
 * the row reads back as value(code_i) * 2^-s (exact in fp32).  The page
 * header is one tier byte per physical page.
 * ------------------------------------------------------------------------ */
typedef struct dashkv_tier_view {
    uint8_t *tier;  /* device u8 [num_pages]: 0 = bf16 rows, 1 = FP8 rows.  The caller
                       zero-fills it once and zeroes the byte of a page it reassigns */
    uint8_t *k8;    /* device u8 [num_pages][page][Hkv][d] FP8 keys (16-byte aligned) */
    uint8_t *v8;    /* device u8 [num_pages][page][Hkv][d] FP8 values (16-byte aligned) */
    int8_t *exps;   /* device i8 [num_pages][page][Hkv][2]: s of the K row, then of the V row
                       (4-byte aligned) */
} dashkv_tier_view;

/* The tier controller.  For every sequence b and logical page p whose tokens
 * [p page, (p + 1) page) all lie in [S, seq_lens[b] - W) -- no sink, no window
 * token -- and whose physical page is still tier 0 and not protected
 * (protect: optional device u8 [num_pages], nonzero = keep bf16), the page's K
 * and V rows of every kv head are quantized into tv->k8 / tv->v8 / tv->exps
 * and its tier byte is set to 1.  Pages already tier 1 are left alone (their
 * rows must not change afterwards).  A page-table entry outside
 * [0, num_pages) sets the device error word and is skipped.  A physical page
 * must belong to one sequence.  DASHKV_ERR_UNSUPPORTED for dense caches. */
dashkv_status dashkv_demote_pages(dashkv_ctx *ctx, const dashkv_kv_view *kv, const dashkv_tier_view *tv,
                                  const int32_t *seq_lens, const uint8_t *protect, void *stream);

/* dashkv_sparse_decode over a tiered paged cache: the same selection, the
 * same exact fp32 attention, with the rows of tier-1 pages read from tv (their
 * dequantized FP8 values) and the others from kv->k / kv->v.  Same arguments,
 * workspace and error behaviour as dashkv_sparse_decode; in addition
 * DASHKV_ERR_INVALID_ARG for a missing or misaligned tier view and
 * DASHKV_ERR_UNSUPPORTED for dense caches. */
dashkv_status dashkv_sparse_decode_tiered(dashkv_ctx *ctx, const dashkv_kv_view *kv, const dashkv_tier_view *tv,
                                          const void *q, const int32_t *seq_lens, const int32_t *sel_idx,
                                          const int32_t *sel_cnt, float *out, float *lse, void *workspace,
                                          size_t workspace_bytes, void *stream);

/* Synchronise `stream`, then read and clear the current device's error
 * word: DASHKV_OK, DASHKV_ERR_TIMEOUT, DASHKV_ERR_DEVICE, DASHKV_ERR_CAPACITY
 * (in that order of precedence), or DASHKV_ERR_CUDA when the stream reports an
 * error. */
dashkv_status dashkv_get_error(void *stream);

/* The hyperplanes a context built with (seed, bits, d) uses, as int8 +1/-1
 * in host memory [bits][d]. */
dashkv_status dashkv_hyperplanes(uint64_t seed, int32_t bits, int32_t head_dim, int8_t *host_out);

/* Number of kernels dashkv_select launches for caches of `max_tokens` tokens
 * per sequence: 1 (fused, clustered) or 2 (score, then collect); 0 when ctx
 * is NULL.  For profiling tools that trace individual kernels. */
int32_t dashkv_select_kernels(const dashkv_ctx *ctx, int64_t max_tokens);

/* Optional kernel tracing for profiling.  While `events` is non-NULL, every
 * following call on this context records events[2k] (a cudaEvent_t) on its
 * stream right before the k-th kernel it launches and events[2k + 1] right
 * after it (k counts from 0 within each call; kernels beyond n_events / 2 are
 * not traced).  The array must stay valid until tracing is turned off with
 * events = NULL.  The caller owns the events. */
dashkv_status dashkv_set_trace(dashkv_ctx *ctx, void **events, int32_t n_events);

/* Static string naming a status. */
const char *dashkv_status_str(dashkv_status status);

#ifdef __cplusplus
}
#endif
#endif /* DASHKV_H */
