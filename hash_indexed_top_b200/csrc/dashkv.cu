// dashkv.cu -- the C ABI declared in include/dashkv.h: host-side validation,
// context, workspace carving and kernel launches.  Every stage of the decode
// step runs in the kernels of encode.cuh, select.cuh, decode.cuh and
// blocks.cuh; this file
// only checks arguments and enqueues them.  The library allocates no device
// memory: the caller passes every buffer, including the workspace.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <type_traits>

#include "../../include/dashkv.h"
#include "blocks.cuh"
#include "common.cuh"
#include "decode.cuh"
#include "encode.cuh"
#include "radius.cuh"
#include "select.cuh"
#include "step_args.cuh"
#include "tiers.cuh"

namespace dkv {
__device__ unsigned g_error_word;  // the device error word (declared in common.cuh)
}  // namespace dkv

using namespace dkv;

struct dashkv_ctx {
    dashkv_config cfg;
    RBits R;
    int device;
    int sm_count;
    int cluster_max;  // CTAs per (b, h) cluster of the clustered step kernel; 0: no cluster launch
    int step_smem;    // dynamic shared memory of a step-kernel launch (the opt-in maximum minus static)
    int force_two_kernel;
    void **trace;   // optional cudaEvent_t pairs around each kernel of a call
    int n_trace;
};

namespace {
// Records the tracing events around the kernels of one call.
struct Tracer {
    const dashkv_ctx *ctx;
    cudaStream_t st;
    int k = 0;
    Tracer(const dashkv_ctx *c, cudaStream_t s) : ctx(c), st(s) {}
    // External records: under stream capture they become event-record nodes of
    // the graph (timeable on every replay) rather than capture dependencies.
    void before() {
        if (ctx->trace && 2 * k + 1 < ctx->n_trace)
            cudaEventRecordWithFlags((cudaEvent_t)ctx->trace[2 * k], st, cudaEventRecordExternal);
    }
    void after() {
        if (ctx->trace && 2 * k + 1 < ctx->n_trace)
            cudaEventRecordWithFlags((cudaEvent_t)ctx->trace[2 * k + 1], st, cudaEventRecordExternal);
        ++k;
    }
};
}  // namespace

namespace {

// splitmix64: output number n (n >= 1) of the stream that starts at `seed`.
uint64_t splitmix64_at(uint64_t seed, uint64_t n) {
    uint64_t z = seed + n * 0x9E3779B97F4A7C15ULL;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

// R[j][i] = -1 iff the top bit of output j*d+i+1 is set; packed as sign bits.
void build_rbits(uint64_t seed, int bits, int d, RBits *R) {
    memset(R, 0, sizeof(*R));
    for (int j = 0; j < bits; ++j)
        for (int i = 0; i < d; ++i)
            if (splitmix64_at(seed, (uint64_t)j * d + i + 1) >> 63) R->w[j * (d / 32) + i / 32] |= 1u << (i % 32);
}

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

dashkv_status check_config(const dashkv_config *c) {
    if (!c) return DASHKV_ERR_INVALID_ARG;
    if (c->batch <= 0 || c->num_kv_heads <= 0 || c->num_q_heads <= 0 || c->topk <= 0 || c->sink < 0 ||
        c->window < 0 || c->page_size < 0 || (c->flags & ~DASHKV_FLAG_TWO_KERNEL_SELECT))
        return DASHKV_ERR_INVALID_ARG;
    if (c->num_q_heads % c->num_kv_heads) return DASHKV_ERR_INVALID_ARG;
    const int G = c->num_q_heads / c->num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return DASHKV_ERR_UNSUPPORTED;
    if (c->head_dim != 64 && c->head_dim != 128) return DASHKV_ERR_UNSUPPORTED;
    if (c->bits != 32 && c->bits != 64 && c->bits != 128) return DASHKV_ERR_UNSUPPORTED;
    if (c->page_size && (c->page_size % 32 || c->page_size > 1024)) return DASHKV_ERR_UNSUPPORTED;
    if (c->num_kv_heads > 32) return DASHKV_ERR_UNSUPPORTED;
    if ((int64_t)c->topk + c->sink + c->window > 0x7fffffff / 2) return DASHKV_ERR_INVALID_ARG;
    return DASHKV_OK;
}

dashkv_status check_view(const dashkv_ctx *ctx, const dashkv_kv_view *kv, bool need_kv, bool need_codes) {
    if (!kv) return DASHKV_ERR_INVALID_ARG;
    const dashkv_config &c = ctx->cfg;
    if (need_kv && (!kv->k || !kv->v || !aligned(kv->k, 16) || !aligned(kv->v, 16))) return DASHKV_ERR_INVALID_ARG;
    if (need_codes && (!kv->codes || !aligned(kv->codes, c.bits == 128 ? 16 : 8))) return DASHKV_ERR_INVALID_ARG;
    if (c.page_size) {
        if (!kv->page_table || kv->max_pages <= 0 || kv->num_pages <= 0) return DASHKV_ERR_INVALID_ARG;
    } else {
        if (kv->page_table || kv->n_cap <= 0) return DASHKV_ERR_INVALID_ARG;
    }
    const int64_t cap = c.page_size ? (int64_t)kv->max_pages * c.page_size : kv->n_cap;
    if (cap > 0x7fffffffLL) return DASHKV_ERR_INVALID_ARG;  // token ids are int32
    return DASHKV_OK;
}

KV make_kv(const dashkv_ctx *ctx, const dashkv_kv_view *kv) {
    KV o;
    o.k = static_cast<__nv_bfloat16 *>(kv->k);
    o.v = static_cast<__nv_bfloat16 *>(kv->v);
    o.codes = kv->codes;
    o.n_cap = kv->n_cap;
    o.page_table = kv->page_table;
    o.max_pages = kv->max_pages;
    o.num_pages = kv->num_pages;
    o.page_size = ctx->cfg.page_size;
    o.Hkv = ctx->cfg.num_kv_heads;
    o.d = ctx->cfg.head_dim;
    o.W = ctx->cfg.bits >= 64 ? ctx->cfg.bits / 64 : 1;
    o.len_shift = 0;
    o.radius = nullptr;
    return o;
}

// log2 of a power of two in [1, 1024], else -1.
int block_shift(int32_t m) {
    for (int s = 0; s <= 10; ++s)
        if (m == (1 << s)) return s;
    return -1;
}

// Block summaries: the codes and block size are valid, and the block capacity
// lies in [1, token capacity] (so the selection workspace laid out for the
// token capacity also serves the block selection).
dashkv_status check_blocks(const dashkv_ctx *ctx, const dashkv_kv_view *kv, const dashkv_block_view *blk) {
    if (!blk || !blk->codes || block_shift(blk->block) < 0 || blk->reserved) return DASHKV_ERR_INVALID_ARG;
    if (!aligned(blk->codes, ctx->cfg.bits == 128 ? 16 : 8)) return DASHKV_ERR_INVALID_ARG;
    const int64_t cap = ctx->cfg.page_size ? (int64_t)kv->max_pages * ctx->cfg.page_size : kv->n_cap;
    if (blk->nb_cap < 1 || blk->nb_cap > cap) return DASHKV_ERR_INVALID_ARG;
    return DASHKV_OK;
}

// The block codes as a dense cache of N >> log2(m) entries per sequence (no
// keys or values behind it).
KV make_blk(const dashkv_ctx *ctx, const dashkv_block_view *blk) {
    KV o;
    o.k = nullptr;
    o.v = nullptr;
    o.codes = blk->codes;
    o.n_cap = blk->nb_cap;
    o.page_table = nullptr;
    o.max_pages = 0;
    o.num_pages = 0;
    o.page_size = 0;
    o.Hkv = ctx->cfg.num_kv_heads;
    o.d = ctx->cfg.head_dim;
    o.W = ctx->cfg.bits >= 64 ? ctx->cfg.bits / 64 : 1;
    o.len_shift = block_shift(blk->block);
    o.radius = nullptr;
    return o;
}

int64_t view_capacity(const dashkv_ctx *ctx, const dashkv_kv_view *kv) {
    return ctx->cfg.page_size ? (int64_t)kv->max_pages * ctx->cfg.page_size : kv->n_cap;
}

// ---- workspace: [scores | cand | ckey | hist | state | arrive(3 x BH lines) | seg_cnt | partials | block ids |
// per-sequence arrival lines]
struct WsLayout {
    size_t scores, cand, ckey, hist, state, arrive, seg_cnt, part, blk, seqarr, total;
};

size_t align_up(size_t x) { return (x + 255) & ~(size_t)255; }

// Internal score / candidate rows are padded to a multiple of 64 tokens.
int64_t row_ld(int64_t max_tokens) { return (max_tokens + 63) / 64 * 64; }

WsLayout ws_layout(const dashkv_config &c, int64_t max_tokens) {
    const size_t BH = (size_t)c.batch * c.num_kv_heads;
    const size_t G = (size_t)(c.num_q_heads / c.num_kv_heads);
    const size_t ld = (size_t)row_ld(max_tokens);
    WsLayout L;
    size_t o = 0;
    L.scores = o;  o = align_up(o + BH * ld * 4);
    L.cand = o;    o = align_up(o + BH * ld * 4);
    L.ckey = o;    o = align_up(o + BH * ld * 4);
    L.hist = o;    o = align_up(o + BH * kBins * 4);
    L.state = o;   o = align_up(o + BH * sizeof(SelState));
    L.arrive = o;  o = align_up(o + 3 * BH * kSyncStride * 4);
    L.seg_cnt = o; o = align_up(o + BH * kMaxSelCtas * 4);
    L.part = o;    o = align_up(o + BH * kMaxSplits * G * (c.head_dim + 2) * 4);
    L.blk = o;     o = align_up(o + BH * ((size_t)c.topk + 1) * 4);  // selected block ids + counts
    L.seqarr = o;  o = align_up(o + (size_t)c.batch * kSyncStride * 4);  // decode step: clusters done with a length
    L.total = o;
    return L;
}

// Launch with programmatic stream serialization: the kernel may be scheduled
// while its predecessor drains; it synchronises itself with griddep_wait().
template <typename... KArgs, typename... Args>
void launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

dashkv_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? DASHKV_OK : DASHKV_ERR_CUDA;
}

// CTAs per (b, kv head) for a kernel with `per_sm` resident CTAs per SM.
int sel_ctas(const dashkv_ctx *ctx, int64_t cap, int per_sm) {
    const int BH = ctx->cfg.batch * ctx->cfg.num_kv_heads;
    int n = (per_sm * ctx->sm_count) / BH;
    if (n < 1) n = 1;
    const int64_t by_tokens = ceil_div(cap, 1024);
    if (n > by_tokens) n = (int)by_tokens;
    if (n > kMaxSelCtas) n = kMaxSelCtas;
    return n < 1 ? 1 : n;
}

int attn_splits(const dashkv_ctx *ctx) {
    const int BH = ctx->cfg.batch * ctx->cfg.num_kv_heads;
    const int64_t cap_sel = (int64_t)ctx->cfg.topk + ctx->cfg.sink + ctx->cfg.window;
    int64_t n = (2 * ctx->sm_count) / BH;  // one wave of two CTAs per SM
    const int64_t by_rows = ceil_div(cap_sel, 64);
    if (n > by_rows) n = by_rows;
    if (n > kMaxSplits - 1) n = kMaxSplits - 1;  // at least one slot stays for a window CTA
    return n < 1 ? 1 : (int)n;
}

// ---- template dispatch
// The scorer places its LUT at the first 64 KB boundary above its low region;
// that needs the static shared memory (plus the 1 KB the system reserves) to
// leave room for the low region below 64 KB.
template <int BITS, int D>
bool score_layout_ok() {
    cudaFuncAttributes a[2];
    cudaFuncGetAttributes(&a[0], score_hist_kernel<BITS, D, false>);
    cudaFuncGetAttributes(&a[1], score_hist_kernel<BITS, D, true>);
    for (auto &x : a)
        if (x.sharedSizeBytes + 1024 + ScoreShape<BITS>::LOW_BYTES > 65536) return false;
    return true;
}

// ---- the clustered step kernel (instantiated in step_inst.cu)
StepKern step_kern(int bits, int d, int G, bool paged, bool radius) {
    if (d == 64) {
        if (bits == 32) return step_kern_32_64(G, paged, radius);
        if (bits == 64) return step_kern_64_64(G, paged, radius);
        return step_kern_128_64(G, paged, radius);
    }
    if (bits == 32) return step_kern_32_128(G, paged, radius);
    if (bits == 64) return step_kern_64_128(G, paged, radius);
    return step_kern_128_128(G, paged, radius);
}

// Dynamic shared memory of the context's step kernels (the device's per-block
// opt-in maximum minus their static part; the kernels lay out what they get),
// with the attributes their launches need; 0 when a kernel cannot get enough.
int setup_step_kernels(const dashkv_ctx *c) {
    int optin = 0;
    if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, c->device) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    const int G = c->cfg.num_q_heads / c->cfg.num_kv_heads;
    int smem = optin;
    StepKern ks[6];
    int nk = 0;
    for (int paged = 0; paged < 2; ++paged) {
        ks[nk++] = step_kern(c->cfg.bits, c->cfg.head_dim, 0, paged, false);
        ks[nk++] = step_kern(c->cfg.bits, c->cfg.head_dim, 0, paged, true);
        ks[nk++] = step_kern(c->cfg.bits, c->cfg.head_dim, G, paged, false);
    }
    for (int i = 0; i < nk; ++i) {
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, ks[i]) != cudaSuccess) { cudaGetLastError(); return 0; }
        if (optin - (int)fa.sharedSizeBytes < smem) smem = optin - (int)fa.sharedSizeBytes;
    }
    // the layout needs the low region below the LUT's 64 KB boundary, the LUT, the
    // code ring and some candidate room above it
    const int code_b = c->cfg.bits >= 64 ? c->cfg.bits / 8 : 8;
    const int ring = kRingStages * kStreamWarps * 32 * (c->cfg.bits == 128 ? 2 : 4) * code_b;
    if (smem < 2 * 65536 + ring + 4096) return 0;
    for (int i = 0; i < nk; ++i) {
        cudaFuncSetAttribute(ks[i], cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        cudaFuncSetAttribute(ks[i], cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    }
    if (cudaGetLastError() != cudaSuccess) return 0;
    return smem;
}

template <int BITS, int D>
void set_attrs_bd() {
    cudaFuncSetAttribute(encode_keys_kernel<BITS, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)EncodeShape<BITS, D>::SMEM);
    cudaFuncSetAttribute(encode_blocks_kernel<BITS, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)EncodeShape<BITS, D>::SMEM);
    cudaFuncSetAttribute(score_hist_kernel<BITS, D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)ScoreShape<BITS>::SMEM);
    cudaFuncSetAttribute(score_hist_kernel<BITS, D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)ScoreShape<BITS>::SMEM);
    cudaFuncSetAttribute(select_fused_kernel<BITS, D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)ScoreShape<BITS>::SMEM);
    cudaFuncSetAttribute(select_fused_kernel<BITS, D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)ScoreShape<BITS>::SMEM);
    cudaFuncSetAttribute(select_fused_kernel<BITS, D, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)ScoreShape<BITS>::SMEM);
    cudaFuncSetAttribute(select_fused_kernel<BITS, D, true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)ScoreShape<BITS>::SMEM);
    cudaFuncSetAttribute(select_fused_kernel<BITS, D, false>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    cudaFuncSetAttribute(select_fused_kernel<BITS, D, true>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    cudaFuncSetAttribute(select_fused_kernel<BITS, D, false, true>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    cudaFuncSetAttribute(select_fused_kernel<BITS, D, true, true>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
}

template <int D, int G>
void set_attr_decode() {
    cudaFuncSetAttribute(sparse_decode_kernel<D, G, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)DecodeShape<D, G>::SMEM);
    cudaFuncSetAttribute(sparse_decode_kernel<D, G, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)(DecodeShape<D, G>::SMEM + DecodeShape<D, G>::EX_BYTES));
}

void set_attrs() {
    set_attr_decode<64, 1>();  set_attr_decode<64, 2>();  set_attr_decode<64, 4>();  set_attr_decode<64, 8>();
    set_attr_decode<128, 1>(); set_attr_decode<128, 2>(); set_attr_decode<128, 4>(); set_attr_decode<128, 8>();
    cudaFuncSetAttribute(collect_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(CollectSmem));
    set_attrs_bd<32, 64>();  set_attrs_bd<32, 128>();
    set_attrs_bd<64, 64>();  set_attrs_bd<64, 128>();
    set_attrs_bd<128, 64>(); set_attrs_bd<128, 128>();
}

template <int BITS, int D>
void launch_encode_bd(const dashkv_ctx *ctx, const KV &kv, const int32_t *seq_lens, cudaStream_t st) {
    using S = EncodeShape<BITS, D>;
    const int BH = ctx->cfg.batch * ctx->cfg.num_kv_heads;
    const int64_t tiles = ceil_div(kv.capacity(), S::KT);
    int64_t gx = ceil_div(8 * ctx->sm_count, BH);
    if (gx > tiles) gx = tiles;
    if (gx < 1) gx = 1;
    encode_keys_kernel<BITS, D><<<dim3((unsigned)gx, BH), S::THREADS, S::SMEM, st>>>(kv, seq_lens, ctx->R, tiles);
}

template <int D>
void launch_encode_d(const dashkv_ctx *ctx, const KV &kv, const int32_t *s, cudaStream_t st) {
    switch (ctx->cfg.bits) {
        case 32: launch_encode_bd<32, D>(ctx, kv, s, st); break;
        case 64: launch_encode_bd<64, D>(ctx, kv, s, st); break;
        default: launch_encode_bd<128, D>(ctx, kv, s, st); break;
    }
}

template <int BITS, int D>
void launch_append_bd(const dashkv_ctx *ctx, const KV &kv, const void *kn, const void *vn, int32_t *seq,
                      cudaStream_t st) {
    // one cluster of C CTAs per sequence (early start behind the preceding kernel)
    const int Hkv = ctx->cfg.num_kv_heads;
    int C = (Hkv * BITS + kAppendSpan - 1) / kAppendSpan;
    if (C > kAppendCluster) C = kAppendCluster;
    if (C > Hkv) C = Hkv;
    const int hpc = (Hkv + C - 1) / C;  // <= 1024 / BITS heads per CTA (Hkv * BITS <= 8 * 512)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C, ctx->cfg.batch);
    cfg.blockDim = dim3(hpc * BITS);
    cfg.dynamicSmemBytes = (size_t)hpc * (D * 4 + BITS / 8);
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaLaunchKernelEx(&cfg, append_keys_kernel<BITS, D>, kv, static_cast<const __nv_bfloat16 *>(kn),
                       static_cast<const __nv_bfloat16 *>(vn), seq, ctx->R, hpc);
}

template <int D>
void launch_append_d(const dashkv_ctx *ctx, const KV &kv, const void *kn, const void *vn, int32_t *seq,
                     cudaStream_t st) {
    switch (ctx->cfg.bits) {
        case 32: launch_append_bd<32, D>(ctx, kv, kn, vn, seq, st); break;
        case 64: launch_append_bd<64, D>(ctx, kv, kn, vn, seq, st); break;
        default: launch_append_bd<128, D>(ctx, kv, kn, vn, seq, st); break;
    }
}

// What one selection takes: k (top-k), S sinks, W window, the row length of
// sel_idx.  The token selection uses the context's values; the block selection
// takes k blocks and no sinks or window.
struct SelArgs {
    int topk, sink, window, cap_sel;
};

template <int BITS, int D>
void launch_score_bd(const dashkv_ctx *ctx, const KV &kv, const void *q, const int32_t *seq, const SelWS &ws,
                     int nctas, int topk, cudaStream_t st) {
    const int BH = ctx->cfg.batch * ctx->cfg.num_kv_heads;
    const int G = ctx->cfg.num_q_heads / ctx->cfg.num_kv_heads;
    auto kern = kv.page_size ? score_hist_kernel<BITS, D, true> : score_hist_kernel<BITS, D, false>;
    launch_pdl(kern, dim3(nctas, BH), dim3(kScoreThreads), ScoreShape<BITS>::SMEM, st, kv,
               static_cast<const __nv_bfloat16 *>(q), ctx->cfg.num_q_heads, G, seq, ctx->R, ws, topk, nctas);
}

// Fused selection whenever cluster launches are available (and not disabled).
bool use_fused(const dashkv_ctx *ctx) { return !ctx->force_two_kernel && ctx->cluster_max > 0; }

// CTAs per cluster for one call: at most the context's choice, and no more
// than one per 1024 tokens of capacity.
int fused_cluster(const dashkv_ctx *ctx, int64_t cap) {
    const int64_t by_tokens = ceil_div(cap, 1024);
    const int c = ctx->cluster_max < by_tokens ? ctx->cluster_max : (int)by_tokens;
    return c < 1 ? 1 : c;
}

// Largest cluster size C <= kMaxCluster for which all B * Hkv clusters of the
// step kernel are resident at once (one wave, one CTA per SM); 1 when even
// single CTAs need several waves; 0 without cluster launch support.
int pick_cluster(const dashkv_ctx *ctx) {
    int ok = 0;
    if (!ctx->step_smem || cudaDeviceGetAttribute(&ok, cudaDevAttrClusterLaunch, ctx->device) != cudaSuccess || !ok) {
        cudaGetLastError();
        return 0;
    }
    const StepKern kern = step_kern(ctx->cfg.bits, ctx->cfg.head_dim, 0, false, false);
    const int BH = ctx->cfg.batch * ctx->cfg.num_kv_heads;
    int c = ctx->sm_count / BH;
    if (c > kMaxCluster) c = kMaxCluster;
    for (; c > 1; --c) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(c, BH);
        cfg.blockDim = dim3(kStepThreads);
        cfg.dynamicSmemBytes = ctx->step_smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = c;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int nclusters = 0;
        if (cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg) == cudaSuccess && nclusters >= BH) break;
        cudaGetLastError();
    }
    return c < 1 ? 1 : c;
}

// The step kernel on a grid of (C, B * Hkv) CTAs in clusters of C (one
// cluster per (b, h)), allowed to start early behind the preceding kernel.
void launch_step(const dashkv_ctx *ctx, StepKern kern, int nctas, const StepArgs &args, cudaStream_t st) {
    const int BH = ctx->cfg.batch * ctx->cfg.num_kv_heads;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(nctas, BH);
    cfg.blockDim = dim3(kStepThreads);
    cfg.dynamicSmemBytes = ctx->step_smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = nctas;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaLaunchKernelEx(&cfg, kern, args, ctx->R);
}

// Arguments of a selection-only step launch over `kv` (token codes or block
// summaries).
StepArgs select_args(const dashkv_ctx *ctx, const KV &kv, const void *q, const int32_t *seq, const SelWS &ws,
                     const SelArgs &a, int32_t *sel_idx, int32_t *sel_cnt, float *scores, int64_t ld_out) {
    StepArgs s = {};
    s.kv = kv;
    s.q = static_cast<const __nv_bfloat16 *>(q);
    s.Hq = ctx->cfg.num_q_heads;
    s.G = ctx->cfg.num_q_heads / ctx->cfg.num_kv_heads;
    s.seq_lens = const_cast<int32_t *>(seq);  // not written without an append
    s.k_new = nullptr;
    s.v_new = nullptr;
    s.ws = ws;
    s.topk = a.topk;
    s.S = a.sink;
    s.W = a.window;
    s.cap_sel = a.cap_sel;
    s.sel_idx = sel_idx;
    s.sel_cnt = sel_cnt;
    s.scores_out = scores;
    s.ld_out = ld_out;
    s.out = nullptr;
    s.lse = nullptr;
    s.scale_log2 = 0.0f;
    s.seq_arrive = nullptr;
    s.smem_bytes = ctx->step_smem;
    return s;
}

template <int D>
void launch_score_d(const dashkv_ctx *ctx, const KV &kv, const void *q, const int32_t *seq, const SelWS &ws,
                    int nctas, int topk, cudaStream_t st) {
    switch (ctx->cfg.bits) {
        case 32: launch_score_bd<32, D>(ctx, kv, q, seq, ws, nctas, topk, st); break;
        case 64: launch_score_bd<64, D>(ctx, kv, q, seq, ws, nctas, topk, st); break;
        default: launch_score_bd<128, D>(ctx, kv, q, seq, ws, nctas, topk, st); break;
    }
}

// Window CTAs per (b, h) (leading rows of the decode grid) when the lengths
// are given and at least one per (b, h) fits on the SMs the fused selection
// leaves free (two decode CTAs per SM), so that they run while it streams: as
// many as make a window CTA's share of the sinks + window about a top-k
// split's, as long as all of them fit there.  0: no window CTAs.
int window_ctas(const dashkv_ctx *ctx, int64_t cap, const int32_t *seq_lens, int splits) {
    if (!seq_lens || !use_fused(ctx)) return 0;
    const int BH = ctx->cfg.batch * ctx->cfg.num_kv_heads;
    const int64_t sel_ctas = (int64_t)fused_cluster(ctx, cap) * BH;
    if (sel_ctas >= ctx->sm_count) return 0;
    const int64_t slots = 2 * (ctx->sm_count - sel_ctas);
    if (BH > slots) return 0;
    const int64_t per_split = ceil_div(ctx->cfg.topk, splits);
    int64_t nw = ceil_div((int64_t)ctx->cfg.sink + ctx->cfg.window, per_split);
    if (nw > slots / BH) nw = slots / BH;
    if (nw > kMaxSplits - splits) nw = kMaxSplits - splits;
    return nw < 1 ? 1 : (int)nw;
}

template <int D, int G>
void launch_decode_dg(const dashkv_ctx *ctx, const KV &kv, const void *q, const int32_t *si, const int32_t *sc,
                      float *out, float *lse, const AttnWS &ws, const int32_t *seq_lens, int64_t cap,
                      const Tiers *tiers, cudaStream_t st) {
    const int BH = ctx->cfg.batch * ctx->cfg.num_kv_heads;
    const int splits = attn_splits(ctx);
    const int nw = window_ctas(ctx, cap, seq_lens, splits);
    const int wy = (BH * nw + splits - 1) / splits;  // grid rows of window CTAs
    const int cap_sel = ctx->cfg.topk + ctx->cfg.sink + ctx->cfg.window;
    const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
    const Tiers tr = tiers ? *tiers : Tiers{};
    const size_t smem = DecodeShape<D, G>::SMEM + (tiers ? DecodeShape<D, G>::EX_BYTES : 0);
    launch_pdl(tiers ? sparse_decode_kernel<D, G, true> : sparse_decode_kernel<D, G, false>, dim3(splits, BH + wy),
               dim3(kAttnThreads), smem, st, kv, static_cast<const __nv_bfloat16 *>(q),
               ctx->cfg.num_q_heads, si, sc, cap_sel, out, lse, ws, splits, scale_log2, seq_lens, ctx->cfg.sink,
               ctx->cfg.window, ctx->cfg.topk, wy, nw > 0 ? nw : 1, tr);
}

template <int D>
void launch_decode_d(const dashkv_ctx *ctx, const KV &kv, const void *q, const int32_t *si, const int32_t *sc,
                     float *out, float *lse, const AttnWS &ws, const int32_t *seq, int64_t cap, const Tiers *tiers,
                     cudaStream_t st) {
    switch (ctx->cfg.num_q_heads / ctx->cfg.num_kv_heads) {
        case 1: launch_decode_dg<D, 1>(ctx, kv, q, si, sc, out, lse, ws, seq, cap, tiers, st); break;
        case 2: launch_decode_dg<D, 2>(ctx, kv, q, si, sc, out, lse, ws, seq, cap, tiers, st); break;
        case 4: launch_decode_dg<D, 4>(ctx, kv, q, si, sc, out, lse, ws, seq, cap, tiers, st); break;
        default: launch_decode_dg<D, 8>(ctx, kv, q, si, sc, out, lse, ws, seq, cap, tiers, st); break;
    }
}


// The selection's view of a workspace laid out by L for rows of `cap` tokens.
SelWS carve_selws(const WsLayout &L, char *w, int64_t cap, float *scores) {
    SelWS ws;
    ws.scores = reinterpret_cast<float *>(w + L.scores);
    ws.ld = row_ld(cap);
    ws.scores_out = scores;
    ws.ld_out = cap;
    ws.cand = reinterpret_cast<int32_t *>(w + L.cand);
    ws.ckey = reinterpret_cast<uint32_t *>(w + L.ckey);
    ws.hist = reinterpret_cast<uint32_t *>(w + L.hist);
    ws.state = reinterpret_cast<SelState *>(w + L.state);
    ws.arrive = reinterpret_cast<uint32_t *>(w + L.arrive);
    ws.seg_cnt = reinterpret_cast<int32_t *>(w + L.seg_cnt);
    return ws;
}

// Fused selection: a grid of (C, B * Hkv) CTAs in clusters of C (one cluster
// per (b, h)) that may also start early behind the preceding kernel.
template <int BITS, int D>
void launch_fused_bd(const dashkv_ctx *ctx, const KV &kv, const void *q, const int32_t *seq, const SelWS &ws,
                     int nctas, const SelArgs &a, int32_t *sel_idx, int32_t *sel_cnt, cudaStream_t st) {
    const int BH = ctx->cfg.batch * ctx->cfg.num_kv_heads;
    const int G = ctx->cfg.num_q_heads / ctx->cfg.num_kv_heads;
    auto kern = kv.radius ? (kv.page_size ? select_fused_kernel<BITS, D, true, true>
                                          : select_fused_kernel<BITS, D, false, true>)
                          : (kv.page_size ? select_fused_kernel<BITS, D, true> : select_fused_kernel<BITS, D, false>);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(nctas, BH);
    cfg.blockDim = dim3(kScoreThreads);
    cfg.dynamicSmemBytes = ScoreShape<BITS>::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = nctas;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaLaunchKernelEx(&cfg, kern, kv, static_cast<const __nv_bfloat16 *>(q), ctx->cfg.num_q_heads, G, seq, ctx->R,
                       ws, a.topk, a.sink, a.window, a.cap_sel, sel_idx, sel_cnt);
}

template <int D>
void launch_fused_d(const dashkv_ctx *ctx, const KV &kv, const void *q, const int32_t *seq, const SelWS &ws,
                    int nctas, const SelArgs &a, int32_t *si, int32_t *sc, cudaStream_t st) {
    switch (ctx->cfg.bits) {
        case 32: launch_fused_bd<32, D>(ctx, kv, q, seq, ws, nctas, a, si, sc, st); break;
        case 64: launch_fused_bd<64, D>(ctx, kv, q, seq, ws, nctas, a, si, sc, st); break;
        default: launch_fused_bd<128, D>(ctx, kv, q, seq, ws, nctas, a, si, sc, st); break;
    }
}

// One selection over `k` (the token cache, or the block codes): the fused
// clustered selection, or score + collect, followed by the optional copy of the
// scores (rows of length cap).  The workspace is carved as L lays it out.
void run_select(const dashkv_ctx *ctx, const KV &k, int64_t cap, const WsLayout &L, char *w, const void *q,
                const int32_t *seq_lens, const SelArgs &a, int32_t *sel_idx, int32_t *sel_cnt, float *scores,
                Tracer &tr, cudaStream_t st) {
    const int BH = ctx->cfg.batch * ctx->cfg.num_kv_heads;
    const SelWS ws = carve_selws(L, w, cap, scores);
    const int nscore = sel_ctas(ctx, cap, 1);    // score kernel: one 1024-thread CTA per SM
    const int ncollect = sel_ctas(ctx, cap, 2);  // collect kernel: two 512-thread CTAs per SM
    auto copy_scores = [&]() {
        if (!scores) return;
        const int gx = (int)((cap + 255) / 256 < 64 ? (cap + 255) / 256 : 64);
        launch_pdl(copy_scores_kernel, dim3(gx > 0 ? gx : 1, BH), dim3(256), 0, st,
                   (const float *)ws.scores, ws.ld, scores, ws.ld_out, seq_lens, ctx->cfg.num_kv_heads, cap,
                   (int)k.len_shift);
    };
    if (use_fused(ctx)) {
        const int nc = fused_cluster(ctx, cap);
        tr.before();
        if (ctx->cfg.head_dim == 64) launch_fused_d<64>(ctx, k, q, seq_lens, ws, nc, a, sel_idx, sel_cnt, st);
        else launch_fused_d<128>(ctx, k, q, seq_lens, ws, nc, a, sel_idx, sel_cnt, st);
        tr.after();
        copy_scores();
        return;
    }
    tr.before();
    if (ctx->cfg.head_dim == 64) launch_score_d<64>(ctx, k, q, seq_lens, ws, nscore, a.topk, st);
    else launch_score_d<128>(ctx, k, q, seq_lens, ws, nscore, a.topk, st);
    tr.after();
    tr.before();
    launch_pdl(collect_kernel, dim3(ncollect, BH), dim3(kSelThreads), sizeof(CollectSmem), st, ws, ncollect, a.sink,
               a.window, a.cap_sel, sel_idx, sel_cnt);
    tr.after();
    copy_scores();
}

// ---- block summaries
template <int BITS, int D>
void launch_encode_blocks_bd(const dashkv_ctx *ctx, const KV &kv, const KV &blk, const int32_t *seq_lens,
                             cudaStream_t st) {
    using S = EncodeShape<BITS, D>;
    const int BH = ctx->cfg.batch * ctx->cfg.num_kv_heads;
    const int64_t tiles = ceil_div(blk.n_cap, S::KT);
    int64_t gx = ceil_div(8 * ctx->sm_count, BH);
    if (gx > tiles) gx = tiles;
    if (gx < 1) gx = 1;
    encode_blocks_kernel<BITS, D><<<dim3((unsigned)gx, BH), S::THREADS, S::SMEM, st>>>(kv, blk, seq_lens, ctx->R,
                                                                                      tiles);
}

template <int BITS, int D>
void launch_append_blocks_bd(const dashkv_ctx *ctx, const KV &kv, const KV &blk, const int32_t *seq_lens,
                             cudaStream_t st) {
    const int Hkv = ctx->cfg.num_kv_heads;
    const int C = (Hkv * BITS + 1023) / 1024;  // CTAs per sequence
    const int hpc = (Hkv + C - 1) / C;         // heads per CTA: hpc * BITS <= 1024
    launch_pdl(append_blocks_kernel<BITS, D>, dim3(C, ctx->cfg.batch), dim3(hpc * BITS),
               (size_t)hpc * (D * 4 + BITS / 8), st, kv, blk, seq_lens, ctx->R, hpc);
}

template <int D>
void launch_radius_d(const dashkv_ctx *ctx, bool whole, const KV &kv, const int32_t *seq_lens, uint8_t *out,
                     cudaStream_t st) {
    const int BH = ctx->cfg.batch * ctx->cfg.num_kv_heads;
    if (whole) {
        int64_t gx = ceil_div(kv.capacity(), kRadiusThreads);
        const int64_t cap_x = ceil_div(8 * ctx->sm_count, BH);
        if (gx > cap_x) gx = cap_x;
        if (gx < 1) gx = 1;
        radius_codes_kernel<D><<<dim3((unsigned)gx, BH), kRadiusThreads, 0, st>>>(kv, seq_lens, out);
    } else {
        launch_pdl(append_radius_kernel<D>, dim3(ctx->cfg.batch), dim3(32), 0, st, kv, seq_lens, out);
    }
}

template <int D>
void launch_blocks_d(const dashkv_ctx *ctx, bool whole, const KV &kv, const KV &blk, const int32_t *s,
                     cudaStream_t st) {
    switch (ctx->cfg.bits) {
        case 32: whole ? launch_encode_blocks_bd<32, D>(ctx, kv, blk, s, st) : launch_append_blocks_bd<32, D>(ctx, kv, blk, s, st); break;
        case 64: whole ? launch_encode_blocks_bd<64, D>(ctx, kv, blk, s, st) : launch_append_blocks_bd<64, D>(ctx, kv, blk, s, st); break;
        default: whole ? launch_encode_blocks_bd<128, D>(ctx, kv, blk, s, st) : launch_append_blocks_bd<128, D>(ctx, kv, blk, s, st); break;
    }
}
}  // namespace

// ---------------------------------------------------------------------------- static scratch
// Scratch of dashkv_select_static: one fixed array in this library's device
// image (per device), for callers that may not allocate device memory.  No
// call here allocates: the address comes from cudaGetSymbolAddress.
constexpr size_t kStaticScratchBytes = (size_t)24 << 20;  // 24 MiB
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

namespace {
constexpr int kMaxStaticDevices = 64;
// Per device: the scratch's device address (once set up) and the regions of
// the last selection layout whose counter words are known to be zero.  The
// histogram and arrival words sit at offsets that depend on B * Hkv and the
// capacity, so a call with another layout may find rows an earlier call left
// there; those words are zeroed again (on the call's stream) whenever the
// layout changes or after a call that failed.
struct StaticScratch {
    void *addr;
    size_t hist_off, hist_bytes, arrive_off, arrive_bytes;  // all 0: nothing known to be zero
};
StaticScratch g_static[kMaxStaticDevices];
std::mutex g_static_mu;

// First use on a device: look the scratch up and zero it whole.  The memset
// and the device synchronisation cannot be captured, so this refuses to run
// while `st` is capturing.  The caller holds g_static_mu.
dashkv_status static_scratch_setup(int dev, cudaStream_t st) {
    if (g_static[dev].addr) return DASHKV_OK;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return DASHKV_ERR_CUDA;
    if (cs != cudaStreamCaptureStatusNone) return DASHKV_ERR_INVALID_ARG;
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return DASHKV_ERR_CUDA;
    if (cudaMemset(p, 0, kStaticScratchBytes) != cudaSuccess) return DASHKV_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return DASHKV_ERR_CUDA;
    g_static[dev] = StaticScratch{p, 0, 0, 0, 0};
    return DASHKV_OK;
}

// Make the counter words of layout L zero before a selection on `st`: nothing
// to do when the previous successful call used the same regions (it left them
// zero); otherwise they are cleared with stream-ordered (capturable) memsets.
// Under capture the record is not updated, since the graph may never run.
dashkv_status static_scratch_prepare(int dev, const WsLayout &L, size_t hist_bytes, size_t arrive_bytes,
                                     cudaStream_t st) {
    StaticScratch &s = g_static[dev];
    if (s.hist_off == L.hist && s.hist_bytes == hist_bytes && s.arrive_off == L.arrive &&
        s.arrive_bytes == arrive_bytes)
        return DASHKV_OK;
    char *w = static_cast<char *>(s.addr);
    if (cudaMemsetAsync(w + L.hist, 0, hist_bytes, st) != cudaSuccess) return DASHKV_ERR_CUDA;
    if (cudaMemsetAsync(w + L.arrive, 0, arrive_bytes, st) != cudaSuccess) return DASHKV_ERR_CUDA;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return DASHKV_ERR_CUDA;
    if (cs == cudaStreamCaptureStatusNone) {
        s.hist_off = L.hist;
        s.hist_bytes = hist_bytes;
        s.arrive_off = L.arrive;
        s.arrive_bytes = arrive_bytes;
    }
    return DASHKV_OK;
}

// After a failed call nothing is known about the counter words any more.
void static_scratch_forget(int dev) {
    StaticScratch &s = g_static[dev];
    s.hist_off = s.hist_bytes = s.arrive_off = s.arrive_bytes = 0;
}

// Tier view of a paged cache (tiers.cuh): all four arrays, FP8 rows 16-byte
// aligned, exponents 4-byte aligned (the decode copies them in 4-byte words).
dashkv_status check_tiers(const dashkv_ctx *ctx, const dashkv_tier_view *tv) {
    if (!tv || !tv->tier || !tv->k8 || !tv->v8 || !tv->exps) return DASHKV_ERR_INVALID_ARG;
    if (!ctx->cfg.page_size) return DASHKV_ERR_UNSUPPORTED;  // tiers are per page
    if (!aligned(tv->k8, 16) || !aligned(tv->v8, 16) || !aligned(tv->exps, 4)) return DASHKV_ERR_INVALID_ARG;
    return DASHKV_OK;
}

Tiers make_tiers(const dashkv_tier_view *tv) {
    Tiers t;
    t.tier = tv->tier;
    t.k8 = tv->k8;
    t.v8 = tv->v8;
    t.exps = tv->exps;
    return t;
}

// dashkv_sparse_decode, with FP8 rows for the tier-1 pages when `tiers` is set.
dashkv_status run_decode(dashkv_ctx *ctx, const dashkv_kv_view *kv, const Tiers *tiers, const void *q,
                         const int32_t *seq_lens, const int32_t *sel_idx, const int32_t *sel_cnt, float *out,
                         float *lse, void *workspace, size_t workspace_bytes, void *stream) {
    if (!ctx || !q || !sel_idx || !sel_cnt || !out || !aligned(q, 16)) return DASHKV_ERR_INVALID_ARG;
    dashkv_status s = check_view(ctx, kv, true, false);
    if (s != DASHKV_OK) return s;
    const WsLayout L = ws_layout(ctx->cfg, view_capacity(ctx, kv));
    if (!workspace || workspace_bytes < L.total || !aligned(workspace, 256)) return DASHKV_ERR_WORKSPACE;
    char *w = static_cast<char *>(workspace);
    const int BH = ctx->cfg.batch * ctx->cfg.num_kv_heads;
    AttnWS ws;
    ws.part = reinterpret_cast<float *>(w + L.part);
    ws.arrive = reinterpret_cast<uint32_t *>(w + L.arrive) + 2 * BH * kSyncStride;
    const KV k = make_kv(ctx, kv);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Tracer tr(ctx, st);
    tr.before();
    const int64_t cap = view_capacity(ctx, kv);
    if (ctx->cfg.head_dim == 64)
        launch_decode_d<64>(ctx, k, q, sel_idx, sel_cnt, out, lse, ws, seq_lens, cap, tiers, st);
    else
        launch_decode_d<128>(ctx, k, q, sel_idx, sel_cnt, out, lse, ws, seq_lens, cap, tiers, st);
    tr.after();
    return launch_status();
}

}  // namespace

// ============================================================================ C ABI
extern "C" {

const char *dashkv_status_str(dashkv_status s) {
    switch (s) {
        case DASHKV_OK: return "ok";
        case DASHKV_ERR_INVALID_ARG: return "invalid argument";
        case DASHKV_ERR_UNSUPPORTED: return "unsupported configuration";
        case DASHKV_ERR_WORKSPACE: return "workspace missing or too small";
        case DASHKV_ERR_CAPACITY: return "sequence length beyond cache capacity";
        case DASHKV_ERR_CUDA: return "CUDA error";
        case DASHKV_ERR_DEVICE: return "page id out of range";
        case DASHKV_ERR_NO_DEVICE: return "no CUDA device";
        case DASHKV_ERR_TIMEOUT: return "a bounded wait in a kernel gave up";
    }
    return "unknown status";
}

dashkv_status dashkv_hyperplanes(uint64_t seed, int32_t bits, int32_t d, int8_t *host_out) {
    if (!host_out || bits <= 0 || d <= 0 || bits > kMaxBits || d > kMaxDim || d % 32) return DASHKV_ERR_INVALID_ARG;
    RBits R;
    build_rbits(seed, bits, d, &R);
    for (int j = 0; j < bits; ++j)
        for (int i = 0; i < d; ++i) host_out[j * d + i] = ((R.w[j * (d / 32) + i / 32] >> (i % 32)) & 1u) ? -1 : 1;
    return DASHKV_OK;
}

dashkv_status dashkv_create(const dashkv_config *cfg, dashkv_ctx **out) {
    if (!out) return DASHKV_ERR_INVALID_ARG;
    *out = nullptr;
    dashkv_status st = check_config(cfg);
    if (st != DASHKV_OK) return st;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return DASHKV_ERR_NO_DEVICE;
    }
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        sms = kSmCountFallback;
    dashkv_ctx *c = static_cast<dashkv_ctx *>(calloc(1, sizeof(dashkv_ctx)));
    if (!c) return DASHKV_ERR_INVALID_ARG;
    c->cfg = *cfg;
    c->device = dev;
    c->sm_count = sms;
    c->force_two_kernel = (cfg->flags & DASHKV_FLAG_TWO_KERNEL_SELECT) != 0;
    build_rbits(cfg->seed, cfg->bits, cfg->head_dim, &c->R);
    set_attrs();
    c->step_smem = setup_step_kernels(c);
    c->cluster_max = pick_cluster(c);
    const bool layout_ok =
        cfg->head_dim == 64
            ? (cfg->bits == 32 ? score_layout_ok<32, 64>() : cfg->bits == 64 ? score_layout_ok<64, 64>() : score_layout_ok<128, 64>())
            : (cfg->bits == 32 ? score_layout_ok<32, 128>() : cfg->bits == 64 ? score_layout_ok<64, 128>() : score_layout_ok<128, 128>());
    if (!layout_ok) {
        free(c);
        return DASHKV_ERR_UNSUPPORTED;
    }
    if (cudaGetLastError() != cudaSuccess) {
        free(c);
        return DASHKV_ERR_CUDA;
    }
    *out = c;
    return DASHKV_OK;
}

void dashkv_destroy(dashkv_ctx *ctx) { free(ctx); }

size_t dashkv_workspace_size(const dashkv_ctx *ctx, int64_t max_tokens) {
    if (!ctx || max_tokens < 0) return 0;
    return ws_layout(ctx->cfg, max_tokens).total;
}

dashkv_status dashkv_encode_keys(dashkv_ctx *ctx, const dashkv_kv_view *kv, const int32_t *seq_lens, void *stream) {
    if (!ctx || !seq_lens) return DASHKV_ERR_INVALID_ARG;
    dashkv_status s = check_view(ctx, kv, true, true);
    if (s != DASHKV_OK) return s;
    const KV k = make_kv(ctx, kv);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Tracer tr(ctx, st);
    tr.before();
    if (ctx->cfg.head_dim == 64) launch_encode_d<64>(ctx, k, seq_lens, st);
    else launch_encode_d<128>(ctx, k, seq_lens, st);
    tr.after();
    return launch_status();
}

dashkv_status dashkv_append_keys(dashkv_ctx *ctx, const dashkv_kv_view *kv, const void *k_new, const void *v_new,
                                 int32_t *seq_lens, void *stream) {
    if (!ctx || !seq_lens || !k_new || !v_new || !aligned(k_new, 16) || !aligned(v_new, 16))
        return DASHKV_ERR_INVALID_ARG;
    dashkv_status s = check_view(ctx, kv, true, true);
    if (s != DASHKV_OK) return s;
    const KV k = make_kv(ctx, kv);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Tracer tr(ctx, st);
    tr.before();
    if (ctx->cfg.head_dim == 64) launch_append_d<64>(ctx, k, k_new, v_new, seq_lens, st);
    else launch_append_d<128>(ctx, k, k_new, v_new, seq_lens, st);
    tr.after();
    return launch_status();
}

dashkv_status dashkv_select(dashkv_ctx *ctx, const dashkv_kv_view *kv, const void *q, const int32_t *seq_lens,
                            int32_t *sel_idx, int32_t *sel_cnt, float *scores, void *workspace,
                            size_t workspace_bytes, void *stream) {
    if (!ctx || !q || !seq_lens || !sel_idx || !sel_cnt || !aligned(q, 16)) return DASHKV_ERR_INVALID_ARG;
    dashkv_status s = check_view(ctx, kv, false, true);
    if (s != DASHKV_OK) return s;
    const int64_t cap = view_capacity(ctx, kv);
    const WsLayout L = ws_layout(ctx->cfg, cap);
    if (!workspace || workspace_bytes < L.total || !aligned(workspace, 256)) return DASHKV_ERR_WORKSPACE;
    const SelArgs a{ctx->cfg.topk, ctx->cfg.sink, ctx->cfg.window,
                    ctx->cfg.topk + ctx->cfg.sink + ctx->cfg.window};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Tracer tr(ctx, st);
    run_select(ctx, make_kv(ctx, kv), cap, L, static_cast<char *>(workspace), q, seq_lens, a, sel_idx, sel_cnt,
               scores, tr, st);
    return launch_status();
}

// dashkv_select on the library's static scratch (see StaticScratch above):
// for callers that cannot allocate the workspace themselves.
dashkv_status dashkv_select_static(dashkv_ctx *ctx, const dashkv_kv_view *kv, const void *q,
                                   const int32_t *seq_lens, int32_t *sel_idx, int32_t *sel_cnt, float *scores,
                                   void *stream) {
    if (!ctx) return DASHKV_ERR_INVALID_ARG;
    const dashkv_status v = check_view(ctx, kv, false, true);
    if (v != DASHKV_OK) return v;
    const WsLayout L = ws_layout(ctx->cfg, view_capacity(ctx, kv));
    if (L.total > kStaticScratchBytes) return DASHKV_ERR_WORKSPACE;
    // the scratch address belongs to the current device: it must be the context's
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return DASHKV_ERR_CUDA;
    if (cur != ctx->device) return DASHKV_ERR_INVALID_ARG;
    if (cur < 0 || cur >= kMaxStaticDevices) return DASHKV_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t BH = (size_t)ctx->cfg.batch * ctx->cfg.num_kv_heads;
    std::lock_guard<std::mutex> lock(g_static_mu);
    dashkv_status s = static_scratch_setup(cur, st);
    if (s == DASHKV_OK) s = static_scratch_prepare(cur, L, BH * kBins * 4, 3 * BH * kSyncStride * 4, st);
    if (s == DASHKV_OK)
        s = dashkv_select(ctx, kv, q, seq_lens, sel_idx, sel_cnt, scores, g_static[cur].addr, kStaticScratchBytes,
                          stream);
    if (s != DASHKV_OK && g_static[cur].addr) static_scratch_forget(cur);
    return s;
}

dashkv_status dashkv_sparse_decode(dashkv_ctx *ctx, const dashkv_kv_view *kv, const void *q,
                                   const int32_t *seq_lens, const int32_t *sel_idx, const int32_t *sel_cnt,
                                   float *out, float *lse, void *workspace, size_t workspace_bytes,
                                   void *stream) {
    return run_decode(ctx, kv, nullptr, q, seq_lens, sel_idx, sel_cnt, out, lse, workspace, workspace_bytes,
                      stream);
}

dashkv_status dashkv_demote_pages(dashkv_ctx *ctx, const dashkv_kv_view *kv, const dashkv_tier_view *tv,
                                  const int32_t *seq_lens, const uint8_t *protect, void *stream) {
    if (!ctx || !seq_lens) return DASHKV_ERR_INVALID_ARG;
    dashkv_status s = check_view(ctx, kv, true, false);
    if (s == DASHKV_OK) s = check_tiers(ctx, tv);
    if (s != DASHKV_OK) return s;
    const KV k = make_kv(ctx, kv);
    const Tiers tr = make_tiers(tv);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Tracer trc(ctx, st);
    trc.before();
    const dim3 grid((unsigned)kv->max_pages, (unsigned)ctx->cfg.batch);
    if (ctx->cfg.head_dim == 64)
        demote_pages_kernel<64><<<grid, kDemoteThreads, 0, st>>>(k, tr, protect, seq_lens, ctx->cfg.sink,
                                                                 ctx->cfg.window);
    else
        demote_pages_kernel<128><<<grid, kDemoteThreads, 0, st>>>(k, tr, protect, seq_lens, ctx->cfg.sink,
                                                                  ctx->cfg.window);
    trc.after();
    return launch_status();
}

dashkv_status dashkv_sparse_decode_tiered(dashkv_ctx *ctx, const dashkv_kv_view *kv, const dashkv_tier_view *tv,
                                          const void *q, const int32_t *seq_lens, const int32_t *sel_idx,
                                          const int32_t *sel_cnt, float *out, float *lse, void *workspace,
                                          size_t workspace_bytes, void *stream) {
    if (!ctx) return DASHKV_ERR_INVALID_ARG;
    const dashkv_status s = check_tiers(ctx, tv);
    if (s != DASHKV_OK) return s;
    const Tiers tr = make_tiers(tv);
    return run_decode(ctx, kv, &tr, q, seq_lens, sel_idx, sel_cnt, out, lse, workspace, workspace_bytes, stream);
}

dashkv_status dashkv_decode_step(dashkv_ctx *ctx, const dashkv_kv_view *kv, const void *q, const void *k_new,
                                 const void *v_new, int32_t *seq_lens, int32_t *sel_idx, int32_t *sel_cnt,
                                 float *out, float *lse, void *workspace, size_t workspace_bytes, void *stream) {
    if (!ctx || !q || !k_new || !v_new || !seq_lens || !sel_idx || !sel_cnt || !out || !aligned(q, 16) ||
        !aligned(k_new, 16) || !aligned(v_new, 16))
        return DASHKV_ERR_INVALID_ARG;
    dashkv_status s = check_view(ctx, kv, true, true);
    if (s != DASHKV_OK) return s;
    const int64_t cap = view_capacity(ctx, kv);
    const WsLayout L = ws_layout(ctx->cfg, cap);
    if (!workspace || workspace_bytes < L.total || !aligned(workspace, 256)) return DASHKV_ERR_WORKSPACE;
    if (!use_fused(ctx)) {  // the three calls, one after the other
        s = dashkv_append_keys(ctx, kv, k_new, v_new, seq_lens, stream);
        if (s == DASHKV_OK)
            s = dashkv_select(ctx, kv, q, seq_lens, sel_idx, sel_cnt, nullptr, workspace, workspace_bytes, stream);
        if (s == DASHKV_OK)
            s = dashkv_sparse_decode(ctx, kv, q, seq_lens, sel_idx, sel_cnt, out, lse, workspace, workspace_bytes,
                                     stream);
        return s;
    }
    char *w = static_cast<char *>(workspace);
    const SelArgs a{ctx->cfg.topk, ctx->cfg.sink, ctx->cfg.window, ctx->cfg.topk + ctx->cfg.sink + ctx->cfg.window};
    StepArgs args = select_args(ctx, make_kv(ctx, kv), q, seq_lens, carve_selws(L, w, cap, nullptr), a, sel_idx,
                                sel_cnt, nullptr, cap);
    args.k_new = static_cast<const __nv_bfloat16 *>(k_new);
    args.v_new = static_cast<const __nv_bfloat16 *>(v_new);
    args.out = out;
    args.lse = lse;
    args.scale_log2 = (float)(1.4426950408889634 / sqrt((double)ctx->cfg.head_dim));
    args.seq_arrive = reinterpret_cast<uint32_t *>(w + L.seqarr);
    const int G = ctx->cfg.num_q_heads / ctx->cfg.num_kv_heads;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Tracer tr(ctx, st);
    tr.before();
    launch_step(ctx, step_kern(ctx->cfg.bits, ctx->cfg.head_dim, G, ctx->cfg.page_size != 0, false),
                fused_cluster(ctx, cap), args, st);
    tr.after();
    return launch_status();
}

dashkv_status dashkv_encode_blocks(dashkv_ctx *ctx, const dashkv_kv_view *kv, const dashkv_block_view *blk,
                                   const int32_t *seq_lens, void *stream) {
    if (!ctx || !seq_lens) return DASHKV_ERR_INVALID_ARG;
    dashkv_status s = check_view(ctx, kv, true, false);
    if (s == DASHKV_OK) s = check_blocks(ctx, kv, blk);
    if (s != DASHKV_OK) return s;
    const KV k = make_kv(ctx, kv), b = make_blk(ctx, blk);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Tracer tr(ctx, st);
    tr.before();
    if (ctx->cfg.head_dim == 64) launch_blocks_d<64>(ctx, true, k, b, seq_lens, st);
    else launch_blocks_d<128>(ctx, true, k, b, seq_lens, st);
    tr.after();
    return launch_status();
}

dashkv_status dashkv_append_blocks(dashkv_ctx *ctx, const dashkv_kv_view *kv, const dashkv_block_view *blk,
                                   const int32_t *seq_lens, void *stream) {
    if (!ctx || !seq_lens) return DASHKV_ERR_INVALID_ARG;
    dashkv_status s = check_view(ctx, kv, true, false);
    if (s == DASHKV_OK) s = check_blocks(ctx, kv, blk);
    if (s != DASHKV_OK) return s;
    const KV k = make_kv(ctx, kv), b = make_blk(ctx, blk);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Tracer tr(ctx, st);
    tr.before();
    if (ctx->cfg.head_dim == 64) launch_blocks_d<64>(ctx, false, k, b, seq_lens, st);
    else launch_blocks_d<128>(ctx, false, k, b, seq_lens, st);
    tr.after();
    return launch_status();
}

dashkv_status dashkv_select_blocks(dashkv_ctx *ctx, const dashkv_kv_view *kv, const dashkv_block_view *blk,
                                   const void *q, const int32_t *seq_lens, int32_t *sel_idx, int32_t *sel_cnt,
                                   float *block_scores, void *workspace, size_t workspace_bytes, void *stream) {
    if (!ctx || !q || !seq_lens || !sel_idx || !sel_cnt || !aligned(q, 16)) return DASHKV_ERR_INVALID_ARG;
    dashkv_status s = check_view(ctx, kv, false, false);
    if (s == DASHKV_OK) s = check_blocks(ctx, kv, blk);
    if (s != DASHKV_OK) return s;
    const int shift = block_shift(blk->block);
    const int kb = ctx->cfg.topk >> shift;  // blocks whose tokens fill the top-k budget
    if (kb < 1 || ctx->cfg.window < blk->block - 1) return DASHKV_ERR_UNSUPPORTED;
    const int64_t cap = view_capacity(ctx, kv);
    const WsLayout L = ws_layout(ctx->cfg, cap);
    if (!workspace || workspace_bytes < L.total || !aligned(workspace, 256)) return DASHKV_ERR_WORKSPACE;
    char *w = static_cast<char *>(workspace);
    const int BH = ctx->cfg.batch * ctx->cfg.num_kv_heads;
    int32_t *blk_idx = reinterpret_cast<int32_t *>(w + L.blk);
    int32_t *blk_cnt = blk_idx + (size_t)BH * kb;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Tracer tr(ctx, st);
    // top kb blocks by the score of their summary codes (no sinks, no window)
    run_select(ctx, make_blk(ctx, blk), blk->nb_cap, L, w, q, seq_lens, SelArgs{kb, 0, 0, kb}, blk_idx, blk_cnt,
               block_scores, tr, st);
    const int cap_sel = ctx->cfg.topk + ctx->cfg.sink + ctx->cfg.window;
    tr.before();
    launch_pdl(expand_blocks_kernel, dim3(BH), dim3(kExpandThreads), 0, st, (const int32_t *)blk_idx,
               (const int32_t *)blk_cnt, kb, seq_lens, cap, ctx->cfg.num_kv_heads, shift, ctx->cfg.sink,
               ctx->cfg.window, cap_sel, sel_idx, sel_cnt);
    tr.after();
    return launch_status();
}

dashkv_status dashkv_encode_radius(dashkv_ctx *ctx, const dashkv_kv_view *kv, const int32_t *seq_lens,
                                   uint8_t *radius, void *stream) {
    if (!ctx || !seq_lens || !radius) return DASHKV_ERR_INVALID_ARG;
    const dashkv_status s = check_view(ctx, kv, true, false);
    if (s != DASHKV_OK) return s;
    const KV k = make_kv(ctx, kv);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Tracer tr(ctx, st);
    tr.before();
    if (ctx->cfg.head_dim == 64) launch_radius_d<64>(ctx, true, k, seq_lens, radius, st);
    else launch_radius_d<128>(ctx, true, k, seq_lens, radius, st);
    tr.after();
    return launch_status();
}

dashkv_status dashkv_append_radius(dashkv_ctx *ctx, const dashkv_kv_view *kv, const int32_t *seq_lens,
                                   uint8_t *radius, void *stream) {
    if (!ctx || !seq_lens || !radius) return DASHKV_ERR_INVALID_ARG;
    const dashkv_status s = check_view(ctx, kv, true, false);
    if (s != DASHKV_OK) return s;
    const KV k = make_kv(ctx, kv);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Tracer tr(ctx, st);
    tr.before();
    if (ctx->cfg.head_dim == 64) launch_radius_d<64>(ctx, false, k, seq_lens, radius, st);
    else launch_radius_d<128>(ctx, false, k, seq_lens, radius, st);
    tr.after();
    return launch_status();
}

dashkv_status dashkv_select_radius(dashkv_ctx *ctx, const dashkv_kv_view *kv, const uint8_t *radius, const void *q,
                                   const int32_t *seq_lens, int32_t *sel_idx, int32_t *sel_cnt, float *scores,
                                   void *workspace, size_t workspace_bytes, void *stream) {
    if (!ctx || !radius || !q || !seq_lens || !sel_idx || !sel_cnt || !aligned(q, 16)) return DASHKV_ERR_INVALID_ARG;
    const dashkv_status s = check_view(ctx, kv, false, true);
    if (s != DASHKV_OK) return s;
    if (!use_fused(ctx)) return DASHKV_ERR_UNSUPPORTED;  // the fused selection only
    const int64_t cap = view_capacity(ctx, kv);
    const WsLayout L = ws_layout(ctx->cfg, cap);
    if (!workspace || workspace_bytes < L.total || !aligned(workspace, 256)) return DASHKV_ERR_WORKSPACE;
    KV k = make_kv(ctx, kv);
    k.radius = radius;
    const SelArgs a{ctx->cfg.topk, ctx->cfg.sink, ctx->cfg.window,
                    ctx->cfg.topk + ctx->cfg.sink + ctx->cfg.window};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Tracer tr(ctx, st);
    run_select(ctx, k, cap, L, static_cast<char *>(workspace), q, seq_lens, a, sel_idx, sel_cnt, scores, tr, st);
    return launch_status();
}

int32_t dashkv_select_kernels(const dashkv_ctx *ctx, int64_t max_tokens) {
    if (!ctx) return 0;
    (void)max_tokens;
    return use_fused(ctx) ? 1 : 2;
}

dashkv_status dashkv_set_trace(dashkv_ctx *ctx, void **events, int32_t n_events) {
    if (!ctx || n_events < 0 || (events && n_events < 2)) return DASHKV_ERR_INVALID_ARG;
    ctx->trace = events;
    ctx->n_trace = events ? n_events : 0;
    return DASHKV_OK;
}

dashkv_status dashkv_get_error(void *stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return DASHKV_ERR_CUDA;
    unsigned w = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&w, g_error_word, sizeof(w)) != cudaSuccess) return DASHKV_ERR_CUDA;
    if (w && cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) return DASHKV_ERR_CUDA;
    if (w & kErrTimeout) return DASHKV_ERR_TIMEOUT;
    if (w & kErrPage) return DASHKV_ERR_DEVICE;
    if (w & kErrCapacity) return DASHKV_ERR_CAPACITY;
    return DASHKV_OK;
}

}  // extern "C"
