// select.cuh -- stages 2 and 3: asymmetric scoring of every cached key from its
// code, then exact top-k with sinks and a recent window.
//
// Scoring (DASH-KV page, section "DASH-KV的核心创新：非对称深度哈希": the query
// stays in full precision while keys are hashed; Spherical KV page, section 2.1
// ADA: logits are computed straight from the packed codes, no dense key is
// rebuilt):
//     Qp_j = sum_{h in group} sum_i R[j][i] q_h[i]
//     s_t  = sum_j Qp_j (2 bit_tj - 1)
// evaluated as sum over code bytes c of LUT_c[byte_c(code_t)], where
// LUT_c[v] = sum_{u<8} Qp_{8c+u} (2 bit_u(v) - 1) is built per (b, kv head) in
// shared memory.  Summing the G query heads before projecting is the same
// linear map (R (sum_h q_h) = sum_h R q_h).
//
// Selection (DeepSeek DSA->CSA/HCA page, section "从 DSA 说起": an indexer
// scores the history, real attention runs on the top-k only; SWA paragraph of
// the CSA section: a recent window stays exact; DySCO page, Q3: attention sink
// tokens): top-k over all N tokens ordered by (score desc, index asc), united
// with [0, S) and [N - W, N), written ascending.
//
// Kernels (grid = (ctas per (b, h), B * Hkv)):
//   score_hist_kernel : LUT prologue, stream the codes, write fp32 scores, build
//                       a 4096-bin histogram of the scores over [-A, A]
//                       (A = sum_j |Qp_j| bounds every |s_t|); the last CTA of a
//                       (b, h) finds the bin T1 holding the k-th largest score.
//   collect_kernel    : ordered compaction of the tokens whose bin is >= T1
//                       into per-CTA segments; the last CTA of a (b, h) resolves
//                       the exact threshold inside bin T1 (score, then index)
//                       and writes the final ascending selection.
// No kernel waits on another CTA: "last CTA" is decided by an atomic arrival
// counter, which the last CTA resets, so the workspace is left clean.
#pragma once
#include "common.cuh"

namespace dkv {

constexpr int kBins = 4096;
constexpr int kSelThreads = 512;
constexpr int kMaxSelCtas = 512;
constexpr int kCandSmem = 2048;   // in-bin candidates ranked in shared memory
constexpr int kListSmem = 8192;   // candidate list held in shared memory by the resolver
constexpr int kCollectTile = kSelThreads * 16;

enum : int { kStateNormal = 0, kStateAll = 1, kStateEmpty = 2 };

struct SelState {
    int32_t T1;       // threshold bin
    int32_t above1;   // tokens in bins > T1
    int32_t cnt_T1;   // tokens in bin T1
    int32_t flags;
    float inv2A;      // 1 / (2 A): scores map to [0, 1] over [-A, A]
    float pad;
    int32_t kk;       // min(topk, N)
    int32_t n;        // N (clamped)
};

struct SelWS {
    float *scores;       // [BH][ld] internal score rows (ld multiple of 64)
    float *scores_out;   // optional user copy [BH][ld_out]
    int64_t ld, ld_out;
    int32_t *cand;       // [BH][ld]
    uint32_t *hist;      // [BH][kBins]        zero between calls
    SelState *state;     // [BH]
    uint32_t *arrive;    // [2][BH]            zero between calls
    int32_t *seg_cnt;    // [BH][kMaxSelCtas]
};

// Monotone map of a score to one of kBins bins (x in [0, 1] over [-A, A]).
__device__ __forceinline__ int score_bin(float s, float inv2A) {
    const float x = __saturatef(fmaf(s, inv2A, 0.5f));
    return (int)(x * (float)(kBins - 1));
}

// Token range [t0, t1) of CTA `c` of `nctas` over a length-n sequence; ranges
// are 64-aligned so a warp's 32 tokens never straddle a page.
__device__ __forceinline__ void cta_range(int64_t n, int c, int nctas, int64_t &t0, int64_t &t1) {
    int64_t per = ceil_div(ceil_div(n, nctas), 64) * 64;
    t0 = (int64_t)c * per;
    t1 = t0 + per < n ? t0 + per : n;
    if (t0 > n) t0 = n;
}

// Block-wide exclusive scan of one int per thread (blockDim = NT).
// Returns the exclusive prefix; *total gets the block sum.  All threads must call.
template <int NT = kSelThreads>
__device__ __forceinline__ int block_excl_scan(int v, int *s_warp, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < NT / 32 ? s_warp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < NT / 32) s_warp[lane] = w;  // inclusive warp prefix
    }
    __syncthreads();
    int before = warp ? s_warp[warp - 1] : 0;
    *total = s_warp[NT / 32 - 1];
    __syncthreads();  // s_warp may be reused right after
    return before + x - v;
}

// ---------------------------------------------------------------------------
// Score + histogram.
//
// One CTA of 1024 threads per SM.  The byte-LUT (256 rows x 256 B; row v holds
// LUT_c[v] for the T tables, replicated 32/T times) sits at a shared address
// whose low 16 bits are zero, so one byte-permute of (code word, per-lane
// offset) yields the complete shared address of a lookup:
//   addr = lut_base | byte << 8 | 4 * (copy * T + table).
// Lane l reads its token's bytes rotated by rho = l % T, so at each step the
// 32 lanes touch 32 distinct banks.
constexpr int kScoreThreads = 1024;

template <int BITS>
struct ScoreShape {
    static constexpr int T = BITS / 8;         // byte tables
    static constexpr int COPIES = 32 / T;      // interleaved copies: lanes hit distinct banks
    static constexpr int NW = BITS / 32;       // 32-bit code words per token
    static constexpr uint32_t LUT_BYTES = 256 * 256;
    static constexpr uint32_t LOW_BYTES = kBins * 4 + (kMaxDim + kMaxBits + 64) * 4;  // hist + scratch
    // dynamic smem: low region, then the LUT at the next 64 KB boundary
    static constexpr size_t SMEM = 2 * 65536 + LOW_BYTES;
    using Vec = typename std::conditional<BITS == 128, uint4, uint2>::type;  // one token's code
};

// Rotate the token's code bytes by rho (byte r of the result = byte (r + rho)
// mod 4*NW of the input).
// Branch-free: word rotation by rho / 4 as two select stages, then a funnel
// shift by 8 (rho % 4) bits across neighbouring words.
template <int NW>
__device__ __forceinline__ void rotate_bytes(uint32_t (&w)[NW], bool by8, bool by4, uint32_t sh) {
    uint32_t a[NW], c[NW];
#pragma unroll
    for (int k = 0; k < NW; ++k) a[k] = (NW == 4 && by8) ? w[(k + 2) % NW] : w[k];
#pragma unroll
    for (int k = 0; k < NW; ++k) c[k] = (NW >= 2 && by4) ? a[(k + 1) % NW] : a[k];
#pragma unroll
    for (int k = 0; k < NW; ++k) w[k] = __funnelshift_r(c[k], c[(k + 1) % NW], sh);
}

template <int BITS>
__device__ __forceinline__ void unpack_code(const typename ScoreShape<BITS>::Vec &x, uint32_t (&w)[BITS / 32]) {
    if constexpr (BITS == 128) {
        w[0] = x.x; w[1] = x.y; w[2] = x.z; w[3] = x.w;
    } else if constexpr (BITS == 64) {
        w[0] = x.x; w[1] = x.y;
    } else {
        w[0] = x.x;
    }
}

// Shared-memory load from a 32-bit shared address.  Not volatile: its address
// always depends on code words loaded after the barrier that publishes the LUT,
// so it cannot be scheduled before that barrier.
__device__ __forceinline__ float lds_f32(uint32_t addr) {
    float v;
    asm("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

// Score of one (rotated) code: sum over its T bytes of the lane's table entries.
template <int BITS>
__device__ __forceinline__ float lut_score(const uint32_t (&w)[BITS / 32], const uint32_t (&off)[BITS / 8]) {
    constexpr int T = BITS / 8;
    float s0 = 0.0f, s1 = 0.0f;
#pragma unroll
    for (int r = 0; r < T; r += 2) {
        s0 += lds_f32(__byte_perm(w[r >> 2], off[r], 0x7604u | ((uint32_t)(r & 3) << 4)));
        s1 += lds_f32(__byte_perm(w[(r + 1) >> 2], off[r + 1], 0x7604u | ((uint32_t)((r + 1) & 3) << 4)));
    }
    return (s0 + s1) + 0.0f;  // + 0 turns a -0 into +0
}

template <int BITS, int D>
__global__ void __launch_bounds__(kScoreThreads, 1)
score_hist_kernel(KV kv, const __nv_bfloat16 *__restrict__ q, int Hq, int G,
                  const int32_t *__restrict__ seq_lens, const RBits R, SelWS ws, int topk, int nctas) {
    using S = ScoreShape<BITS>;
    using Vec = typename S::Vec;
    constexpr int T = S::T, NW = S::NW;
    constexpr int NWARPS = kScoreThreads / 32;
    extern __shared__ __align__(1024) unsigned char smem[];
    uint32_t *hist = reinterpret_cast<uint32_t *>(smem);                  // [kBins]
    float *qsum = reinterpret_cast<float *>(hist + kBins);                // [D]
    float *Qp = qsum + kMaxDim;                                           // [BITS]
    float *red = Qp + kMaxBits;                                           // [64]
    const uint32_t smem_s = (uint32_t)__cvta_generic_to_shared(smem);
    const uint32_t lut_s = (smem_s + S::LOW_BYTES + 65535u) & ~65535u;     // 64 KB aligned
    unsigned char *lut = smem + (lut_s - smem_s);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bh = blockIdx.y, b = bh / kv.Hkv, h = bh % kv.Hkv;
    if (lut_s + 65536u > smem_s + (uint32_t)S::SMEM) {  // cannot happen with a small static region
        if (tid == 0) raise_error(kErrCapacity);
        return;
    }
    for (int i = tid; i < kBins; i += kScoreThreads) hist[i] = 0;
    for (int i = tid; i < D; i += kScoreThreads) {
        const __nv_bfloat16 *qh = q + ((int64_t)b * Hq + (int64_t)h * G) * D + i;
        float s = 0.0f;
        for (int g = 0; g < G; ++g) s += __bfloat162float(qh[(int64_t)g * D]);
        qsum[i] = s;
    }
    __syncthreads();
    // Qp_j: four threads per hyperplane, each a quarter of the dims.
    if (tid < 4 * BITS) {
        const int j = tid >> 2, part = tid & 3;
        float acc = 0.0f;
        for (int i = part * (D / 4); i < (part + 1) * (D / 4); ++i) {
            float rf = ((R.w[j * (D / 32) + i / 32] >> (i % 32)) & 1u) ? -1.0f : 1.0f;
            acc = fmaf(rf, qsum[i], acc);
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        if (part == 0) Qp[j] = acc;
    }
    __syncthreads();
    if (warp == 0) {
        float a = 0.0f;
        for (int j = lane; j < BITS; j += 32) a += fabsf(Qp[j]);
#pragma unroll
        for (int o = 16; o; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        if (lane == 0) red[0] = a > 0.0f ? 0.5f / a : 0.0f;
    }
    // LUT rows: word (v * 64 + copy * T + c) holds LUT_c[v]; lane l fills word l
    // of each row it owns (copy = l / T, c = l % T), so stores never conflict.
    {
        const int c = lane % T;
        float qv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) qv[u] = Qp[8 * c + u];
        for (int v = warp; v < 256; v += NWARPS) {
            float val = 0.0f;
#pragma unroll
            for (int u = 0; u < 8; ++u) val += ((v >> u) & 1) ? qv[u] : -qv[u];
            reinterpret_cast<float *>(lut + v * 256)[lane] = val;
        }
    }
    __syncthreads();
    const float inv2A = red[0];
    // everything above depends on q only; codes and lengths come from the append
    griddep_wait();
    const int64_t n = clamp_len(kv, seq_lens, b);

    int64_t t0, t1;
    cta_range(n, blockIdx.x, nctas, t0, t1);
    const int rho = lane % T, copy = lane / T;
    const bool rot8 = (rho & 8) != 0, rot4 = (rho & 4) != 0;
    const uint32_t rot_sh = 8u * (uint32_t)(rho & 3);
    uint32_t off[T];
#pragma unroll
    for (int r = 0; r < T; ++r) off[r] = lut_s | 4u * (uint32_t)(copy * T + (rho + r) % T);

    float *srow = ws.scores + (int64_t)bh * ws.ld;
    float *urow = ws.scores_out ? ws.scores_out + (int64_t)bh * ws.ld_out : nullptr;
    const int nloc = (int)(t1 - t0);  // tokens of this CTA (< 2^31)
    // lane's code pointer for local token index i (dense layout; paged via page table)
    const Vec *dense = reinterpret_cast<const Vec *>(kv.codes) + ((int64_t)bh * kv.n_cap + t0);
    auto fetch = [&](int i) -> Vec {  // i: local index of this lane's token (i < nloc)
        if (!kv.page_size) return __ldcs(dense + i);
        const int64_t c = kv.code(b, h, t0 + i);
        return c >= 0 ? __ldcs(reinterpret_cast<const Vec *>(kv.codes + c)) : Vec{};
    };

    constexpr int STEP = NWARPS * 32;
    int i = warp * 32 + lane;
    Vec nxt0 = i < nloc ? fetch(i) : Vec{};
    Vec nxt1 = i + STEP < nloc ? fetch(i + STEP) : Vec{};
    for (int g = warp * 32; g < nloc; g += 2 * STEP, i += 2 * STEP) {
        const Vec cur0 = nxt0, cur1 = nxt1;
        if (i + 2 * STEP < nloc) nxt0 = fetch(i + 2 * STEP);
        if (i + 3 * STEP < nloc) nxt1 = fetch(i + 3 * STEP);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int iu = i + u * STEP;
            uint32_t w[NW];
            unpack_code<BITS>(u ? cur1 : cur0, w);
            rotate_bytes<NW>(w, rot8, rot4, rot_sh);
            const float s = lut_score<BITS>(w, off);
            if (iu < nloc) {
                srow[t0 + iu] = s;
                if (urow) urow[t0 + iu] = s;
                atomicAdd(&hist[score_bin(s, inv2A)], 1u);
            }
        }
    }
    griddep_trigger();
    __syncthreads();
    uint32_t *ghist = ws.hist + (int64_t)bh * kBins;
    for (int k = tid; k < kBins; k += kScoreThreads)
        if (hist[k]) atomicAdd(ghist + k, hist[k]);

    // ---- last CTA of this (b, h): locate the threshold bin
    __shared__ int s_last;
    __shared__ int s_warp[32];
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(ws.arrive + bh, 1u) == (unsigned)(nctas - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int k = tid; k < kBins; k += kScoreThreads) {
        hist[k] = __ldcg(ghist + k);
        ghist[k] = 0;
    }
    __syncthreads();
    const int64_t kk = topk < n ? topk : n;
    constexpr int PER = kBins / kScoreThreads;  // bins per thread, thread 0 owns the top
    int local = 0;
    const int top = kBins - 1 - tid * PER;
#pragma unroll
    for (int e = 0; e < PER; ++e) local += hist[top - e];
    int total;
    const int before = block_excl_scan<kScoreThreads>(local, s_warp, &total);
    if (tid == 0) {
        SelState st;
        st.inv2A = inv2A; st.pad = 0.0f; st.kk = (int32_t)kk; st.n = (int32_t)n;
        st.T1 = kBins; st.above1 = 0; st.cnt_T1 = 0;
        st.flags = n == 0 ? kStateEmpty : (kk >= n ? kStateAll : kStateNormal);
        ws.state[bh] = st;
    }
    __syncthreads();
    if (n > 0 && kk < n && before < kk && before + local >= kk) {
        int run = before;
        for (int e = 0; e < PER; ++e) {
            const int bin = top - e;
            if (run + (int)hist[bin] >= kk) {
                ws.state[bh].T1 = bin;
                ws.state[bh].above1 = run;
                ws.state[bh].cnt_T1 = (int)hist[bin];
                break;
            }
            run += hist[bin];
        }
    }
    if (tid == 0) ws.arrive[bh] = 0;
}

// ---------------------------------------------------------------------------
// Collect + resolve.
//
// The candidate list of a (b, h) is the concatenation, in CTA order, of every
// CTA's segment (tokens of its range with bin >= T1, ascending), so the list
// is in ascending token order.  The resolver addresses it through a ListView:
// either a shared-memory copy (tokens + order keys) or, when the list is too
// long for that, the segments in global memory.
struct ListView {
    const int32_t *s_t;        // shared copy (or null)
    const uint32_t *s_key;
    const int32_t *cand;       // global segments
    const float *srow;
    const int *s_seg_off;      // exclusive prefix of the segment sizes [nctas + 1]
    int nctas, n;

    __device__ __forceinline__ void get(int e, int &t, uint32_t &key) const {
        if (s_t) {
            t = s_t[e];
            key = s_key[e];
            return;
        }
        int lo = 0, hi = nctas;  // segment c with s_seg_off[c] <= e < s_seg_off[c + 1]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (s_seg_off[mid] <= e) lo = mid; else hi = mid;
        }
        int64_t t0, t1;
        cta_range(n, lo, nctas, t0, t1);
        t = __ldcg(cand + t0 + (e - s_seg_off[lo]));
        key = float_key(__ldcg(srow + t));
    }
};

__device__ __forceinline__ float key_to_float(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// For every list element in order, f(e, t, key) -> bool; returns, per thread,
// the exclusive rank of its first kept element and the block total.  Each thread
// owns a contiguous run of elements so one block scan orders everything.
template <class Pred, class Emit>
__device__ __forceinline__ int ordered_pass(const ListView &L, int M, int *s_warp, Pred &&pred, Emit &&emit) {
    const int per = (M + kSelThreads - 1) / kSelThreads;
    const int e0 = threadIdx.x * per;
    const int e1 = min(M, e0 + per);
    int cnt = 0;
    for (int e = e0; e < e1; ++e) {
        int t; uint32_t key;
        L.get(e, t, key);
        cnt += pred(t, key) ? 1 : 0;
    }
    int total;
    int r = block_excl_scan(cnt, s_warp, &total);
    if (cnt)
        for (int e = e0; e < e1; ++e) {
            int t; uint32_t key;
            L.get(e, t, key);
            if (pred(t, key)) emit(r++, t);
        }
    return total;
}

struct CollectSmem {
    int32_t list_t[kListSmem];
    uint32_t list_key[kListSmem];
    uint32_t ck[kCandSmem];
    int32_t ci[kCandSmem];
    uint32_t h[2048];
    int seg_off[kMaxSelCtas + 1];
    int warp[32];
    int misc[8];
    int last;
};

__global__ void __launch_bounds__(kSelThreads)
collect_kernel(SelWS ws, int nctas, int S, int W, int cap_sel, int32_t *sel_idx, int32_t *sel_cnt) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    CollectSmem &sm = *reinterpret_cast<CollectSmem *>(smem_raw);
    const int tid = threadIdx.x;
    const int bh = blockIdx.y;
    griddep_wait();
    const SelState st = ws.state[bh];
    const int n = st.n;
    int32_t *cand = ws.cand + (int64_t)bh * ws.ld;
    const float *srow = ws.scores + (int64_t)bh * ws.ld;

    // ---- this CTA's segment: tokens of [t0, t1) with bin >= T1, ascending
    int count = 0;
    if (st.flags == kStateNormal) {
        int64_t t0, t1;
        cta_range(n, blockIdx.x, nctas, t0, t1);
        for (int64_t base = t0; base < t1; base += kCollectTile) {
            const int64_t tb = base + (int64_t)tid * 16;
            uint32_t flags = 0;
            if (tb + 16 <= t1) {
                const float4 *p = reinterpret_cast<const float4 *>(srow + tb);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const float4 x = __ldcg(p + v);
                    flags |= (uint32_t)(score_bin(x.x, st.inv2A) >= st.T1) << (4 * v + 0);
                    flags |= (uint32_t)(score_bin(x.y, st.inv2A) >= st.T1) << (4 * v + 1);
                    flags |= (uint32_t)(score_bin(x.z, st.inv2A) >= st.T1) << (4 * v + 2);
                    flags |= (uint32_t)(score_bin(x.w, st.inv2A) >= st.T1) << (4 * v + 3);
                }
            } else {
                for (int j = 0; j < 16; ++j)
                    if (tb + j < t1) flags |= (uint32_t)(score_bin(__ldcg(srow + tb + j), st.inv2A) >= st.T1) << j;
            }
            int tot;
            int r = block_excl_scan(__popc(flags), sm.warp, &tot);
            while (flags) {
                const int j = __ffs(flags) - 1;
                flags &= flags - 1;
                cand[t0 + count + r++] = (int32_t)(tb + j);
            }
            count += tot;
        }
    }
    griddep_trigger();
    if (tid == 0) ws.seg_cnt[(int64_t)bh * kMaxSelCtas + blockIdx.x] = count;
    __threadfence();
    __syncthreads();
    if (tid == 0) sm.last = atomicAdd(ws.arrive + gridDim.y + bh, 1u) == (unsigned)(nctas - 1);
    __syncthreads();
    if (!sm.last) return;
    __threadfence();

    // ---- the last CTA of (b, h): list offsets, exact threshold, final selection
    {
        const int c = tid;
        const int v = c < nctas ? __ldcg(ws.seg_cnt + (int64_t)bh * kMaxSelCtas + c) : 0;
        int tot;
        const int ex = block_excl_scan(v, sm.warp, &tot);
        if (c < nctas) sm.seg_off[c] = ex;
        if (c == 0) sm.seg_off[nctas] = tot;
    }
    __syncthreads();
    const int M = sm.seg_off[nctas];
    ListView L{nullptr, nullptr, cand, srow, sm.seg_off, nctas, n};
    if (st.flags == kStateNormal && M <= kListSmem) {
        // one parallel round over the whole list (each element finds its segment)
        for (int e = tid; e < M; e += kSelThreads) {
            int t; uint32_t key;
            L.get(e, t, key);
            sm.list_t[e] = t;
            sm.list_key[e] = key;
        }
        __syncthreads();
        L.s_t = sm.list_t;
        L.s_key = sm.list_key;
    }

    const float inv2A = st.inv2A;
    const int T1 = st.T1;
    uint32_t Tkey = 0;
    int IT = 0x7fffffff;
    if (st.flags == kStateNormal) {
        const int need1 = st.kk - st.above1;  // 1 <= need1 <= cnt_T1
        auto in_bin = [&](uint32_t key) { return score_bin(key_to_float(key), inv2A) == T1; };
        if (need1 < st.cnt_T1 && st.cnt_T1 <= kCandSmem) {
            // rank the in-bin candidates by (score desc, token asc)
            if (tid == 0) sm.misc[0] = 0;
            __syncthreads();
            for (int e = tid; e < M; e += kSelThreads) {
                int t; uint32_t key;
                L.get(e, t, key);
                if (in_bin(key)) {
                    const int slot = atomicAdd(&sm.misc[0], 1);
                    sm.ck[slot] = key;
                    sm.ci[slot] = t;
                }
            }
            __syncthreads();
            const int c1 = sm.misc[0];
            for (int e = tid; e < c1; e += kSelThreads) {
                const uint32_t ke = sm.ck[e];
                const int ie = sm.ci[e];
                int rank = 0;
                for (int f = 0; f < c1; ++f) {
                    const uint32_t kf = sm.ck[f];
                    rank += (kf > ke) || (kf == ke && sm.ci[f] < ie);
                }
                if (rank == need1 - 1) { sm.misc[1] = (int)ke; sm.misc[2] = ie; }
            }
            __syncthreads();
            Tkey = (uint32_t)sm.misc[1];
            IT = sm.misc[2];
        } else if (need1 < st.cnt_T1) {
            // Large, tie-heavy bin: radix-select the order key over the in-bin
            // tokens (11/11/10 bits), then the need-th tied token in list order.
            uint32_t prefix = 0, mask = 0;
            int need = need1;
#pragma unroll 1
            for (int p = 0; p < 3; ++p) {
                const int sh = p == 0 ? 21 : (p == 1 ? 10 : 0);
                const int nb = p == 2 ? 1024 : 2048;
                for (int i = tid; i < 2048; i += kSelThreads) sm.h[i] = 0;
                __syncthreads();
                for (int e = tid; e < M; e += kSelThreads) {
                    int t; uint32_t key;
                    L.get(e, t, key);
                    if (in_bin(key) && (key & mask) == prefix) atomicAdd(&sm.h[(key >> sh) & (nb - 1)], 1u);
                }
                __syncthreads();
                if (tid == 0) {
                    int run = 0, dd = nb - 1;
                    for (; dd > 0; --dd) {
                        if (run + (int)sm.h[dd] >= need) break;
                        run += sm.h[dd];
                    }
                    sm.misc[3] = dd;
                    sm.misc[4] = need - run;
                }
                __syncthreads();
                prefix |= (uint32_t)sm.misc[3] << sh;
                mask |= (uint32_t)(nb - 1) << sh;
                need = sm.misc[4];
                __syncthreads();
            }
            Tkey = prefix;
            if (tid == 0) sm.misc[5] = 0x7fffffff;
            __syncthreads();
            const int want = need;
            ordered_pass(L, M, sm.warp,
                         [&](int t, uint32_t key) { return in_bin(key) && key == Tkey; },
                         [&](int rank, int t) { if (rank + 1 == want) sm.misc[5] = t; });
            __syncthreads();
            IT = sm.misc[5];
        }
    }

    // ---- emit: sinks, kept list tokens in the middle range, window
    int32_t *out = sel_idx + (int64_t)bh * cap_sel;
    const int s_end = S < n ? S : n;                  // sinks [0, s_end)
    const int w_beg = n - W > s_end ? n - W : s_end;  // window [w_beg, n)
    int pos;
    if (st.flags == kStateAll) {
        for (int t = tid; t < n; t += kSelThreads) out[t] = t;
        pos = n;
    } else if (st.flags == kStateEmpty) {
        pos = 0;
    } else {
        for (int t = tid; t < s_end; t += kSelThreads) out[t] = t;
        pos = s_end;
        const int kept = ordered_pass(
            L, M, sm.warp,
            [&](int t, uint32_t key) {
                if (t < s_end || t >= w_beg) return false;
                const int bin = score_bin(key_to_float(key), inv2A);
                return bin > T1 || (bin == T1 && (key > Tkey || (key == Tkey && t <= IT)));
            },
            [&](int rank, int t) { if (pos + rank < cap_sel) out[pos + rank] = t; });
        pos += kept;
        for (int t = w_beg + tid; t < n; t += kSelThreads)
            if (pos + (t - w_beg) < cap_sel) out[pos + (t - w_beg)] = t;
        pos += n - w_beg;
        if (pos > cap_sel) pos = cap_sel;  // unreachable when the threshold is consistent
    }
    for (int r = pos + tid; r < cap_sel; r += kSelThreads) out[r] = -1;
    if (tid == 0) sel_cnt[bh] = pos;
    if (tid == 0) ws.arrive[gridDim.y + bh] = 0;
}

}  // namespace dkv
