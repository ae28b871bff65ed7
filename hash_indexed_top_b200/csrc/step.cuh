// step.cuh -- one decode step in one kernel: (append the step's key) -> score
// every cached key from its code -> exact top-k united with sinks and window
// -> (exact attention over the selection).
//
// DASH-KV page, "DASH-KV的核心创新：非对称深度哈希" (the query stays in full
// precision, keys are hashed) and "从平方到线性" (hash codes, then top-K
// candidate pruning); Spherical KV page, section 2.1 ADA (logits straight from
// the packed codes); DeepSeek DSA->CSA/HCA page, "从 DSA 说起" (an indexer
// scores the whole history, attention runs on the top-k only) and the SWA
// paragraph of its CSA section (a recent window stays exact); DySCO page, Q3
// (attention sinks).
//
// Grid: one thread-block cluster of C CTAs (16 consumer warps and one producer
// warp, one CTA per SM) per (sequence, kv head); CTA c owns a contiguous,
// 64-aligned token range.
//
//  stream   the CTA streams its codes in stages of 16 KB through a ring in
//           shared memory: dense caches by one bulk copy per stage
//           (cp.async.bulk, completion counted in bytes on the stage's full
//           mbarrier), issued by the producer warp as soon as every consumer
//           warp has released the slot on its empty mbarrier; paged caches by
//           per-thread cp.async of each thread's own tokens (warp 15 idles).
//           A consumer warp (0..14)
//           reads the next stage's codes into registers before it scores the
//           current one, and releases a slot as soon as its codes are in
//           registers.  Consumer warp w
//           takes a 32- or 64-token slice of every stage and lane l scores the
//           tokens t = l (mod 32) with the byte-LUT of the query (the codes are
//           stored byte-rotated by t mod T, see store_code_rotated).  A token
//           whose score reaches the CTA's threshold is kept with its exact
//           order key in the warp's candidate list in shared memory; after the
//           stream every warp counts its list into the CTA histogram.
//  estimate the threshold comes from a stratified sample of the whole
//           sequence scored before the stream (the same 32-token blocks in
//           every CTA of the cluster): the bin of a sample rank set a few
//           standard deviations above the one the k-th largest score is
//           expected at.  It is an estimate and nothing rests on it: when the
//           cluster's k-th largest counted score lies below the threshold (or
//           fewer than k are counted) the estimate was too high, and a full
//           candidate list means it was far too low; either way the exact slow
//           path runs.
//  select   the cluster sums its histograms through distributed shared
//           memory and finds the bin T1 holding the k-th largest score (exact:
//           every CTA counted every token of every bin at or above its
//           threshold, and no threshold is above T1); the warps classify their
//           candidates, rank the few of bin T1 exactly (score desc, index
//           asc), mark the kept tokens in a bitmap of the CTA's range and
//           write them in order.  Heavy ties (more than kInbinMax tokens in
//           T1), a full candidate list or a threshold estimate above T1 take
//           an exact slow path (re-score and count every token into the
//           workspace, CTA 0 runs the two-kernel path's resolver).
//  attend   (G > 0) every CTA attends over its own kept tokens (listed in
//           shared memory as it emits them), its share of the window and, in
//           CTA 0, the sinks (the slow path: an equal slice of the emitted
//           list).  Warps copy the K / V rows into shared memory with 16-byte
//           cp.async (a row per warp instruction; two tiles in flight per warp)
//           and run an online softmax in fp32.  Each CTA
//           pushes its partial state, element by element, into the shared
//           memory of the CTA that merges that element, and after one cluster
//           barrier every CTA merges and writes the elements it owns.
//  append   (k_new given) the CTA that owns position seq_lens[b] encodes the
//           new key, writes its code and K/V rows there and scores it from
//           the code it computed; the last cluster of a sequence to finish
//           increments seq_lens[b] (every CTA read it at its start).
#pragma once
#include "decode.cuh"
#include "select.cuh"
#include "step_args.cuh"

namespace dkv {

// fp32 LUT score of one token's (rotated) code words for a token t (any lane):
// lane offset t mod 32 keeps the table order right (t mod T = lane mod T).
template <int BITS>
__device__ __forceinline__ float lut_score_any(const uint32_t (&w)[BITS / 32], uint32_t lut_s, int64_t t) {
    return lut_score<BITS>(w, lut_s | (4u * (uint32_t)(t & 31)));
}

// Code words of token t of (b, h) loaded with a plain load (slow paths), or
// false when its page is out of range.
template <int BITS>
__device__ __forceinline__ bool load_code_plain(const KV &kv, int b, int h, int64_t t, uint32_t (&w)[BITS / 32]) {
    const int64_t c = kv.code(b, h, t);
    if (c < 0) return false;
    if constexpr (BITS == 128) {
        const uint4 x = __ldg(reinterpret_cast<const uint4 *>(kv.codes + c));
        w[0] = x.x; w[1] = x.y; w[2] = x.z; w[3] = x.w;
    } else if constexpr (BITS == 64) {
        const uint2 x = __ldg(reinterpret_cast<const uint2 *>(kv.codes + c));
        w[0] = x.x; w[1] = x.y;
    } else {
        w[0] = __ldg(reinterpret_cast<const uint32_t *>(kv.codes + c));
    }
    return true;
}

// r~ = (c + 1/2) / 4 of token t's radius code (radius-scaled scores).
__device__ __forceinline__ float radius_of_token(const KV &kv, int b, int h, int64_t t) {
    const int64_t r = kv.radius_index(b, h, t);
    return r >= 0 ? ((float)__ldg(kv.radius + r) + 0.5f) * 0.25f : 0.0f;
}

template <int BITS, int D, int G, bool PAGED, bool RADIUS>
__global__ void __launch_bounds__(kStepThreads, 1) step_kernel(const StepArgs a, const RBits R) {
    using SS = StepShape<BITS>;
    constexpr int NS = kRingStages;
    constexpr int NWARP = kStepWarps, NT = kStepThreads, NCONS = kStreamWarps;
    constexpr int CODE_B = SS::CODE_B, TPL = SS::TPL, STG_TOK = SS::STG_TOK, STG_B = SS::STG_B;
    constexpr int T = BITS / 8;
    extern __shared__ __align__(1024) unsigned char smem[];
    const KV &kv = a.kv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bh = blockIdx.y, cta = blockIdx.x, nctas = gridDim.x;
    const int b = bh / kv.Hkv, h = bh % kv.Hkv;
    const uint32_t lt = (1u << lane) - 1u;

    const uint32_t smem_s = (uint32_t)__cvta_generic_to_shared(smem);
    uint32_t *hist = reinterpret_cast<uint32_t *>(smem + StepLow::HIST);
    uint32_t *sup = reinterpret_cast<uint32_t *>(smem + StepLow::SUP);
    uint32_t *shist = reinterpret_cast<uint32_t *>(smem + StepLow::SHIST);
    uint32_t *ssup = reinterpret_cast<uint32_t *>(smem + StepLow::SSUP);
    float *qsum = reinterpret_cast<float *>(smem + StepLow::QSUM);
    float *Qp = reinterpret_cast<float *>(smem + StepLow::QP);
    float *knew = reinterpret_cast<float *>(smem + StepLow::KNEW);
    int *misc = reinterpret_cast<int *>(smem + StepLow::MISC);
    uint32_t *newc = reinterpret_cast<uint32_t *>(smem + StepLow::NEWC);
    uint32_t *newr = reinterpret_cast<uint32_t *>(smem + StepLow::NEWR);
    int *s_wdef = reinterpret_cast<int *>(smem + StepLow::WDEF);
    int (*s_cnt)[2] = reinterpret_cast<int (*)[2]>(smem + StepLow::CNT);
    int *s_mid = reinterpret_cast<int *>(smem + StepLow::MID);
    int *s_warp = reinterpret_cast<int *>(smem + StepLow::WARPSCAN);
    const uint32_t mbar_full = smem_s + StepLow::MBAR;         // [NS]
    const uint32_t mbar_empty = smem_s + StepLow::MBAR_EMPTY;  // [NS]
    const bool consumer = warp < NCONS;  // (during the stream; warp NCONS is its producer)
    const uint32_t lut_s = (smem_s + StepLow::END + 65535u) & ~65535u;  // 64 KB aligned
    unsigned char *lut = smem + (lut_s - smem_s);
    const uint32_t ring_s = lut_s + 65536u;
    unsigned char *ring = lut + 65536;
    // candidate list of this warp: cap entries (token in the CTA's range, order
    // key) between the low region and the attention merge's inbox below the LUT
    const uint32_t recv_s = lut_s - (uint32_t)kRecvBytes;  // the attention merge's inbox (G > 0)
    // (NCONS lists: warp NCONS has none and keeps ncand = 0)
    const int cap = (int)((recv_s - (smem_s + StepLow::END)) / (8u * NCONS));
    uint2 *cand = reinterpret_cast<uint2 *>(smem + StepLow::END) + warp * cap;

    // ---- set-up: counters, barriers, this warp's hyperplane words
    for (int i = tid; i < kBins; i += NT) hist[i] = 0;
    for (int i = tid; i < kSampleBins; i += NT) shist[i] = 0;
    if (tid < 64) { sup[tid] = 0; ssup[tid] = 0; misc[tid] = 0; }
    if (tid < 4) newc[tid] = 0;
    if (tid < NS) { mbar_init(mbar_full + 8u * tid, 1); mbar_init(mbar_empty + 8u * tid, NCONS); }
    if (tid < NS) fence_mbar_init();
    static_assert(BITS % NWARP == 0, "hyperplanes per warp");
    uint32_t rw[BITS / NWARP][D / 32];
#pragma unroll
    for (int m = 0; m < BITS / NWARP; ++m)
#pragma unroll
        for (int k = 0; k < D / 32; ++k) rw[m][k] = R.w[(warp + NWARP * m) * (D / 32) + k];

    // everything the kernel reads may come from the preceding kernel of the stream
    griddep_wait();
    griddep_trigger();

    // ---- lengths (and the append's position)
    const bool appending = a.k_new != nullptr;
    const int64_t capn = kv.capacity();
    int64_t pos = -1;  // position of the appended token, or -1
    int64_t n;
    bool app_ok = false;
    if (appending) {
        const int64_t p0 = __ldcg(a.seq_lens + b);
        app_ok = p0 >= 0 && p0 < capn;
        if (app_ok && PAGED) {
            const int32_t pg = __ldg(kv.page_table + (int64_t)b * kv.max_pages + p0 / kv.page_size);
            app_ok = pg >= 0 && pg < kv.num_pages;
            if (!app_ok && cta == 0 && tid == 0) raise_error(kErrPage);
        } else if (!app_ok && cta == 0 && tid == 0) {
            raise_error(kErrCapacity);
        }
        if (app_ok) pos = p0;
        n = app_ok ? p0 + 1 : (p0 < 0 ? 0 : (p0 > capn ? capn : p0));
    } else {
        n = clamp_len(kv, a.seq_lens, b);
    }
    int64_t t0, t1;
    cta_range(n, cta, nctas, t0, t1);
    const int s_end = (int)(a.S < n ? a.S : n);  // sinks [0, s_end), window [w_beg, n)
    const int w_beg = (int)(n - a.W > s_end ? n - a.W : s_end);
    // this CTA's share of the window rows for the attention: [wt0, wt0 + nw)
    const int per_w = (int)ceil_div(n - w_beg, (int64_t)nctas);
    const int64_t wt0 = w_beg + (int64_t)cta * per_w;
    const int nw = (int)max((int64_t)0, min((int64_t)per_w, n - wt0));
    const int nloc = (int)(t1 - t0);
    const int nstg = (nloc + STG_TOK - 1) / STG_TOK;  // stages of this CTA
    const bool own_new = pos >= t0 && pos < t1;
    const int pos_loc = own_new ? (int)(pos - t0) : -1;

    // ---- the code ring.  Dense: stage s is one bulk copy of the stage's codes
    // (when they lie inside the capacity at a 16-byte aligned address; else its
    // tokens are read with plain loads), issued by whichever warp is the last
    // to release the slot.  Paged: every thread copies its own tokens of the
    // stage with cp.async (a stage's 32-token warp slices lie in single pages
    // for pages of 64 or more tokens) and reads only what it copied.  Either
    // way a warp reads stage s + 1 into registers before it scores stage s, and
    // releases a slot once the codes it read from there have been scored.
    const unsigned char *codes_b = reinterpret_cast<const unsigned char *>(kv.codes);
    const unsigned char *dense_base = codes_b + ((int64_t)bh * kv.n_cap + t0) * CODE_B;
    auto stage_tokens = [&](int s) { return min(STG_TOK, nloc - s * STG_TOK); };
    // bytes of dense stage s's bulk copy, or 0 when it is read with plain loads
    auto stage_bulk_bytes = [&](int s) -> uint32_t {
        if constexpr (PAGED) return 0u;
        const int cnt = stage_tokens(s);
        const uint32_t bytes = ((uint32_t)(cnt * CODE_B) + 15u) & ~15u;
        const unsigned char *src = dense_base + (int64_t)s * STG_B;
        const bool inside = (t0 + (int64_t)s * STG_TOK) * CODE_B + bytes <= kv.n_cap * CODE_B;
        return (inside && !(reinterpret_cast<uintptr_t>(src) & 15u)) ? bytes : 0u;
    };
    auto issue_dense = [&](int s) {  // one thread
        const uint32_t mb = mbar_full + 8u * (uint32_t)(s % NS);
        const uint32_t bytes = stage_bulk_bytes(s);
        if (bytes) {
            mbar_arrive_expect_tx(mb, bytes);
            // codes are read once: first out of L2, ahead of the K / V rows kept there
            bulk_g2s_hint(ring_s + (uint32_t)((s % NS) * STG_B), dense_base + (int64_t)s * STG_B, bytes, mb,
                          l2_policy_evict_first());
        } else {
            mbar_arrive(mb);  // completes the phase with no data
        }
    };
    // PAGED: physical page of this lane's token u of stage s (-1: none, -2: out of range)
    auto lane_page = [&](int s, int u) -> int {
        const int i = s * STG_TOK + warp * 32 * TPL + 32 * u + lane;
        if (s >= nstg || i >= nloc) return -1;
        const int32_t p = __ldg(kv.page_table + (int64_t)b * kv.max_pages + (t0 + i) / kv.page_size);
        return (p < 0 || p >= kv.num_pages) ? -2 : p;
    };
    uint32_t pbad = 0;  // PAGED: bit (slot * TPL + u) set when that token's page is out of range
    auto issue_paged = [&](int s, const int (&pg)[TPL]) {  // every thread, one commit group per stage
        const int slot = s % NS;
#pragma unroll
        for (int u = 0; u < TPL; ++u) {
            const int li = warp * 32 * TPL + 32 * u + lane;  // token within the stage
            const int i = s * STG_TOK + li;
            const void *src = codes_b;
            uint32_t sz = 0;
            const uint32_t bit = 1u << (slot * TPL + u);
            pbad &= ~bit;
            if (pg[u] >= 0) {
                src = codes_b + (((int64_t)pg[u] * kv.Hkv + h) * kv.page_size + (t0 + i) % kv.page_size) * CODE_B;
                sz = CODE_B;
            } else if (pg[u] == -2) {
                raise_error(kErrPage);
                pbad |= bit;
            }
            const uint32_t dst = ring_s + (uint32_t)(slot * STG_B + li * CODE_B);
            if constexpr (CODE_B == 16)
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(sz) : "memory");
            else
                asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(dst), "l"(src), "r"(sz) : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    int pgn[TPL];  // PAGED: pages of this lane's tokens of the next stage to issue

    // the group's summed query and the appended key (their loads overlap the
    // barrier set-up)
    for (int i = tid; i < D; i += NT) {
        const __nv_bfloat16 *qh = a.q + ((int64_t)b * a.Hq + (int64_t)h * a.G) * D + i;
        float s = 0.0f;
        for (int g = 0; g < a.G; ++g) s += __bfloat162float(qh[(int64_t)g * D]);
        qsum[i] = s;
    }
    if (own_new && tid < D) knew[tid] = __bfloat162float(a.k_new[((int64_t)b * kv.Hkv + h) * D + tid]);
    __syncthreads();  // barriers initialised; qsum, knew ready
    if constexpr (PAGED) {
        for (int s = 0; s < NS && consumer; ++s) {
            int pg[TPL];
#pragma unroll
            for (int u = 0; u < TPL; ++u) pg[u] = lane_page(s, u);
            issue_paged(s, pg);
        }
#pragma unroll
        for (int u = 0; u < TPL; ++u) pgn[u] = lane_page(NS, u);
    } else {
        if (tid == NCONS * 32)  // the producer
            for (int s = 0; s < NS && s < nstg; ++s) issue_dense(s);
    }

    // ---- the threshold estimate's sample: one 32-token block of each of
    // `nstrata` strata of the whole sequence, at a pseudo-random offset in the
    // stratum (the same blocks in every CTA of the cluster; the appended token
    // is left out).  Its codes are loaded now; they are scored once the LUT is
    // built.
    const int64_t kk = a.topk < n ? a.topk : n;
    const bool normal = n > 0 && kk < n;
    const int nblk_all = (int)(n >> 5);
    const int nstrata = normal ? min(kSampleStrata, nblk_all / 16) : 0;
    constexpr int SPW = kSampleStrata / NWARP;  // blocks per warp
    uint32_t smp[SPW][BITS / 32];
    float smr[SPW];
    bool sok[SPW];
#pragma unroll
    for (int q = 0; q < SPW; ++q) {
        const int j = warp + NWARP * q;
        sok[q] = false;
        smr[q] = 0.0f;
#pragma unroll
        for (int k = 0; k < BITS / 32; ++k) smp[q][k] = 0u;
        if (j < nstrata) {
            const int stride = nblk_all / nstrata;
            uint32_t hsh = (uint32_t)j * 0x9E3779B1u ^ ((uint32_t)bh * 0x85EBCA77u);
            hsh ^= hsh >> 15;
            hsh *= 0x2C1B3C6Du;
            hsh ^= hsh >> 12;
            const int64_t t = 32 * ((int64_t)j * stride + (int64_t)(hsh % (uint32_t)stride)) + lane;
            if (t != pos) sok[q] = load_code_plain<BITS>(kv, b, h, t, smp[q]);
            if constexpr (RADIUS) smr[q] = sok[q] ? radius_of_token(kv, b, h, t) : 0.0f;
        }
    }

    // ---- LUT of the group's summed query (as the two-kernel scorer builds it)
    // Qp_j = sum_i R[j][i] qsum[i] (and, in the CTA that appends, the new key's
    // projections): warp w takes hyperplanes w, w + 32, ... and lane l the dims
    // l, l + 32, ...; a shuffle tree sums the lanes.  Exact on grid inputs.
#pragma unroll
    for (int m = 0; m < BITS / NWARP; ++m) {
        float acc = 0.0f, kacc = 0.0f;
#pragma unroll
        for (int k = 0; k < D / 32; ++k) {
            const float sg = ((rw[m][k] >> lane) & 1u) ? -1.0f : 1.0f;
            acc = fmaf(sg, qsum[32 * k + lane], acc);
            if (own_new) kacc = fmaf(sg, knew[32 * k + lane], kacc);
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            acc += __shfl_xor_sync(0xffffffffu, acc, o);
            kacc += __shfl_xor_sync(0xffffffffu, kacc, o);
        }
        if (lane == 0) {
            Qp[warp + NWARP * m] = acc;
            // hyperplane j = warp + NWARP m is bit j % 32 of code word j / 32 (a tie at 0 gives 1)
            const int j = warp + NWARP * m;
            if (own_new && kacc >= 0.0f) atomicOr(newc + (j >> 5), 1u << (j & 31));
        }
    }
    __syncthreads();
    float inv2A;
    {
        float s = 0.0f;
        for (int j = lane; j < BITS; j += 32) s += fabsf(Qp[j]);
#pragma unroll
        for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (RADIUS) s *= kRadiusMax;
        inv2A = s > 0.0f ? 0.5f / s : 0.0f;
    }
    {   // LUT rows: word j of row v holds LUT_{j mod T}[v] (see score_phase)
        static_assert(256 % NWARP == 0 && (256 / NWARP) <= 16, "rows per warp");
        constexpr int RPW = 256 / NWARP;
        constexpr int RB = RPW >= 16 ? 4 : (RPW >= 8 ? 3 : (RPW >= 4 ? 2 : (RPW >= 2 ? 1 : 0)));  // log2 RPW
        const int c = lane % T;
        float qv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) qv[u] = Qp[8 * c + u];
        const int v0 = warp * RPW;
        float base = 0.0f;
#pragma unroll
        for (int u = 0; u < 8; ++u) base += ((v0 >> u) & 1) ? qv[u] : -qv[u];
#pragma unroll
        for (int dd = 0; dd < RPW; ++dd) {
            float val = base;
#pragma unroll
            for (int u = 0; u < RB; ++u)
                if ((dd >> u) & 1) val += 2.0f * qv[u];
            float *row = reinterpret_cast<float *>(lut + (v0 + dd) * 256);
            row[lane] = val;
            row[lane + 32] = val;
        }
    }
    // the appended token: its K / V rows and code go to the cache (the
    // attention below reads its rows from k_new / v_new, and this kernel
    // scores it from newr)
    if (own_new) {
        if (tid < 2 * (D / 8)) {
            const bool isv = tid >= D / 8;
            const int part = isv ? tid - D / 8 : tid;
            const int64_t r = kv.row(b, h, pos);
            const uint4 x = __ldg(reinterpret_cast<const uint4 *>((isv ? a.v_new : a.k_new) +
                                                                  ((int64_t)b * kv.Hkv + h) * D) + part);
            if (r >= 0) reinterpret_cast<uint4 *>((isv ? kv.v : kv.k) + r)[part] = x;
        }
        if (tid == 64) {
            uint32_t w32[BITS / 32];
#pragma unroll
            for (int k = 0; k < BITS / 32; ++k) w32[k] = newc[k];
            const int64_t c = kv.code(b, h, pos);
            if (c >= 0) store_code_rotated<BITS>(kv.codes + c, w32, pos);
            rotate_code<BITS>(w32, pos);  // the order the scorer reads codes in
#pragma unroll
            for (int k = 0; k < BITS / 32; ++k) newr[k] = w32[k];
        }
    }
    if (tid == 0) misc[kMTloc] = normal ? 0 : kBins;  // kBins: nothing is kept
    __syncthreads();  // LUT, newr, tloc ready
    const uint32_t lbase = lut_s | (4u * (uint32_t)lane);

    // ---- threshold estimate: the sample's histogram gives the bin of sample
    // rank r_s = e + 3.5 sqrt(e) + 8, where e = k m / n is the number of sample
    // tokens expected at or above the k-th largest score (m sample tokens).
    if (nstrata > 0) {
        int cnt = 0;
#pragma unroll
        for (int q = 0; q < SPW; ++q) {
            if (sok[q]) {
                float sc = lut_score<BITS>(smp[q], lbase);  // (t = lane mod 32)
                if constexpr (RADIUS) sc = __fmul_rn(sc, smr[q]);
                const int bin = score_bin(sc, inv2A);
                atomicAdd(&shist[bin / kSampleDiv], 1u);
                atomicAdd(&ssup[bin >> 6], 1u);
            }
            cnt += __popc(__ballot_sync(0xffffffffu, sok[q]));
        }
        if (lane == 0 && cnt) atomicAdd(misc + kMSamp, cnt);
        __syncthreads();
        if (warp == 0) {
            const int m = misc[kMSamp];
            const float e = (float)kk * (float)m / (float)n;
            const int64_t rs = (int64_t)ceilf(e + 3.5f * sqrtf(e) + 8.0f);
            const int cb = rs <= m ? cluster_threshold<kSampleBins / 64, true>(ssup, shist, 1, rs, nullptr) : -1;
            if (lane == 0 && cb > 0) misc[kMTloc] = cb * kSampleDiv;
        }
        __syncthreads();
    }

    // ---- stream: score every token of the CTA's range, stage by stage
    const int wsl = warp * 32 * TPL;  // this warp's slice of a stage
    int ncand = 0;
    bool ovf = false, tmo = false;
    float *srow_out = a.scores_out ? a.scores_out + (int64_t)bh * a.ld_out + t0 : nullptr;
    // the candidate test: a score at or above thr_f, a little below the lowest
    // score of bin tl (so every token of bins >= tl is kept: its bin is exact
    // and checked when the lists are counted)
    const int tl = misc[kMTloc];
    const float thr_f = tl <= 0 || inv2A == 0.0f ? -INFINITY
                        : (tl >= kBins ? INFINITY
                                       : (((float)tl / (float)(kBins - 1) - 0.5f) - 1e-5f) / inv2A);
    float rad[TPL];
#pragma unroll
    for (int u = 0; u < TPL; ++u) rad[u] = 0.0f;
    auto load_radius = [&](int s) {
#pragma unroll
        for (int u = 0; u < TPL; ++u) {
            const int i = s * STG_TOK + wsl + 32 * u + lane;
            rad[u] = (s < nstg && i < nloc) ? radius_of_token(kv, b, h, t0 + i) : 0.0f;
        }
    };
    if constexpr (RADIUS) load_radius(0);
    // every stage but the last is full: one check covers them (the alignment of
    // a stage is that of the first, and the last full one is the one nearest
    // the capacity)
    const bool bulk_mid = nstg > 1 && stage_bulk_bytes(nstg - 2) != 0u;
    const bool bulk_last = nstg > 0 && stage_bulk_bytes(nstg - 1) != 0u;
    // stage s's codes for this lane into w (dense: once the slot's copy landed);
    // false when the wait gave up
    auto read_stage = [&](int s, uint32_t (&w)[TPL][BITS / 32]) -> bool {
        const int slot = s % NS;
        if constexpr (!PAGED) {
            if (!mbar_wait(mbar_full + 8u * (uint32_t)slot, (uint32_t)((s / NS) & 1))) return false;
        }
        const bool from_ring = PAGED || (s + 1 < nstg ? bulk_mid : bulk_last);
#pragma unroll
        for (int u = 0; u < TPL; ++u) {
            const int li = wsl + 32 * u + lane;  // token within the stage
            if (from_ring) {
                const unsigned char *src = ring + slot * STG_B + li * CODE_B;
                if constexpr (BITS == 128) {
                    const uint4 x = *reinterpret_cast<const uint4 *>(src);
                    w[u][0] = x.x; w[u][1] = x.y; w[u][2] = x.z; w[u][3] = x.w;
                } else if constexpr (BITS == 64) {
                    const uint2 x = *reinterpret_cast<const uint2 *>(src);
                    w[u][0] = x.x; w[u][1] = x.y;
                } else {
                    w[u][0] = *reinterpret_cast<const uint32_t *>(src);
                }
            } else {
#pragma unroll
                for (int k = 0; k < BITS / 32; ++k) w[u][k] = 0u;
                const int i = s * STG_TOK + li;
                if (i < nloc) load_code_plain<BITS>(kv, b, h, t0 + i, w[u]);
            }
        }
        return true;
    };
    uint32_t cur[TPL][BITS / 32];
    int s = 0;
    if (!consumer) {
        // ---- the producer: refills a slot with stage r as soon as every
        // consumer warp has released it from stage r - NS
        if constexpr (!PAGED) {
            if (lane == 0)
                for (int r = NS; r < nstg; ++r) {
                    if (!mbar_wait(mbar_empty + 8u * (uint32_t)(r % NS), (uint32_t)((r / NS - 1) & 1))) break;
                    issue_dense(r);
                }
            __syncwarp();
        }
    } else {
        if (nstg > 0) {
            if constexpr (PAGED) asm volatile("cp.async.wait_group %0;" ::"n"(NS - 1) : "memory");
            tmo = !read_stage(0, cur);
            __syncwarp();
            if (!PAGED && lane == 0) mbar_arrive(mbar_empty);  // stage 0's codes are in registers
        }
#pragma unroll 1
        for (; s < nstg && !tmo; ++s) {
            uint32_t nxt[TPL][BITS / 32];
            if (s + 1 < nstg) {
                if constexpr (PAGED) asm volatile("cp.async.wait_group %0;" ::"n"(NS - 2) : "memory");
                tmo = !read_stage(s + 1, nxt);  // (stage s is still scored)
            }
            float rnow[TPL];
#pragma unroll
            for (int u = 0; u < TPL; ++u) rnow[u] = rad[u];
            if constexpr (RADIUS) load_radius(s + 1);
            const int sbase = s * STG_TOK;
            if (pos_loc >= sbase && pos_loc < sbase + STG_TOK) {
                // the appended token is scored from the code computed above
#pragma unroll
                for (int u = 0; u < TPL; ++u)
                    if (sbase + wsl + 32 * u + lane == pos_loc) {
#pragma unroll
                        for (int k = 0; k < BITS / 32; ++k) cur[u][k] = newr[k];
                    }
            }
            float sc[TPL];
#pragma unroll
            for (int u = 0; u < TPL; ++u) {
                sc[u] = lut_score<BITS>(cur[u], lbase);
                if constexpr (RADIUS) sc[u] = __fmul_rn(sc[u], rnow[u]);
            }
            const bool full_stage = sbase + STG_TOK <= nloc;
            bool isc[TPL];
            bool mine = false;
#pragma unroll
            for (int u = 0; u < TPL; ++u) {
                const int i = sbase + wsl + 32 * u + lane;
                bool valid = full_stage || i < nloc;
                if constexpr (PAGED) valid = valid && !((pbad >> ((s % NS) * TPL + u)) & 1u);
                if (srow_out && valid) srow_out[i] = sc[u];
                isc[u] = valid && sc[u] >= thr_f;
                mine |= isc[u];
            }
            if (__any_sync(0xffffffffu, mine) && !ovf) {
#pragma unroll
                for (int u = 0; u < TPL; ++u) {
                    const uint32_t ball = __ballot_sync(0xffffffffu, isc[u]);
                    const int nb = __popc(ball);
                    if (ncand + nb > cap) {  // full: the exact slow path takes over
                        ovf = true;
                        if (lane == 0) misc[kMOvf] = 1;
                        break;
                    }
                    if (isc[u]) {
                        const int i = sbase + wsl + 32 * u + lane;
                        cand[ncand + __popc(ball & lt)] = make_uint2((uint32_t)i, float_key(sc[u]));
                    }
                    ncand += nb;
                }
            }
            __syncwarp();
            if constexpr (PAGED) {
                // refill slot s % NS (its codes were read a stage ago) with stage s + NS
                int pg[TPL];
#pragma unroll
                for (int u = 0; u < TPL; ++u) pg[u] = pgn[u];
#pragma unroll
                for (int u = 0; u < TPL; ++u) pgn[u] = lane_page(s + NS + 1, u);
                issue_paged(s + NS, pg);
            } else {
                // release stage s + 1's slot: its codes are in registers (the
                // arrive orders the loads before it)
                if (lane == 0 && s + 1 < nstg && !tmo) mbar_arrive(mbar_empty + 8u * (uint32_t)((s + 1) % NS));
            }
#pragma unroll
            for (int u = 0; u < TPL; ++u)
#pragma unroll
                for (int k = 0; k < BITS / 32; ++k) cur[u][k] = nxt[u][k];
        }
        if constexpr (PAGED) asm volatile("cp.async.wait_group 0;" ::: "memory");
        if (tmo) {  // give the copies still in flight a bounded chance to land before the buffers are reused
            for (int c = s; c < nstg && c < s + NS; ++c) mbar_wait(mbar_full + 8u * (c % NS), (uint32_t)((c / NS) & 1));
            if (lane == 0) misc[kMOvf] = 1;
            ovf = true;
        }
        // the CTA histogram of the kept tokens of bins >= tl, from this warp's list
        if (!ovf)
            for (int j = lane; j < ncand; j += 32) {
                const int bin = score_bin(key_to_float(cand[j].y), inv2A);
                if (bin >= tl) {
                    atomicAdd(&hist[bin], 1u);
                    atomicAdd(&sup[bin >> 6], 1u);
                }
            }
    }
    __syncthreads();  // every warp's list and the histogram are complete

    // ---- the cluster's threshold bin T1 (exact when found: every CTA counted
    // every token of every bin at or above its threshold, and no CTA's
    // threshold is above T1; not found: the estimate was too high)
    if (tid == 0) { misc[kMT1] = kBins; misc[kMAbove] = 0; misc[kMCntT1] = 0; misc[kMNinb] = 0; misc[kMKept] = 0; }
    cluster_sync();  // (1)
    if (normal && warp == 0) cluster_threshold(sup, hist, nctas, kk, misc + kMT1);
    if (warp == 1) {
        // any CTA's list overflowed, and the highest CTA threshold (T1 below it
        // means that CTA did not count every token of bin T1 and above)
        const int f = lane < nctas ? (int)ld_cluster_u32(cluster_addr(misc + kMOvf, lane)) : 0;
        int tmax = lane < nctas ? (int)ld_cluster_u32(cluster_addr(misc + kMTloc, lane)) : 0;
#pragma unroll
        for (int o = 16; o; o >>= 1) tmax = max(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
        const uint32_t any = __ballot_sync(0xffffffffu, f != 0);
        if (lane == 0) { misc[kMAnyOvf] = any != 0; misc[kMTmax] = tmax; }
    }
    __syncthreads();
    const int T1 = misc[kMT1], above1 = misc[kMAbove], cnt_T1 = misc[kMCntT1];
    int32_t *out = a.sel_idx + (int64_t)bh * a.cap_sel;
    // the kept tokens of this CTA are placed through a bitmap of its range
    // (after the in-bin lists in the idle ring); a range too long for it takes
    // the slow path
    uint4 *s_loc = reinterpret_cast<uint4 *>(ring);              // this CTA's in-bin tokens
    uint4 *s_inb = reinterpret_cast<uint4 *>(ring) + kInbinMax;  // the cluster's
    uint32_t *bmap = reinterpret_cast<uint32_t *>(ring + 2 * kInbinMax * 16);
    constexpr int kBmapWords = (SS::RING_B - 2 * kInbinMax * 16) / 4;
    const int nwords = (nloc + 31) / 32;
    // (the same decision in every CTA of the cluster: the bitmap bound uses the
    // longest range cta_range gives any CTA)
    const int64_t max_range = ceil_div(ceil_div(n, nctas), 64) * 64;
    // the attention list of this CTA (G > 0), in the candidate area once the
    // candidates are emitted: its kept middle tokens (after the sinks in CTA 0)
    int32_t *att_list = reinterpret_cast<int32_t *>(smem + StepLow::END);
    const int att_cap = (int)((recv_s - (smem_s + StepLow::END)) / 4u);
    int att_n = 0;
    const bool slow = !normal || T1 == kBins || T1 < misc[kMTmax] || misc[kMAnyOvf] != 0 || cnt_T1 > kInbinMax ||
                      ceil_div(max_range, 32) > kBmapWords || (G > 0 && kk + a.S > att_cap);

    if (!slow) {
        // ---- fast path: classify this warp's candidates (definite: bin > T1,
        // in the threshold bin: listed for the cluster)
        for (int x = tid; x < nwords; x += NT) bmap[x] = 0u;
        int ndef = 0;
        for (int jb = 0; jb < ncand; jb += 32) {
            const int jj = jb + lane;
            uint2 e = make_uint2(0u, 0u);
            if (jj < ncand) e = cand[jj];
            const int t = (int)(t0 + (int)e.x);
            const int bin = score_bin(key_to_float(e.y), inv2A);
            const bool inb = jj < ncand && bin == T1;
            const bool def = jj < ncand && bin > T1 && t >= s_end && t < w_beg;
            ndef += __popc(__ballot_sync(0xffffffffu, def)) * (lane == 0);
            const uint32_t ib = __ballot_sync(0xffffffffu, inb);
            if (ib) {
                int base = 0;
                if (lane == 0) base = atomicAdd(misc + kMNinb, __popc(ib));
                base = __shfl_sync(0xffffffffu, base, 0);
                const int slot = base + __popc(ib & lt);
                if (inb && slot < kInbinMax) s_loc[slot] = make_uint4(e.y, (uint32_t)t, (uint32_t)cta, 0u);
            }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) ndef += __shfl_xor_sync(0xffffffffu, ndef, o);
        if (lane == 0) s_wdef[warp] = ndef;
        __syncthreads();
        if (warp == 0) {  // publish (in-bin entries, definite middle tokens) into every CTA's s_cnt[cta]
            int dsum = lane < NWARP ? s_wdef[lane] : 0;
#pragma unroll
            for (int o = 16; o; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
            const int ni = min(misc[kMNinb], kInbinMax);
            if (lane < nctas) {
                st_cluster_u32(cluster_addr(&s_cnt[cta][0], lane), (uint32_t)ni);
                st_cluster_u32(cluster_addr(&s_cnt[cta][1], lane), (uint32_t)dsum);
            }
        }
        cluster_sync();  // (2)
        const int c1 = cnt_T1;
        {   // entry e of the cluster's in-bin list comes from the CTA whose list holds it
            const int ni = lane < nctas ? s_cnt[lane][0] : 0;
            int incl = ni;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const int excl = incl - ni;
            for (int e0 = warp * 32; e0 < c1; e0 += NT) {
                const int e = e0 + lane;
                int r = 0;
                for (int qq = 1; qq < nctas; ++qq) r = __shfl_sync(0xffffffffu, excl, qq) <= e ? qq : r;
                const int off = e - __shfl_sync(0xffffffffu, excl, r);
                if (e < c1) s_inb[e] = ld_cluster_v4(cluster_addr(s_loc + off, r));
            }
        }
        __syncthreads();
        cluster_arrive();  // (3): done with the other CTAs' shared memory
        // rank the in-bin list: the need1-th (score desc, token asc) is the last
        // selected; count the selected middle ones per CTA (output offsets)
        const int need1 = (int)kk - above1;
        if (c1 <= 32) {
            if (warp == 0) {
                const uint4 en = lane < c1 ? s_inb[lane] : make_uint4(0u, 0u, 0u, 0u);
                uint32_t Tkey = 0u;
                int IT = 0x7fffffff;
                if (need1 < c1) {
                    int rank = 0;
                    for (int f = 0; f < c1; ++f) {
                        const uint32_t kf = __shfl_sync(0xffffffffu, en.x, f);
                        const uint32_t tf = __shfl_sync(0xffffffffu, en.y, f);
                        rank += (kf > en.x) || (kf == en.x && tf < en.y);
                    }
                    const int src = __ffs(__ballot_sync(0xffffffffu, lane < c1 && rank == need1 - 1)) - 1;
                    Tkey = __shfl_sync(0xffffffffu, en.x, src);
                    IT = (int)__shfl_sync(0xffffffffu, en.y, src);
                }
                const int t = (int)en.y;
                const bool sel = lane < c1 && t >= s_end && t < w_beg && (en.x > Tkey || (en.x == Tkey && t <= IT));
                int mid = 0;
                for (int r = 0; r < nctas; ++r) {
                    const int cr = __popc(__ballot_sync(0xffffffffu, sel && (int)en.z == r));
                    if (lane == r) mid = s_cnt[r][1] + cr;
                }
                int before = lane < cta ? mid : 0, tot = mid;
#pragma unroll
                for (int o = 16; o; o >>= 1) {
                    before += __shfl_xor_sync(0xffffffffu, before, o);
                    tot += __shfl_xor_sync(0xffffffffu, tot, o);
                }
                if (lane == 0) { misc[kMTkey] = (int)Tkey; misc[kMIT] = IT; misc[kMBefore] = before; misc[kMTotal] = tot; }
            }
        } else {
            if (tid == 0) { misc[kMTkey] = 0; misc[kMIT] = 0x7fffffff; }
            if (tid < nctas) s_mid[tid] = s_cnt[tid][1];
            __syncthreads();
            if (need1 < c1) {
                for (int e = tid; e < c1; e += NT) {
                    const uint32_t ke = s_inb[e].x, ie = s_inb[e].y;
                    int rank = 0;
                    for (int f = 0; f < c1; ++f) {
                        const uint32_t kf = s_inb[f].x;
                        rank += (kf > ke) || (kf == ke && s_inb[f].y < ie);
                    }
                    if (rank == need1 - 1) { misc[kMTkey] = (int)ke; misc[kMIT] = (int)ie; }
                }
            }
            __syncthreads();
            const uint32_t Tkey = (uint32_t)misc[kMTkey];
            const int IT = misc[kMIT];
            for (int e = tid; e < c1; e += NT) {
                const uint4 en = s_inb[e];
                const int t = (int)en.y;
                if (t >= s_end && t < w_beg && (en.x > Tkey || (en.x == Tkey && t <= IT))) atomicAdd(&s_mid[en.z], 1);
            }
            __syncthreads();
            if (tid == 0) {
                int before = 0, tot = 0;
                for (int r = 0; r < nctas; ++r) {
                    before += r < cta ? s_mid[r] : 0;
                    tot += s_mid[r];
                }
                misc[kMBefore] = before;
                misc[kMTotal] = tot;
            }
        }
        __syncthreads();
        const uint32_t Tkey = (uint32_t)misc[kMTkey];
        const int IT = misc[kMIT];
        const int total_mid = misc[kMTotal];
        // kept middle tokens of this CTA into the bitmap, then written in
        // token order after those of CTAs < cta
        for (int jb = 0; jb < ncand; jb += 32) {
            const int jj = jb + lane;
            if (jj < ncand) {
                const uint2 e = cand[jj];
                const int t = (int)(t0 + (int)e.x);
                const int bin = score_bin(key_to_float(e.y), inv2A);
                if (t >= s_end && t < w_beg && (bin > T1 || (bin == T1 && (e.y > Tkey || (e.y == Tkey && t <= IT)))))
                    atomicOr(bmap + (e.x >> 5), 1u << (e.x & 31));
            }
        }
        __syncthreads();
        {
            const int per = (nwords + NT - 1) / NT;
            const int w0 = tid * per, w1 = min(nwords, w0 + per);
            int cnt = 0;
            for (int x = w0; x < w1; ++x) cnt += __popc(bmap[x]);
            int tot;
            const int lp = block_excl_scan<NT>(cnt, s_warp, &tot);
            int p = s_end + misc[kMBefore] + lp;
            int q = (cta == 0 ? s_end : 0) + lp;  // (the candidate lists are dead: the bitmap holds them)
            for (int x = w0; x < w1; ++x) {
                uint32_t m = bmap[x];
                while (m) {
                    const int bit = __ffs(m) - 1;
                    m &= m - 1;
                    const int32_t tok = (int32_t)(t0 + 32 * x + bit);
                    if (p < a.cap_sel) out[p] = tok;
                    if constexpr (G > 0) att_list[q] = tok;
                    ++p;
                    ++q;
                }
            }
            att_n = (cta == 0 ? s_end : 0) + tot;
            if constexpr (G > 0)
                if (cta == 0)
                    for (int x = tid; x < s_end; x += NT) att_list[x] = x;
        }
        {   // the sinks, the window and the padding, spread over the cluster's CTAs
            const int wpos0 = s_end + total_mid;
            const int nwin = (int)(n - w_beg);
            const int total = min(wpos0 + nwin, a.cap_sel);
            const int nall = s_end + nwin + (a.cap_sel - total);
            for (int x = cta * NT + tid; x < nall; x += nctas * NT) {
                if (x < s_end) {
                    out[x] = x;
                } else if (x < s_end + nwin) {
                    const int tw = x - s_end;
                    if (wpos0 + tw < a.cap_sel) out[wpos0 + tw] = w_beg + tw;
                } else {
                    out[total + (x - s_end - nwin)] = -1;
                }
            }
            if (cta == 0 && tid == 0) a.sel_cnt[bh] = total;
        }
        __syncthreads();  // the attention list is complete
        cluster_wait();  // (3): no CTA reads this one's ring any more
    } else {
        // ---- exact slow path (heavy ties, a full candidate list, a threshold
        // estimate above T1, or all / none selected): re-score the CTA's range
        // into the workspace rows counting every token (the stream counted
        // only those at or above its threshold; a token whose page is out of
        // range scores as the all-zero code, as in the two-kernel scorer), find
        // T1 from the full histograms, list the tokens of bins >= T1 per CTA,
        // and let CTA 0 resolve and emit.
        float *srow = a.ws.scores + (int64_t)bh * a.ws.ld;
        int32_t *cand = a.ws.cand + (int64_t)bh * a.ws.ld;
        int seg = 0;
        if (normal) {
            cluster_sync();  // (s1): no CTA reads the stream's counts any more
            for (int i = tid; i < kBins; i += NT) hist[i] = 0;
            if (tid < 64) sup[tid] = 0;
            if (tid == 0) { misc[kMT1] = kBins; misc[kMAbove] = 0; misc[kMCntT1] = 0; }
            __syncthreads();
            for (int64_t t = t0 + tid; t < t1; t += NT) {
                uint32_t w[BITS / 32];
                if (t == pos) {
#pragma unroll
                    for (int k = 0; k < BITS / 32; ++k) w[k] = newr[k];
                } else if (!load_code_plain<BITS>(kv, b, h, t, w)) {
#pragma unroll
                    for (int k = 0; k < BITS / 32; ++k) w[k] = 0u;
                }
                float sc = lut_score_any<BITS>(w, lut_s, t);
                if constexpr (RADIUS) sc = __fmul_rn(sc, radius_of_token(kv, b, h, t));
                srow[t] = sc;
                const int bin = score_bin(sc, inv2A);
                atomicAdd(&hist[bin], 1u);
                atomicAdd(&sup[bin >> 6], 1u);
            }
            cluster_sync();  // (s2): every CTA's full histogram
            if (warp == 0) cluster_threshold(sup, hist, nctas, kk, misc + kMT1);
            __syncthreads();
            const int T1s = misc[kMT1];
            // (each thread reads back the scores it wrote)
            for (int64_t base = t0; base < t1; base += NT) {
                const int64_t t = base + tid;
                const bool flag = t < t1 && score_bin(srow[t], inv2A) >= T1s;
                const uint32_t fb = __ballot_sync(0xffffffffu, flag);
                int tot;
                const int wex = block_excl_scan<NT>(lane == 0 ? __popc(fb) : 0, s_warp, &tot);
                const int wbase = __shfl_sync(0xffffffffu, wex, 0);
                if (flag) cand[t0 + seg + wbase + __popc(fb & lt)] = (int32_t)t;
                seg += tot;
            }
        }
        if (tid == 0) a.ws.seg_cnt[(int64_t)bh * kMaxSelCtas + cta] = seg;
        __threadfence();
        cluster_sync();  // (2s): segments complete
        if (cta == 0) {
            SelState st;
            st.T1 = misc[kMT1]; st.above1 = misc[kMAbove]; st.cnt_T1 = misc[kMCntT1];
            st.flags = n == 0 ? kStateEmpty : (normal ? kStateNormal : kStateAll);
            st.inv2A = inv2A; st.pad = 0.0f; st.kk = (int32_t)kk; st.n = (int32_t)n;
            resolve_emit<NT, 4096>(a.ws, bh, nctas, st, a.S, a.W, a.cap_sel, a.sel_idx, a.sel_cnt,
                                   *reinterpret_cast<ResolveSmem<4096> *>(lut));
        }
    }

    if constexpr (G > 0) {
        // ---- exact attention over this CTA's share of the selection: n_sl
        // tokens listed in att_list, then the nw window tokens wt0 + j, then
        // n_gl tokens of the global list gl (the slow path's share)
        int n_sl = 0, n_win = 0, n_gl = 0;
        const int32_t *gl = nullptr;
        if (!slow) {
            n_sl = att_n;
            n_win = nw;
        } else {
            cluster_sync();  // (4s): CTA 0's list and count are written (cluster-scope release / acquire)
            const int cnt = __ldcg(a.sel_cnt + bh);
            const int per = (cnt + nctas - 1) / nctas;
            const int r0 = min(cnt, cta * per), r1 = min(cnt, r0 + per);
            gl = a.sel_idx + (int64_t)bh * a.cap_sel + r0;
            n_gl = r1 - r0;
        }
        const int natt = n_sl + n_win + n_gl;
        auto token_of = [&](int r) -> int {
            if (r < n_sl) return att_list[r];
            if (r < n_sl + n_win) return (int)(wt0 + (r - n_sl));
            return __ldcg(gl + (r - n_sl - n_win));
        };
        // Lane l owns dims [DL l, DL l + DL) of every one of the G query heads,
        // and a tile is TR rows.  The G TR partial dot products of a tile are
        // summed over the warp by a transpose butterfly that leaves the one of
        // head lv / TR and row lv % TR (lv: the low log2(G TR) bits of l) in
        // lane l.  At the level that pairs lanes across bit k every lane sends
        // the upper half of its values and keeps the lower half; that is the
        // right half for both lanes because a lane keeps its heads and rows in
        // the order XOR-ed with lv (slot hh holds head hh ^ hperm, slot r row
        // r ^ rperm).
        constexpr int DL = D / 32;               // dims per lane
        constexpr int TR = G >= 4 ? 32 / G : 8;  // rows per tile
        constexpr int V = G * TR;                // partial products per lane
        constexpr int ROW_B = D * 2;
        constexpr int TILE_B = TR * 2 * ROW_B;
        constexpr int WSTAGE_B = 2 * TILE_B + 128;  // two tiles and 32 softmax weights per warp
        static_assert(G <= kMaxG && V <= 32 && (V & (V - 1)) == 0 && (DL == 2 || DL == 4), "tile shape");
        const int lv = lane & (V - 1);
        const int hperm = lv / TR, rperm = lv % TR;
        float qf[G][DL];
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
            const __nv_bfloat16 *qr = a.q + ((int64_t)b * a.Hq + (int64_t)h * G + (hh ^ hperm)) * D + DL * lane;
            if constexpr (DL == 4) {
                const uint2 w = *reinterpret_cast<const uint2 *>(qr);
                qf[hh][0] = bf16_lo(w.x) * a.scale_log2; qf[hh][1] = bf16_hi(w.x) * a.scale_log2;
                qf[hh][2] = bf16_lo(w.y) * a.scale_log2; qf[hh][3] = bf16_hi(w.y) * a.scale_log2;
            } else {
                const uint32_t w = *reinterpret_cast<const uint32_t *>(qr);
                qf[hh][0] = bf16_lo(w) * a.scale_log2; qf[hh][1] = bf16_hi(w) * a.scale_log2;
            }
        }
        float acc[G][DL];
#pragma unroll
        for (int hh = 0; hh < G; ++hh)
#pragma unroll
            for (int d = 0; d < DL; ++d) acc[hh][d] = 0.0f;
        float m = -INFINITY, lsum = 0.0f;  // of head hperm (the same in its TR lanes)
        const int ntiles = (natt + TR - 1) / TR;
        // two staging tiles per warp over the LUT and the code ring (both idle now)
        const uint32_t stage_s = lut_s + (uint32_t)(warp * WSTAGE_B);
        const unsigned char *stage = lut + warp * WSTAGE_B;
        float *s_p = reinterpret_cast<float *>(lut + warp * WSTAGE_B + 2 * TILE_B);  // [TR][G]
        const __nv_bfloat16 *kn_row = appending ? a.k_new + ((int64_t)b * kv.Hkv + h) * D : nullptr;
        const __nv_bfloat16 *vn_row = appending ? a.v_new + ((int64_t)b * kv.Hkv + h) * D : nullptr;
        // the rows of tile `tile` into buffer `buf` with 16-byte cp.async (one
        // commit group per call; rows that are not valid are zero-filled);
        // returns the valid-row mask
        constexpr int CPR = 2 * ROW_B / 16;  // 16-byte chunks per row (K then V)
        constexpr int RPI = 32 / CPR;        // rows per warp-wide copy
        static_assert(CPR * RPI == 32 && TR % RPI == 0, "copy shape");
        // dense rows of (b, h): token t's K / V row starts at element rbase + t D
        const int64_t rbase = ((int64_t)b * kv.Hkv + h) * kv.n_cap * D;
        auto fetch = [&](int tile, int buf) -> uint32_t {
            // lanes < TR resolve row tile TR + lane: PAGED the element offset of
            // the row, dense the token; -2: the appended token, -1: none
            int64_t key = -1;
            if (lane < TR) {
                const int r = tile * TR + lane;
                if (r < natt) {
                    const int tok = token_of(r);
                    if (tok < 0 || tok >= capn) {
                        raise_error(kErrCapacity);
                    } else if (tok == pos) {
                        key = -2;
                    } else if constexpr (PAGED) {
                        key = kv.row(b, h, tok);  // (-1: page out of range)
                    } else {
                        key = tok;
                    }
                }
            }
            const uint32_t vm = __ballot_sync(0xffffffffu, key != -1);
            const int c = lane % CPR;  // this lane's chunk of its row
            const bool isv = c >= CPR / 2;
            const int ce = (isv ? c - CPR / 2 : c) * 8;  // first element of the chunk
            const __nv_bfloat16 *cache = isv ? kv.v : kv.k;
            const __nv_bfloat16 *fresh = (isv ? vn_row : kn_row) + ce;
#pragma unroll 1
            for (int i = 0; i < TR / RPI; ++i) {
                const int r = i * RPI + lane / CPR;
                int64_t o;
                if constexpr (PAGED) {
                    o = __shfl_sync(0xffffffffu, key, r);
                } else {
                    const int tk = __shfl_sync(0xffffffffu, (int)key, r);
                    o = tk >= 0 ? rbase + (int64_t)tk * D : tk;
                }
                const __nv_bfloat16 *src = o >= 0 ? cache + o + ce : (o == -2 ? fresh : kv.k);
                const uint32_t sz = o != -1 ? 16u : 0u;  // (zero-filled when not valid)
                const uint32_t dst = stage_s + (uint32_t)(buf * TILE_B + r * 2 * ROW_B + c * 16);
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(sz) : "memory");
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
            return vm;
        };
        // this lane's DL dims of a staged bf16 row
        auto load_row = [&](const unsigned char *row, float (&f)[DL]) {
            if constexpr (DL == 4) {
                const uint2 w = *reinterpret_cast<const uint2 *>(row + lane * 8);
                f[0] = bf16_lo(w.x); f[1] = bf16_hi(w.x); f[2] = bf16_lo(w.y); f[3] = bf16_hi(w.y);
            } else {
                const uint32_t w = *reinterpret_cast<const uint32_t *>(row + lane * 4);
                f[0] = bf16_lo(w); f[1] = bf16_hi(w);
            }
        };
        int k = 0;
        // two commit groups in flight per lane (empty ones past the last tile);
        // vm0 / vm1: the valid-row masks of the tiles in buffers k & 1 = 0 / 1
        uint32_t vm0 = warp < ntiles ? fetch(warp, 0) : 0u;
        uint32_t vm1 = warp + NWARP < ntiles ? fetch(warp + NWARP, 1) : 0u;
        if (warp >= ntiles) asm volatile("cp.async.commit_group;" ::: "memory");
        if (warp + NWARP >= ntiles) asm volatile("cp.async.commit_group;" ::: "memory");
        for (int tile = warp; tile < ntiles; tile += NWARP, ++k) {
            const int buf = k & 1;
            asm volatile("cp.async.wait_group 1;" ::: "memory");  // this tile's group has landed
            __syncwarp();  // (and every lane's copies are visible to the warp)
            const unsigned char *tb = stage + buf * TILE_B;
            const uint32_t vm = buf ? vm1 : vm0;
            // partial q . k of (slot head hh, slot row r); rows that are not
            // valid are zeros and masked below
            float x[V];
#pragma unroll
            for (int r = 0; r < TR; ++r) {
                float kf[DL];
                load_row(tb + (r ^ rperm) * 2 * ROW_B, kf);
#pragma unroll
                for (int hh = 0; hh < G; hh += 2) {
                    if constexpr (G == 1) {
                        float s = 0.0f;
#pragma unroll
                        for (int d = 0; d < DL; ++d) s = fmaf(qf[0][d], kf[d], s);
                        x[r] = s;
                    } else {
                        float2 s2 = make_float2(0.0f, 0.0f);
#pragma unroll
                        for (int d = 0; d < DL; ++d)
                            s2 = ffma2(make_float2(qf[hh][d], qf[hh + 1][d]), make_float2(kf[d], kf[d]), s2);
                        x[hh * TR + r] = s2.x;
                        x[(hh + 1) * TR + r] = s2.y;
                    }
                }
            }
#pragma unroll
            for (int half = V / 2; half >= 1; half >>= 1)
#pragma unroll
                for (int i = 0; i < half; ++i) x[i] += __shfl_xor_sync(0xffffffffu, x[i + half], half);
#pragma unroll
            for (int o = 16; o >= V; o >>= 1) x[0] += __shfl_xor_sync(0xffffffffu, x[0], o);
            // online softmax of head hperm over the tile's rows (its TR lanes)
            const bool ok = (vm >> rperm) & 1u;
            const float sc = ok ? x[0] : -INFINITY;
            float tmax = sc;
#pragma unroll
            for (int o = TR / 2; o; o >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
            const float mn = fmaxf(m, tmax);
            const float c = m == -INFINITY ? 0.0f : fast_exp2(m - mn);
            const float pv = ok ? fast_exp2(sc - mn) : 0.0f;
            float ps = pv;
#pragma unroll
            for (int o = TR / 2; o; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
            lsum = fmaf(lsum, c, ps);
            m = mn;
            if (lane < V) s_p[rperm * G + hperm] = pv;
            float ch[G];
#pragma unroll
            for (int hh = 0; hh < G; ++hh) ch[hh] = __shfl_sync(0xffffffffu, c, hh * TR);
            __syncwarp();
#pragma unroll
            for (int hh = 0; hh < G; ++hh)
#pragma unroll
                for (int d = 0; d < DL; ++d) acc[hh][d] *= ch[hh];
#pragma unroll 2
            for (int r = 0; r < TR; ++r) {
                // (rows that are not valid are zeros with weight 0)
                float vf[DL];
                load_row(tb + r * 2 * ROW_B + ROW_B, vf);
                float p[G];
#pragma unroll
                for (int hh = 0; hh < G; hh += 4) {
                    if constexpr (G >= 4) {
                        const float4 p4 = *reinterpret_cast<const float4 *>(s_p + r * G + hh);
                        p[hh] = p4.x; p[hh + 1] = p4.y; p[hh + 2] = p4.z; p[hh + 3] = p4.w;
                    } else {
#pragma unroll
                        for (int u = 0; u < G; ++u) p[u] = s_p[r * G + u];
                    }
                }
#pragma unroll
                for (int hh = 0; hh < G; ++hh)
#pragma unroll
                    for (int d = 0; d < DL; d += 2) {
                        const float2 a2 = ffma2(make_float2(p[hh], p[hh]), make_float2(vf[d], vf[d + 1]),
                                                make_float2(acc[hh][d], acc[hh][d + 1]));
                        acc[hh][d] = a2.x;
                        acc[hh][d + 1] = a2.y;
                    }
            }
            __syncwarp();  // the weights and the buffer are refilled next
            if (tile + 2 * NWARP < ntiles) {
                const uint32_t v = fetch(tile + 2 * NWARP, buf);
                if (buf) vm1 = v; else vm0 = v;
            } else {
                asm volatile("cp.async.commit_group;" ::: "memory");
            }
        }
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncthreads();  // every warp is done with its staging buffers
        // CTA merge of the warps' states: [warp][G] (m, l) and [warp][G][D] acc at the LUT base
        float *s_acc = reinterpret_cast<float *>(lut);
        float *s_ml = s_acc + NWARP * G * D;
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
            const float mh = __shfl_sync(0xffffffffu, m, hh * TR);
            const float lh = __shfl_sync(0xffffffffu, lsum, hh * TR);
            if (lane == 0) { s_ml[(warp * G + hh) * 2] = mh; s_ml[(warp * G + hh) * 2 + 1] = lh; }
#pragma unroll
            for (int d = 0; d < DL; ++d) s_acc[(warp * G + hh) * D + DL * lane + d] = acc[hh][d];
        }
        __syncthreads();
        // this CTA's partial (M, L, A) per query head g and dim i, element
        // x = g D + i: A goes to the CTA that merges x (x mod C, slot
        // [cta][x / C] of its inbox), every CTA gets each head's (M, L)
        float *recv_acc = reinterpret_cast<float *>(smem + (recv_s - smem_s));  // [C][slots]
        float *recv_ml = recv_acc + kRecvAccFloats;                              // [C][G][2]
        const int slots = (G * D + nctas - 1) / nctas;
        for (int x2 = tid; x2 < G * D; x2 += NT) {
            const int gg = x2 / D, i = x2 % D;
            float M = -INFINITY;
            for (int w2 = 0; w2 < NWARP; ++w2) M = fmaxf(M, s_ml[(w2 * G + gg) * 2]);
            float L = 0.0f, A = 0.0f;
            if (M != -INFINITY) {
                for (int w2 = 0; w2 < NWARP; ++w2) {
                    const float c = fast_exp2(s_ml[(w2 * G + gg) * 2] - M);
                    L = fmaf(s_ml[(w2 * G + gg) * 2 + 1], c, L);
                    A = fmaf(s_acc[(w2 * G + gg) * D + i], c, A);
                }
            }
            st_cluster_f32(cluster_addr(recv_acc + cta * slots + x2 / nctas, x2 % nctas), A);
            if (i == 0)
                for (int r = 0; r < nctas; ++r) {
                    st_cluster_f32(cluster_addr(recv_ml + (cta * G + gg) * 2, r), M);
                    st_cluster_f32(cluster_addr(recv_ml + (cta * G + gg) * 2 + 1, r), L);
                }
        }
        cluster_sync();  // (5): every partial is in its merging CTA's inbox
        // the cluster merge of the elements this CTA owns (from its inbox only)
        for (int x2 = cta + nctas * tid; x2 < G * D; x2 += nctas * NT) {
            const int gg = x2 / D, i = x2 % D;
            float M = -INFINITY;
            for (int r = 0; r < nctas; ++r) M = fmaxf(M, recv_ml[(r * G + gg) * 2]);
            float L = 0.0f, A = 0.0f;
            if (M != -INFINITY) {
                for (int r = 0; r < nctas; ++r) {
                    const float c = fast_exp2(recv_ml[(r * G + gg) * 2] - M);
                    L = fmaf(recv_ml[(r * G + gg) * 2 + 1], c, L);
                    A = fmaf(recv_acc[r * slots + x2 / nctas], c, A);
                }
            }
            const int64_t oq = (int64_t)b * a.Hq + (int64_t)h * G + gg;
            a.out[oq * D + i] = L > 0.0f ? A / L : 0.0f;
            if (i == 0 && a.lse) a.lse[oq] = L > 0.0f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
        }
    }
    if (appending && cta == 0 && tid == 0) {
        // every CTA of this cluster read seq_lens[b] before barrier (1); the last
        // cluster of the sequence to get here moves its length on
        __threadfence();
        const uint32_t old = atomicAdd(a.seq_arrive + (int64_t)b * kSyncStride, 1u);
        if (old == (uint32_t)(kv.Hkv - 1)) {
            a.seq_arrive[(int64_t)b * kSyncStride] = 0;
            if (app_ok) a.seq_lens[b] = (int32_t)(pos + 1);
        }
    }
}

}  // namespace dkv
