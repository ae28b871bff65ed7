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
// Kernels here (grid = (CTAs per (b, h), B * Hkv)): the two-kernel selection,
// used without cluster launch support or on request --
//   score_hist_kernel  scores every token, builds the 4096-bin histogram over
//                      [-A, A] (A = sum_j |Qp_j| bounds every |s_t|); the last
//                      CTA of a (b, h) (atomic arrival counter, which it
//                      resets: the workspace is left clean) finds the bin T1
//                      holding the k-th largest score;
//   collect_kernel     compacts the tokens with bin >= T1 into per-CTA
//                      segments; its last CTA resolves the threshold bin
//                      exactly and writes the selection.  No CTA waits for
//                      another.
// The clustered selection (step.cuh) shares the scorer, the threshold search
// over distributed shared memory and the exact resolver below.
#pragma once
#include "common.cuh"

namespace dkv {

constexpr int kBins = 4096;
constexpr float kRadiusMax = 63.875f;  // largest radius r~ = (255 + 1/2) / 4
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
    uint32_t *arrive;    // [2][BH] x kSyncStride   zero between calls
    int32_t *seg_cnt;    // [BH][kMaxSelCtas]
    uint32_t *ckey;      // [BH][ld] order keys of spilled candidates (fused selection)
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
// One CTA of 1024 threads per SM.  The byte-LUT (256 rows x 256 B; word j of
// row v holds LUT_{j mod T}[v], j = 0..63) sits at a shared address whose low
// 16 bits are zero.  Lane l handles tokens t = l (mod 32), stored rotated by
// t mod T (stored byte r = code byte (r + l) mod T), so at step r it needs
// table (l + r) mod T, i.e. word l + r of the row of its byte.  One
// byte-permute of (code word, lane base) yields the row address
//   lut_base | byte << 8 | 4 l
// and the load adds the immediate 4 r: one permute, one load and one add per
// byte, with a single per-lane register.  At each step the 32 lanes read
// words l + r of their rows: 32 distinct banks.
constexpr int kScoreThreads = 1024;
constexpr int kScoreThreadsConst = kScoreThreads;

template <int BITS>
struct ScoreShape {
    static constexpr int T = BITS / 8;         // byte tables
    static constexpr int NW = BITS / 32;       // 32-bit code words per token
    static constexpr uint32_t LUT_BYTES = 256 * 256;
    static constexpr uint32_t SCRATCH_BYTES = kBins * 4 + (kMaxDim + kMaxBits + 64) * 4;  // hist + scratch
    static constexpr uint32_t LOW_BYTES = SCRATCH_BYTES;
    using Vec = typename std::conditional<BITS == 128, uint4, uint2>::type;  // one token's code
    // per-thread cp.async ring of upcoming codes (one token per thread per stage)
    static constexpr int STAGES = 5;
    static constexpr uint32_t RING_BYTES = STAGES * kScoreThreadsConst * sizeof(Vec);
    // dynamic smem: low region, the LUT at the next 64 KB boundary, then the ring
    static constexpr size_t SMEM = 2 * 65536 + RING_BYTES;
};

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

// Shared-memory load from a 32-bit shared address plus the byte offset IMM.
// Not volatile: its address always depends on code words loaded after the
// barrier that publishes the LUT, so it cannot be scheduled before it.
template <int IMM>
__device__ __forceinline__ float lds_f32(uint32_t addr) {
    float v;
    asm("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(addr), "n"(IMM));
    return v;
}

// Packed fp32 add (two lanes of fp32 per instruction on sm_100), each lane
// rounded once like a scalar add.
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// Table entry of stored byte r of a (rotated) code for the lane whose row
// address base is `base` (see the scorer below).
template <int BITS, int r>
__device__ __forceinline__ float lut_term(const uint32_t (&w)[BITS / 32], uint32_t base) {
    return lds_f32<4 * r>(__byte_perm(w[r >> 2], base, 0x7604u | ((uint32_t)(r & 3) << 4)));
}

// Terms (r, r + 1) for r = 0, 2, .. R - 2 of a score: even bytes into s.x, odd
// bytes into s.y (each chain ascending), one packed add per pair.
template <int BITS, int R>
struct LutPairs {
    static __device__ __forceinline__ void add(const uint32_t (&w)[BITS / 32], uint32_t base, float2 &s) {
        LutPairs<BITS, R - 2>::add(w, base, s);
        s = fadd2(s, make_float2(lut_term<BITS, R - 2>(w, base), lut_term<BITS, R - 1>(w, base)));
    }
};
template <int BITS>
struct LutPairs<BITS, 0> {
    static __device__ __forceinline__ void add(const uint32_t (&)[BITS / 32], uint32_t, float2 &) {}
};

// Score of one (rotated) code: sum over its T bytes of the lane's table
// entries, the even and the odd bytes in two chains, then the chains added.
template <int BITS>
__device__ __forceinline__ float lut_score(const uint32_t (&w)[BITS / 32], uint32_t base) {
    float2 s = make_float2(0.0f, 0.0f);
    LutPairs<BITS, BITS / 8>::add(w, base, s);
    return (s.x + s.y) + 0.0f;  // + 0 turns a -0 into +0
}

// ---------------------------------------------------------------------------
// Score phase shared by the fused and the two-kernel selection: LUT prologue
// (depends on q only, so it runs before waiting on the preceding kernel), then
// stream this CTA's codes, write the fp32 scores and build the CTA histogram
// in shared memory.  Ends with the histogram complete (after a barrier).
struct ScoreOut {
    int64_t n, t0, t1;
    int R;               // tokens per warp range (multiple of 32)
    float inv2A;
    unsigned char *lut;  // 64 KB LUT region, free for reuse once scoring is done
};

// RADIUS: radius-scaled scores s' = r~ s (Spherical KV page, section 2.1 ADA: a
// quantized key radius beside the angle code scales the logit), r~ = (c + 1/2)/4
// from the token's 8-bit code c in kv.radius; the bins span r~_max times the
// unscaled range.
template <int BITS, int D, bool PAGED, bool RADIUS = false>
__device__ __forceinline__ ScoreOut score_phase(const KV &kv, const __nv_bfloat16 *__restrict__ q, int Hq, int G,
                                                const int32_t *__restrict__ seq_lens, const RBits &R,
                                                const SelWS &ws, int nctas, unsigned char *smem) {
    using S = ScoreShape<BITS>;
    using Vec = typename S::Vec;
    constexpr int T = S::T, NW = S::NW;
    constexpr int NWARPS = kScoreThreads / 32;
    uint32_t *hist = reinterpret_cast<uint32_t *>(smem);                  // [kBins]
    float *qsum = reinterpret_cast<float *>(hist + kBins);                // [D]
    float *Qp = qsum + kMaxDim;                                           // [BITS]
    float *red = Qp + kMaxBits;                                           // [64]
    const uint32_t smem_s = (uint32_t)__cvta_generic_to_shared(smem);
    const uint32_t lut_s = (smem_s + S::LOW_BYTES + 65535u) & ~65535u;     // 64 KB aligned
    unsigned char *lut = smem + (lut_s - smem_s);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bh = blockIdx.y, b = bh / kv.Hkv, h = bh % kv.Hkv;

    // this warp's words of R (hyperplanes warp + NWARPS m): issued first, so their
    // parameter-block misses overlap the loads of q
    static_assert(BITS % NWARPS == 0, "hyperplanes per warp");
    uint32_t rw[BITS / NWARPS][D / 32];
#pragma unroll
    for (int m = 0; m < BITS / NWARPS; ++m)
#pragma unroll
        for (int k = 0; k < D / 32; ++k) rw[m][k] = R.w[(warp + NWARPS * m) * (D / 32) + k];
    for (int i = tid; i < kBins; i += kScoreThreads) hist[i] = 0;
    for (int i = tid; i < D; i += kScoreThreads) {
        const __nv_bfloat16 *qh = q + ((int64_t)b * Hq + (int64_t)h * G) * D + i;
        float s = 0.0f;
        for (int g = 0; g < G; ++g) s += __bfloat162float(qh[(int64_t)g * D]);
        qsum[i] = s;
    }
    __syncthreads();
    // Qp_j = sum_i R[j][i] qsum[i]: warp w takes hyperplanes w, w + NWARPS, ...
    // and lane l the dims l, l + 32, ...; a whole warp then reads the same word of
    // R at a time (a broadcast from the parameter block), and a shuffle tree sums
    // the lanes.
#pragma unroll
    for (int m = 0; m < BITS / NWARPS; ++m) {
        float acc = 0.0f;
#pragma unroll
        for (int k = 0; k < D / 32; ++k) acc = fmaf(((rw[m][k] >> lane) & 1u) ? -1.0f : 1.0f, qsum[32 * k + lane], acc);
#pragma unroll
        for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) Qp[warp + NWARPS * m] = acc;
    }
    __syncthreads();
    if (warp == 0) {
        float a = 0.0f;
        for (int j = lane; j < BITS; j += 32) a += fabsf(Qp[j]);
#pragma unroll
        for (int o = 16; o; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        if (RADIUS) a *= kRadiusMax;
        if (lane == 0) red[0] = a > 0.0f ? 0.5f / a : 0.0f;
    }
    // LUT rows: word j of row v holds LUT_{j mod T}[v]; lane l fills words l and
    // l + 32 (both table l mod T, as 32 is a multiple of T).  Warp w owns the
    // 256 / NWARPS consecutive rows from v0 = w * 256 / NWARPS (low bits zero):
    // row v0 is the full signed sum, each other row adds 2 qv[u] for the low
    // bits u it sets.
    {
        static_assert(256 % NWARPS == 0 && (256 / NWARPS) <= 8, "rows per warp");
        constexpr int RPW = 256 / NWARPS;
        const int c = lane % T;
        float qv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) qv[u] = Qp[8 * c + u];
        const int v0 = warp * RPW;
        float base = 0.0f;
#pragma unroll
        for (int u = 0; u < 8; ++u) base += ((v0 >> u) & 1) ? qv[u] : -qv[u];
#pragma unroll
        for (int d = 0; d < RPW; ++d) {
            float val = base;
#pragma unroll
            for (int u = 0; u < 3; ++u)
                if ((d >> u) & 1) val += 2.0f * qv[u];
            float *row = reinterpret_cast<float *>(lut + (v0 + d) * 256);
            row[lane] = val;
            row[lane + 32] = val;
        }
    }
    __syncthreads();
    ScoreOut o;
    o.inv2A = red[0];
    o.lut = lut;
    // everything above depends on q only; codes and lengths come from the append
    griddep_wait();
    o.n = clamp_len(kv, seq_lens, b);
    cta_range(o.n, blockIdx.x, nctas, o.t0, o.t1);
    const int64_t t0 = o.t0, t1 = o.t1;
    const float inv2A = o.inv2A;

    // Lane l always handles tokens with t % 32 == l, whose stored bytes are
    // rotated by l % T (see store_code_rotated): at step r it reads stored byte
    // r, which is code byte (r + l) % T, from word l + r of the byte's LUT row.
    const uint32_t lbase = lut_s | 4u * (uint32_t)lane;  // row address = lbase | byte << 8

    const int nloc = (int)(t1 - t0);  // tokens of this CTA (< 2^31)
    // Warp w streams the contiguous range [w R, (w + 1) R) of the CTA's tokens,
    // 32 at a time (lane = token), so its scores come out in token order.
    constexpr int NWARP = kScoreThreads / 32;
    const int wlen = (int)(ceil_div(ceil_div(nloc, NWARP), 32) * 32);
    o.R = wlen;
    const int wb = warp * wlen;                               // warp's first local token
    const int we = min(nloc, wb + wlen);                      // one past its last
    const int nk = we > wb ? (we - wb + 31) / 32 : 0;         // 32-token steps of this warp
    // Each thread streams its tokens through its own slots of a STAGES-deep
    // cp.async ring: it only ever reads codes it copied itself, so the ring needs
    // no barriers, and STAGES - 1 codes per thread stay in flight.
    constexpr int NT = kScoreThreads;
    constexpr int STAGES = S::STAGES;
    constexpr int VB = (int)sizeof(Vec);
    const uint32_t ring_s = lut_s + 65536u + (uint32_t)tid * VB;  // this thread's slot of stage 0
    const unsigned char *ring = lut + 65536 + tid * VB;
    const Vec *dense = reinterpret_cast<const Vec *>(kv.codes) + ((int64_t)bh * kv.n_cap + t0);
    float *srow = ws.scores + (int64_t)bh * ws.ld + t0;
    // Step k copies token wb + 32 k + lane into ring slot k % STAGES; the loop
    // is unrolled by STAGES so every slot (and its shared address) is a
    // compile-time constant, and the positions advance by 32 tokens per step.
    // PAGED: a step's 32 tokens lie in one page (t0 and the warp ranges are
    // multiples of 32, pages hold a multiple of 32 tokens), so its physical page
    // is one warp-wide load, made one step before the copy that needs it.
    auto page_of_step = [&](int k) -> int64_t {  // -1: no tokens; -2: page id out of range
        const int i = wb + 32 * k;
        if (k >= nk || i >= we) return -1;
        const int64_t t = t0 + i;
        const int32_t p = __ldg(kv.page_table + (int64_t)b * kv.max_pages + t / kv.page_size);
        return (p < 0 || p >= kv.num_pages) ? -2 : (int64_t)p;
    };
    auto issue = [&](int k, int slot, int64_t pg) {  // copy the code of token wb + 32 k + lane into `slot`
        const int i = wb + 32 * k + lane;
        const void *src = dense;
        int bytes = 0;
        if (k < nk && i < we) {
            if (!PAGED) {
                src = dense + i;
                bytes = VB;
            } else if (pg >= 0) {
                const int64_t t = t0 + i;
                src = kv.codes + ((pg * kv.Hkv + h) * kv.page_size + t % kv.page_size) * kv.W;
                bytes = VB;
            } else if (pg == -2) {
                raise_error(kErrPage);
            }
        }
        const uint32_t dst = ring_s + (uint32_t)(slot * NT * VB);
        if (VB == 16)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes) : "memory");
        else
            asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(dst), "l"(src), "r"(bytes) : "memory");
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    // r~ of token wb + 32 k + lane (read one step ahead of its use), 0 outside
    auto radius_of = [&](int k) -> float {
        const int i = wb + 32 * k + lane;
        if (k >= nk || i >= we) return 0.0f;
        const int64_t r = kv.radius_index(b, h, t0 + i);
        return r >= 0 ? ((float)__ldg(kv.radius + r) + 0.5f) * 0.25f : 0.0f;
    };
    float rnext = 0.0f;
    if constexpr (RADIUS) rnext = radius_of(0);
#pragma unroll
    for (int k = 0; k < STAGES - 1; ++k) issue(k, k, PAGED ? page_of_step(k) : 0);
    int64_t pg_next = PAGED ? page_of_step(STAGES - 1) : 0;  // page of the next step to be issued
    for (int k0 = 0; k0 < nk; k0 += STAGES) {
#pragma unroll
        for (int u = 0; u < STAGES; ++u) {
            const int k = k0 + u;
            if (k >= nk) break;
            const int64_t pg = pg_next;
            if constexpr (PAGED) pg_next = page_of_step(k + STAGES);
            issue(k + STAGES - 1, (u + STAGES - 1) % STAGES, pg);
            float rcur = 0.0f;
            if constexpr (RADIUS) {
                rcur = rnext;
                rnext = radius_of(k + 1);
            }
            asm volatile("cp.async.wait_group %0;" ::"n"(STAGES - 1) : "memory");
            const int i = wb + 32 * k + lane;
            const Vec code = *reinterpret_cast<const Vec *>(ring + u * NT * VB);
            int bin = 0;
            if (i < we) {
                uint32_t w[NW];
                unpack_code<BITS>(code, w);
                float sc = lut_score<BITS>(w, lbase);
                if constexpr (RADIUS) sc = __fmul_rn(sc, rcur);  // one rounding, as the definition
                srow[i] = sc;
                bin = score_bin(sc, inv2A);
                atomicAdd(&hist[bin], 1u);
            }
        }
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    return o;
}

// Optional user copy of the scores: entries [0, seq_lens[b] >> len_shift) of
// every row.
static __global__ void copy_scores_kernel(const float *__restrict__ src, int64_t ld, float *__restrict__ dst, int64_t ld_out,
                                   const int32_t *__restrict__ seq_lens, int Hkv, int64_t cap, int len_shift) {
    griddep_wait();
    const int bh = blockIdx.y;
    int64_t n = seq_lens[bh / Hkv] >> len_shift;
    if (n > cap) n = cap;
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < n; t += (int64_t)gridDim.x * blockDim.x)
        dst[(int64_t)bh * ld_out + t] = src[(int64_t)bh * ld + t];
}

// Threshold bin from a complete histogram in shared memory: the bin T1 that
// holds the kk-th largest score, the count above it and in it.  All threads
// call; the results land in out[0..2] (shared).  Requires 0 < kk < total.
template <int NT>
__device__ __forceinline__ void threshold_bin(const uint32_t *hist, int64_t kk, int *s_warp, int *out) {
    constexpr int PER = kBins / NT;  // bins per thread, thread 0 owns the top
    const int tid = threadIdx.x;
    int local = 0;
    const int top = kBins - 1 - tid * PER;
#pragma unroll
    for (int e = 0; e < PER; ++e) local += hist[top - e];
    int total;
    const int before = block_excl_scan<NT>(local, s_warp, &total);
    if (before < kk && before + local >= kk) {
        int run = before;
        for (int e = 0; e < PER; ++e) {
            const int bin = top - e;
            if (run + (int)hist[bin] >= kk) {
                out[0] = bin;
                out[1] = run;
                out[2] = (int)hist[bin];
                break;
            }
            run += hist[bin];
        }
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------
// Two-kernel selection, first kernel: score + histogram; the last CTA of a
// (b, h) (arrival counter, no waiting) locates the threshold bin.
template <int BITS, int D, bool PAGED>
__global__ void __launch_bounds__(kScoreThreads, 1)
score_hist_kernel(KV kv, const __nv_bfloat16 *__restrict__ q, int Hq, int G,
                  const int32_t *__restrict__ seq_lens, const RBits R, SelWS ws, int topk, int nctas) {
    extern __shared__ __align__(1024) unsigned char smem[];
    __shared__ int s_last;
    __shared__ int s_warp[32];
    __shared__ int s_thr[4];
    const int tid = threadIdx.x;
    const int bh = blockIdx.y;
    const ScoreOut so = score_phase<BITS, D, PAGED>(kv, q, Hq, G, seq_lens, R, ws, nctas, smem);
    uint32_t *hist = reinterpret_cast<uint32_t *>(smem);
    griddep_trigger();
    uint32_t *ghist = ws.hist + (int64_t)bh * kBins;
    for (int k = tid; k < kBins; k += kScoreThreads)
        if (hist[k]) atomicAdd(ghist + k, hist[k]);
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(ws.arrive + (int64_t)kSyncStride * bh, 1u) == (unsigned)(nctas - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int k = tid; k < kBins; k += kScoreThreads) {
        hist[k] = __ldcg(ghist + k);
        ghist[k] = 0;
    }
    if (tid == 0) { s_thr[0] = kBins; s_thr[1] = 0; s_thr[2] = 0; }
    __syncthreads();
    const int64_t n = so.n;
    const int64_t kk = topk < n ? topk : n;
    if (n > 0 && kk < n) threshold_bin<kScoreThreads>(hist, kk, s_warp, s_thr);
    if (tid == 0) {
        SelState st;
        st.inv2A = so.inv2A; st.pad = 0.0f; st.kk = (int32_t)kk; st.n = (int32_t)n;
        st.T1 = s_thr[0]; st.above1 = s_thr[1]; st.cnt_T1 = s_thr[2];
        st.flags = n == 0 ? kStateEmpty : (kk >= n ? kStateAll : kStateNormal);
        ws.state[bh] = st;
        ws.arrive[(int64_t)kSyncStride * bh] = 0;
    }
}

// ---------------------------------------------------------------------------
// Resolve + emit (one CTA of NT threads per (b, h)).
//
// The candidate list of a (b, h) is the concatenation, in CTA order, of every
// scoring CTA's segment (tokens of its range with bin >= T1, ascending), so the
// list is in ascending token order.  The resolver addresses it through a
// ListView: either a shared-memory copy (tokens + order keys) or, when the
// list is too long for that, the segments in global memory.
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

// For every list element in order, pred(t, key) -> keep; emit(rank, t) for the
// kept ones in list order.  Each thread owns a contiguous run of elements so one
// block scan orders everything.  Returns the number kept.
template <int NT, class Pred, class Emit>
__device__ __forceinline__ int ordered_pass(const ListView &L, int M, int *s_warp, Pred &&pred, Emit &&emit) {
    const int per = (M + NT - 1) / NT;
    const int e0 = threadIdx.x * per;
    const int e1 = min(M, e0 + per);
    int cnt = 0;
    for (int e = e0; e < e1; ++e) {
        int t; uint32_t key;
        L.get(e, t, key);
        cnt += pred(t, key) ? 1 : 0;
    }
    int total;
    int r = block_excl_scan<NT>(cnt, s_warp, &total);
    if (cnt)
        for (int e = e0; e < e1; ++e) {
            int t; uint32_t key;
            L.get(e, t, key);
            if (pred(t, key)) emit(r++, t);
        }
    return total;
}

template <int LIST_CAP>
struct ResolveSmem {
    int32_t list_t[LIST_CAP];
    uint32_t list_key[LIST_CAP];
    uint32_t ck[kCandSmem];
    int32_t ci[kCandSmem];
    uint32_t h[2048];
    int seg_off[kMaxSelCtas + 1];
    int warp[32];
    int misc[8];
    int last;
};

// Exact threshold (Tkey, IT) inside bin T1, then the final ascending selection.
// seg_cnt: the per-CTA segment sizes of this (b, h) in global memory.
template <int NT, int LIST_CAP>
__device__ void resolve_emit(const SelWS &ws, int bh, int nctas, const SelState &st, int S, int W, int cap_sel,
                             int32_t *sel_idx, int32_t *sel_cnt, ResolveSmem<LIST_CAP> &sm) {
    const int tid = threadIdx.x;
    const int n = st.n;
    const int32_t *cand = ws.cand + (int64_t)bh * ws.ld;
    const float *srow = ws.scores + (int64_t)bh * ws.ld;
    {
        const int c = tid;
        const int v = c < nctas ? __ldcg(ws.seg_cnt + (int64_t)bh * kMaxSelCtas + c) : 0;
        int tot;
        const int ex = block_excl_scan<NT>(v, sm.warp, &tot);
        if (c < nctas) sm.seg_off[c] = ex;
        if (c == 0) sm.seg_off[nctas] = tot;
    }
    __syncthreads();
    const int M = sm.seg_off[nctas];
    ListView L{nullptr, nullptr, cand, srow, sm.seg_off, nctas, n};
    if (st.flags == kStateNormal && M <= LIST_CAP) {
        for (int e = tid; e < M; e += NT) {  // one parallel round over the whole list
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
            for (int e = tid; e < M; e += NT) {
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
            for (int e = tid; e < c1; e += NT) {
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
                for (int i = tid; i < 2048; i += NT) sm.h[i] = 0;
                __syncthreads();
                for (int e = tid; e < M; e += NT) {
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
            ordered_pass<NT>(L, M, sm.warp,
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
        for (int t = tid; t < n; t += NT) out[t] = t;
        pos = n;
    } else if (st.flags == kStateEmpty) {
        pos = 0;
    } else {
        for (int t = tid; t < s_end; t += NT) out[t] = t;
        pos = s_end;
        const int kept = ordered_pass<NT>(
            L, M, sm.warp,
            [&](int t, uint32_t key) {
                if (t < s_end || t >= w_beg) return false;
                const int bin = score_bin(key_to_float(key), inv2A);
                return bin > T1 || (bin == T1 && (key > Tkey || (key == Tkey && t <= IT)));
            },
            [&](int rank, int t) { if (pos + rank < cap_sel) out[pos + rank] = t; });
        pos += kept;
        for (int t = w_beg + tid; t < n; t += NT)
            if (pos + (t - w_beg) < cap_sel) out[pos + (t - w_beg)] = t;
        pos += n - w_beg;
        if (pos > cap_sel) pos = cap_sel;  // unreachable when the threshold is consistent
    }
    for (int r = pos + tid; r < cap_sel; r += NT) out[r] = -1;
    if (tid == 0) sel_cnt[bh] = pos;
}

// ---------------------------------------------------------------------------
// Two-kernel selection, second kernel: ordered compaction of each CTA's tokens
// with bin >= T1 into its segment; the last CTA of a (b, h) resolves and emits.
using CollectSmem = ResolveSmem<kListSmem>;

static __global__ void __launch_bounds__(kSelThreads)
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
            int r = block_excl_scan<kSelThreads>(__popc(flags), sm.warp, &tot);
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
    if (tid == 0) sm.last = atomicAdd(ws.arrive + (int64_t)kSyncStride * (gridDim.y + bh), 1u) == (unsigned)(nctas - 1);
    __syncthreads();
    if (!sm.last) return;
    __threadfence();
    resolve_emit<kSelThreads, kListSmem>(ws, bh, nctas, st, S, W, cap_sel, sel_idx, sel_cnt, sm);
    if (tid == 0) ws.arrive[(int64_t)kSyncStride * (gridDim.y + bh)] = 0;
}

// ---------------------------------------------------------------------------
// Limits of the clustered selection (step.cuh): at most kInbinMax tokens in
// the threshold bin are ranked through distributed shared memory (more take its
// exact slow path), and clusters hold at most kMaxCluster CTAs.
constexpr int kInbinMax = 1024;
constexpr int kMaxCluster = 16;

// Threshold of the cluster's summed histogram, computed by one full warp from
// the CTAs' super-bin counts (coarse[64], super-bin s = bins [PER s, PER s +
// PER)) and histograms (hist[64 PER]), both read in place in every CTA's
// shared memory (LOCAL: this CTA's alone, nranks ignored).  Returns the bin
// holding the kk-th largest counted score to every lane, or -1 when fewer than
// kk are counted; out (when not null and the bin exists) = {bin, tokens above
// it, tokens in it} as threshold_bin.
template <int PER = kBins / 64, bool LOCAL = false>
__device__ __forceinline__ int cluster_threshold(const uint32_t *coarse, const uint32_t *hist, int nranks,
                                                 int64_t kk, int *out) {
    static_assert(PER % 2 == 0 && PER <= 64, "fine bins per super-bin");
    const int lane = threadIdx.x & 31;
    if (LOCAL) nranks = 1;
    auto ld = [&](const uint32_t *p, int r) -> uint32_t {
        if constexpr (LOCAL) return *reinterpret_cast<const volatile uint32_t *>(p);
        else return ld_cluster_u32(cluster_addr(p, r));
    };
    // lane l holds super-bins 63 - 2l (upper) and 62 - 2l (lower): lane 0 the top
    uint32_t cu = 0, cl = 0;
    for (int r = 0; r < nranks; ++r) {
        cu += ld(coarse + (63 - 2 * lane), r);
        cl += ld(coarse + (62 - 2 * lane), r);
    }
    int64_t incl = (int64_t)cu + cl;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int64_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    const int64_t excl = incl - cu - cl;
    const bool here = excl < kk && kk <= incl;
    const uint32_t hb = __ballot_sync(0xffffffffu, here);
    if (!hb) return -1;  // fewer than kk counted
    int sb = 0;
    int64_t above = 0;
    if (here) {
        if (excl + cu >= kk) { sb = 63 - 2 * lane; above = excl; }
        else { sb = 62 - 2 * lane; above = excl + cu; }
    }
    sb = __shfl_sync(0xffffffffu, sb, __ffs(hb) - 1);
    above = __shfl_sync(0xffffffffu, above, __ffs(hb) - 1);
    // the PER bins of super-bin sb, the same way (lanes >= PER / 2 hold none)
    const bool has = lane < PER / 2;
    const int bu = PER * sb + PER - 1 - 2 * lane, bl = bu - 1;
    uint32_t fu = 0, fl = 0;
    if (has)
        for (int r = 0; r < nranks; ++r) {
            fu += ld(hist + bu, r);
            fl += ld(hist + bl, r);
        }
    int64_t fincl = (int64_t)fu + fl;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int64_t y = __shfl_up_sync(0xffffffffu, fincl, o);
        if (lane >= o) fincl += y;
    }
    const int64_t fexcl = above + fincl - fu - fl;
    fincl += above;
    const bool hit = has && fexcl < kk && kk <= fincl;
    const uint32_t hm = __ballot_sync(0xffffffffu, hit);
    if (!hm) return -1;  // (counts that did not add up: not reached with settled counts)
    const int t1 = hit ? (fexcl + fu >= kk ? bu : bl) : 0;
    if (hit && out) {
        if (fexcl + fu >= kk) { out[0] = bu; out[1] = (int)fexcl; out[2] = (int)fu; }
        else { out[0] = bl; out[1] = (int)(fexcl + fu); out[2] = (int)fl; }
    }
    return __shfl_sync(0xffffffffu, t1, __ffs(hm) - 1);
}

}  // namespace dkv
