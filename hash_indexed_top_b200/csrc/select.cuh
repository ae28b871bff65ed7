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
// The fused selection records, per 32-token chunk of a CTA's range, the largest
// bin in the chunk (uint16 in shared memory, for the first kCmaxCap chunks).
constexpr int kCmaxCap = 16384;

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
    static constexpr uint32_t LOW_BYTES = SCRATCH_BYTES + kCmaxCap * 2;               // + chunk maxima
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
    uint16_t *cmax;      // [kCmaxCap] largest bin per 32-token chunk (FUSED only)
};

// FUSED: the fused selection -- record the chunk maxima, and let the dependent
// launch (the sparse decode, whose window CTAs need nothing from the selection)
// start right after the wait on the preceding kernel.
// RADIUS: radius-scaled scores s' = r~ s (Spherical KV page, section 2.1 ADA: a
// quantized key radius beside the angle code scales the logit), r~ = (c + 1/2)/4
// from the token's 8-bit code c in kv.radius; the bins span r~_max times the
// unscaled range.
template <int BITS, int D, bool PAGED, bool FUSED = false, bool RADIUS = false>
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
    o.cmax = reinterpret_cast<uint16_t *>(smem + S::SCRATCH_BYTES);
    // everything above depends on q only; codes and lengths come from the append
    griddep_wait();
    if constexpr (FUSED) griddep_trigger();
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
            if constexpr (FUSED) {
                const unsigned m = __reduce_max_sync(0xffffffffu, (unsigned)bin);
                const int c = (wb >> 5) + k;  // chunk of local tokens [32 c, 32 c + 32)
                if (lane == 0 && c < kCmaxCap) o.cmax[c] = (uint16_t)m;
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

// Smallest finite float s with score_bin(s, inv2A) >= T, or +inf if there is
// none, so that for every finite s:  s >= result  <=>  score_bin(s) >= T.
// score_bin is monotone in s (a correctly rounded fma with a non-negative
// factor, a clamp, a scale and a truncation), hence monotone along the
// order-preserving keys.  A full warp first tests the 32 keys around the
// algebraic estimate; if the boundary is not among them it narrows the whole
// key range 32-fold per round.  Every lane returns the result.
__device__ __forceinline__ float bin_floor_value(int T, float inv2A) {
    const int lane = threadIdx.x & 31;
    if (T <= 0) return -INFINITY;
    if (T >= kBins) return INFINITY;
    auto P = [&](uint32_t key) { return score_bin(key_to_float(key), inv2A) >= T; };
    if (inv2A > 0.0f) {
        const float est = ((float)T / (float)(kBins - 1) - 0.5f) / inv2A;
        const uint32_t k0 = float_key(est) - 16u;
        const uint32_t b = __ballot_sync(0xffffffffu, P(k0 + (uint32_t)lane));
        const int f = __ffs(b) - 1;  // a boundary inside the window: false below lane f, true from it
        if (f > 0 && b == (0xffffffffu << f)) return key_to_float(k0 + (uint32_t)f);
    }
    const uint32_t none = 0xff800000u;     // key of +inf: one past the key of FLT_MAX
    uint64_t lo = 0x00800000u, hi = none;  // key of -FLT_MAX; answer in [lo, hi]
    while (lo < hi) {
        const uint64_t n = hi - lo;
        const uint64_t step = (n + 31) / 32;
        const uint64_t x = lo + (uint64_t)lane * step;
        const uint32_t b = __ballot_sync(0xffffffffu, x < hi && P((uint32_t)x));
        if (b) {
            const int f = __ffs(b) - 1;    // false at lo + (f - 1) step, true at lo + f step
            hi = lo + (uint64_t)f * step;
            if (f) lo += (uint64_t)(f - 1) * step + 1;
        } else {                           // every tested point is false
            const uint64_t last = (n - 1) / step < 31 ? (n - 1) / step : 31;
            lo += last * step + 1;
        }
    }
    return key_to_float((uint32_t)lo);     // `none` maps to +inf
}

template <int BITS, int D, bool PAGED, bool RADIUS = false>
__global__ void __launch_bounds__(kScoreThreads, 1)
select_fused_kernel(KV kv, const __nv_bfloat16 *__restrict__ q, int Hq, int G,
                    const int32_t *__restrict__ seq_lens, const RBits R, SelWS ws, int topk, int S, int W,
                    int cap_sel, int32_t *sel_idx, int32_t *sel_cnt) {
    constexpr int NT = kScoreThreads;
    constexpr int NWARP = NT / 32;
    constexpr int CW = 64;  // candidates per warp kept in shared memory (more go to the global segment)
    // hit chunks whose scores one warp stages per round trip: [FB][32] floats per
    // warp in the code ring, which is idle once the scores are written
    constexpr int FB = (int)(ScoreShape<BITS>::RING_BYTES / (NWARP * 32 * 4)) < 16
                           ? (int)(ScoreShape<BITS>::RING_BYTES / (NWARP * 32 * 4)) : 16;
    static_assert(FB >= 1 && (size_t)FB * NWARP * 32 * 4 <= ScoreShape<BITS>::RING_BYTES, "staging exceeds the ring");
    // the LUT region (64 KB) after scoring: in-bin list | warp candidates | gathered list, or the resolver
    static_assert(kInbinMax * 16 <= 16384 && NWARP * CW * 8 <= 16384, "fast-path lists exceed their slots");
    static_assert(sizeof(ResolveSmem<4096>) <= ScoreShape<BITS>::LUT_BYTES, "resolver exceeds the LUT region");
    extern __shared__ __align__(1024) unsigned char smem[];
    __shared__ int s_warp[32];
    __shared__ int s_thr[4];
    __shared__ int s_misc[4];
    __shared__ float s_theta[2];
    __shared__ uint32_t s_coarse[64];      // this CTA's histogram per super-bin (read by the cluster)
    __shared__ int s_cnt[kMaxCluster][2];  // per CTA of the cluster: in-bin entries, definite middle tokens
    __shared__ int s_mid[kMaxCluster];
    __shared__ int s_wkeep[NWARP];
    __shared__ int s_hlist[NWARP][32];     // per warp: its hit chunks of the current group
    __shared__ int s_ninb;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bh = blockIdx.y, cta = blockIdx.x;  // cta = rank in the cluster (cluster = the row of CTAs)
    const int nctas = gridDim.x;
    const ScoreOut so = score_phase<BITS, D, PAGED, true, RADIUS>(kv, q, Hq, G, seq_lens, R, ws, nctas, smem);
    const uint32_t *hist = reinterpret_cast<const uint32_t *>(smem);
    {   // super-bin counts: 16 threads per super-bin, 4 bins each
        uint32_t c = hist[4 * tid] + hist[4 * tid + 1] + hist[4 * tid + 2] + hist[4 * tid + 3];
#pragma unroll
        for (int o = 8; o; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        if ((lane & 15) == 0) s_coarse[tid >> 4] = c;
    }
    const int64_t n = so.n, t0 = so.t0, t1 = so.t1;
    const int64_t kk = topk < n ? topk : n;
    const bool normal = n > 0 && kk < n;
    if (tid == 0) { s_thr[0] = kBins; s_thr[1] = 0; s_thr[2] = 0; s_ninb = 0; }
    cluster_sync();  // (1): every histogram of the cluster is complete
    const float inv2A = so.inv2A;
    if (normal && warp < 2) {  // both find T1; warp 0 then theta(T1), warp 1 theta(T1 + 1)
        const int T1w = cluster_threshold(s_coarse, hist, nctas, kk, warp == 0 ? s_thr : nullptr);
        const float th = bin_floor_value(T1w + warp, inv2A);
        if (lane == 0) s_theta[warp] = th;
    }
    __syncthreads();
    const int T1 = s_thr[0], above1 = s_thr[1], cnt_T1 = s_thr[2];
    const bool fallback = normal && cnt_T1 > kInbinMax;
    const int s_end = (int)(S < n ? S : n);
    const int w_beg = (int)(n - W > s_end ? n - W : s_end);
    int32_t *cand = ws.cand + (int64_t)bh * ws.ld;
    uint32_t *ckey = ws.ckey + (int64_t)bh * ws.ld;
    const float *srow = ws.scores + (int64_t)bh * ws.ld;
    int32_t *out = sel_idx + (int64_t)bh * cap_sel;

    if (!normal || fallback) {
        // ---- exact resolver of the two-kernel path (heavy ties, everything or nothing selected):
        // CTA segments [t0, t0 + seg) of the tokens with bin >= T1, ascending
        int seg = 0;
        if (normal) {
            for (int64_t base = t0; base < t1; base += (int64_t)NT * 32) {
                const int64_t tb = base + (int64_t)tid * 32;
                uint32_t flags = 0;
                for (int e = 0; e < 32; ++e)
                    if (tb + e < t1 && score_bin(__ldcg(srow + tb + e), inv2A) >= T1) flags |= 1u << e;
                int tot;
                int r = block_excl_scan<NT>(__popc(flags), s_warp, &tot);
                while (flags) {
                    const int j = __ffs(flags) - 1;
                    flags &= flags - 1;
                    cand[t0 + seg + r++] = (int32_t)(tb + j);
                }
                seg += tot;
            }
        }
        if (tid == 0) ws.seg_cnt[(int64_t)bh * kMaxSelCtas + cta] = seg;
        __threadfence();
        cluster_sync();  // (2): segments complete (nothing reads another CTA's shared memory after this)
        if (cta != 0) return;
        SelState st;
        st.T1 = T1; st.above1 = above1; st.cnt_T1 = cnt_T1;
        st.flags = n == 0 ? kStateEmpty : (normal ? kStateNormal : kStateAll);
        st.inv2A = inv2A; st.pad = 0.0f; st.kk = (int32_t)kk; st.n = (int32_t)n;
        resolve_emit<NT, 4096>(ws, bh, nctas, st, S, W, cap_sel, sel_idx, sel_cnt,
                               *reinterpret_cast<ResolveSmem<4096> *>(so.lut));
        return;
    }

    // ---- fast path.  Warp w owns the 32-token chunks of its range; only the
    // chunks whose maximum bin reaches T1 are re-read (lane = token, up to FB
    // chunks per memory round trip, staged in shared memory so that the code
    // that runs once per step stays a pair of short loops).  A token is a candidate iff its score >=
    // theta (exactly bin >= T1) and in the threshold bin iff also score <
    // theta2.  The warp keeps its candidates in token order with their order
    // keys -- the first CW in shared memory, the rest in its slice of the global
    // segment -- lists the in-bin ones for the cluster and counts the definite
    // middle ones.
    uint4 *s_loc = reinterpret_cast<uint4 *>(so.lut);                      // this CTA's in-bin tokens
    uint2 *wcand = reinterpret_cast<uint2 *>(so.lut + 16384) + warp * CW;  // per-warp candidates
    uint4 *s_inb = reinterpret_cast<uint4 *>(so.lut + 32768);              // the cluster's in-bin tokens
    const float theta = s_theta[0], theta2 = s_theta[1];
    const int wb = warp * so.R;
    const int we = (int)min((int64_t)(wb + so.R), t1 - t0);
    const int nch = we > wb ? (we - wb + 31) >> 5 : 0;
    const uint32_t lt = (1u << lane) - 1u;
    int ncand = 0, ndef = 0;
    auto chunk_hit = [&](int c) {
        const int gc = (wb >> 5) + c;
        return c < nch && (gc >= kCmaxCap || (int)so.cmax[gc] >= T1);
    };
    // per-warp staging buffer [FB][32] of scores, in the (now idle) code ring,
    // and the warp's list of hit chunks of the current group of 32
    float *fbuf = reinterpret_cast<float *>(so.lut + 65536) + warp * (FB * 32);
    const uint32_t fbuf_s = (uint32_t)__cvta_generic_to_shared(fbuf);
    int *hlist = s_hlist[warp];
    const int wlen = we - wb;  // tokens of this warp
    for (int g0 = 0; g0 < nch; g0 += 32) {
        const bool hc = chunk_hit(g0 + lane);
        const uint32_t hb = __ballot_sync(0xffffffffu, hc);
        if (hc) hlist[__popc(hb & lt)] = g0 + lane;
        __syncwarp();
        const int nh = __popc(hb);
        for (int h0 = 0; h0 < nh; h0 += FB) {
            const int nf = min(FB, nh - h0);
            // stage the scores of chunks h0 .. h0 + nf - 1: 16 bytes per lane, 4 chunks
            // per instruction, all in flight at once (whole chunks: rows are padded
            // to 64 tokens, so a chunk never runs past its row)
#pragma unroll 1
            for (int q = lane; q < 8 * nf; q += 32) {
                const int c = hlist[h0 + (q >> 3)];
                const float *src = srow + t0 + wb + 32 * c + 4 * (q & 7);
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(fbuf_s + 16u * (uint32_t)q), "l"(src)
                             : "memory");
            }
            asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
            __syncwarp();
#pragma unroll 2
            for (int f = 0; f < nf; ++f) {
                const int li = 32 * hlist[h0 + f] + lane;  // warp-local token
                const float sv = fbuf[32 * f + lane];
                const bool hit = li < wlen && sv >= theta;
                const uint32_t ball = __ballot_sync(0xffffffffu, hit);
                if (hit) {
                    const int j = ncand + __popc(ball & lt);
                    const int t = (int)(t0 + wb + li);
                    const uint32_t key = float_key(sv);
                    if (j < CW) wcand[j] = make_uint2((uint32_t)t, key);
                    else { cand[t0 + wb + j] = t; ckey[t0 + wb + j] = key; }
                }
                ncand += __popc(ball);
            }
            __syncwarp();  // the buffer is refilled by the next batch
        }
    }
    auto cand_at = [&](int j, int &t, uint32_t &key) {
        if (j < CW) { const uint2 c = wcand[j]; t = (int)c.x; key = c.y; }
        else { t = __ldcg(cand + t0 + wb + j); key = __ldcg(ckey + t0 + wb + j); }
    };
    __syncwarp();
    // classify the warp's candidates, 32 at a time: in the threshold bin (score <
    // theta2: listed for the cluster, one reservation per group) or definite
    // (counted when in the middle range)
    const uint32_t key2 = float_key(theta2);  // order keys follow scores
    for (int jb = 0; jb < ncand; jb += 32) {
        const int j = jb + lane;
        int t = 0;
        uint32_t key = 0;
        if (j < ncand) cand_at(j, t, key);
        const bool inb = j < ncand && key < key2;
        const bool def = j < ncand && !inb && t >= s_end && t < w_beg;
        ndef += __popc(__ballot_sync(0xffffffffu, def)) * (lane == 0);
        const uint32_t ib = __ballot_sync(0xffffffffu, inb);
        if (ib) {
            int base = 0;
            if (lane == 0) base = atomicAdd(&s_ninb, __popc(ib));
            base = __shfl_sync(0xffffffffu, base, 0);
            const int slot = base + __popc(ib & lt);
            if (inb && slot < kInbinMax) s_loc[slot] = make_uint4(key, (uint32_t)t, (uint32_t)cta, (uint32_t)warp);
        }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) ndef += __shfl_xor_sync(0xffffffffu, ndef, o);
    if (lane == 0) s_wkeep[warp] = ndef;  // kept candidates of the warp: + its selected in-bin ones
    __syncthreads();
    if (warp == 0) {
        // publish (in-bin entries, definite middle tokens) into every CTA's s_cnt[cta]
        int d = s_wkeep[lane];
#pragma unroll
        for (int o = 16; o; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
        const int ni = min(s_ninb, kInbinMax);
        if (lane < nctas) {
            st_cluster_u32(cluster_addr(&s_cnt[cta][0], lane), (uint32_t)ni);
            st_cluster_u32(cluster_addr(&s_cnt[cta][1], lane), (uint32_t)d);
        }
    }
    cluster_sync();  // (2): every CTA's in-bin list is complete and its counts delivered

    // ---- gather the cluster's in-bin lists (their sizes sum to cnt_T1 <= NT):
    // thread e copies entry e from the CTA whose list holds it
    const int c1 = cnt_T1;
    if (warp * 32 < c1) {
        const int ni = lane < nctas ? s_cnt[lane][0] : 0;
        int incl = ni;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const int excl = incl - ni;
        int r = 0;
        for (int q = 1; q < nctas; ++q) r = __shfl_sync(0xffffffffu, excl, q) <= tid ? q : r;
        const int off = tid - __shfl_sync(0xffffffffu, excl, r);
        if (tid < c1) s_inb[tid] = ld_cluster_v4(cluster_addr(s_loc + off, r));
    }
    __syncthreads();
    cluster_arrive();  // (3): done with the other CTAs' shared memory

    // ---- rank the in-bin list (score desc, token asc): the need1-th entry
    // (Tkey, IT) is the last one selected.  Credit the selected middle ones to
    // their CTA (output offsets) and, for this CTA's, to their warp.
    const int need1 = (int)kk - above1;  // 1 <= need1 <= c1
    if (c1 <= 32) {
        if (warp == 0) {  // one warp, entry e in lane e
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
            int mid = 0;  // lane r < nctas: selected middle tokens of CTA r
            for (int r = 0; r < nctas; ++r) {
                const int cr = __popc(__ballot_sync(0xffffffffu, sel && (int)en.z == r));
                if (lane == r) mid = s_cnt[r][1] + cr;
            }
            if (sel && (int)en.z == cta) atomicAdd(&s_wkeep[en.w], 1);
            int before = lane < cta ? mid : 0, total = mid;
#pragma unroll
            for (int o = 16; o; o >>= 1) {
                before += __shfl_xor_sync(0xffffffffu, before, o);
                total += __shfl_xor_sync(0xffffffffu, total, o);
            }
            if (lane == 0) { s_misc[0] = (int)Tkey; s_misc[1] = IT; s_misc[2] = before; s_misc[3] = total; }
        }
    } else {  // a long list: every thread ranks its entries
        if (tid == 0) { s_misc[0] = 0; s_misc[1] = 0x7fffffff; }
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
                if (rank == need1 - 1) { s_misc[0] = (int)ke; s_misc[1] = (int)ie; }
            }
        }
        __syncthreads();
        const uint32_t Tkey = (uint32_t)s_misc[0];
        const int IT = s_misc[1];
        for (int e = tid; e < c1; e += NT) {
            const uint4 en = s_inb[e];
            const int t = (int)en.y;
            if (t >= s_end && t < w_beg && (en.x > Tkey || (en.x == Tkey && t <= IT))) {
                atomicAdd(&s_mid[en.z], 1);
                if ((int)en.z == cta) atomicAdd(&s_wkeep[en.w], 1);
            }
        }
        __syncthreads();
        if (tid == 0) {
            int before = 0, total = 0;
            for (int r = 0; r < nctas; ++r) {
                before += r < cta ? s_mid[r] : 0;
                total += s_mid[r];
            }
            s_misc[2] = before;
            s_misc[3] = total;
        }
    }
    __syncthreads();
    const uint32_t Tkey = (uint32_t)s_misc[0];
    const int IT = s_misc[1];
    const int total_mid = s_misc[3];
    auto keep = [&](int t, uint32_t key) {
        if (t < s_end || t >= w_beg) return false;
        return key_to_float(key) >= theta2 || key > Tkey || (key == Tkey && t <= IT);
    };
    // ---- ordered emission: warp w writes its kept candidates from offset
    // s_end + (this CTA's offset) + (kept candidates of warps < w)
    int wpos = s_end + s_misc[2];
    for (int w2 = 0; w2 < warp; ++w2) wpos += s_wkeep[w2];
    for (int jb = 0; jb < ncand; jb += 32) {
        const int j = jb + lane;
        int t = 0; uint32_t key = 0;
        if (j < ncand) cand_at(j, t, key);
        const bool k2 = j < ncand && keep(t, key);
        const uint32_t ball = __ballot_sync(0xffffffffu, k2);
        if (k2) {
            const int p = wpos + __popc(ball & lt);
            if (p < cap_sel) out[p] = t;
        }
        wpos += __popc(ball);
    }
    {   // the sinks, the window and the padding, spread over the cluster's CTAs
        const int wpos0 = s_end + total_mid;
        const int nwin = (int)(n - w_beg);
        const int total = min(wpos0 + nwin, cap_sel);
        const int nall = s_end + nwin + (cap_sel - total);
        for (int x = cta * NT + tid; x < nall; x += nctas * NT) {
            if (x < s_end) {
                out[x] = x;
            } else if (x < s_end + nwin) {
                const int tw = x - s_end;
                if (wpos0 + tw < cap_sel) out[wpos0 + tw] = w_beg + tw;
            } else {
                out[total + (x - s_end - nwin)] = -1;
            }
        }
        if (cta == 0 && tid == 0) sel_cnt[bh] = total;
    }
    cluster_wait();  // (3): no CTA leaves while another may still read its shared memory
}

}  // namespace dkv
