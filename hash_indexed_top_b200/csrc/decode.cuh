// decode.cuh -- stage 4: exact softmax attention over the selected rows only
// (DeepSeek DSA->CSA/HCA page, section "从 DSA 说起": real attention runs on the
// top-k the indexer picked; DASH-KV page, section "技术架构：动态混合精度机制":
// the tokens that matter are attended in full precision).
//
// Gathered split-K flash-decode: grid = (splits, wy + B * Hkv).  Each of the
// last B * Hkv rows' CTAs takes a contiguous slice of one (b, kv head)'s
// selected ids; the optional first wy rows hold window CTAs (see the kernel).  A lane group of LPR
// lanes owns one row at a time (DPL = d / LPR dims per lane), gathers its K and
// V slices with 16-byte loads once, and serves all G query heads of the group
// from them.  Rows are processed in tiles of RT per lane group: the RT G
// partial logits of the tile are formed first and summed over the group by a
// transpose butterfly that leaves one (row, head) logit per lane; each lane
// updates its head's running max and sum, the weights go back to the group
// through shared memory, and the accumulators are rescaled once per tile
// (fp32, base-2 exponentials).  Each CTA merges its
// lane groups' states in shared memory and writes one partial; the last CTA of
// the (b, h) to arrive (atomic counter, no waiting) merges the partials with a
// log-sum-exp reduction and writes out / lse.
//
// TIERED: rows of tier-1 pages (see tiers.cuh) are gathered as their FP8 K and
// V rows (128 + 128 bytes at d = 128 instead of 256 + 256) into the first half
// of the same staging slots, and read back as value(code) * 2^-s; the owner
// lane of a tile row loads its page's tier byte with the token id, one tile
// ahead, and copies the 4-byte word holding the row's two exponents into
// shared memory with the row's copies (no register waits on it).
#pragma once
#include "common.cuh"
#include "tiers.cuh"

namespace dkv {

constexpr int kAttnThreads = 256;
constexpr int kMaxSplits = 256;  // partial slots per (b, h): top-k splits + the window CTAs

struct AttnWS {
    float *part;        // [BH][kMaxSplits][G][D + 2]  (acc[D], m, l)
    uint32_t *arrive;   // [BH]   zero between calls
};

template <int D, int G>
struct DecodeShape {
    static constexpr int DPL = G >= 4 ? 32 / G : 16;   // dims per lane
    static constexpr int LPR = D / DPL;                // lanes per row
    static constexpr int RPW = 32 / LPR;               // rows per warp step
    static constexpr int NWARP = kAttnThreads / 32;
    static constexpr int NST = NWARP * RPW;            // lane groups (running states) per CTA
    static constexpr int RT0 = RPW >= 8 ? 1 : 8 / RPW;
    static constexpr int RT1 = RT0 * G > 32 ? 32 / G : RT0;
    static constexpr int RT = RT1 * G > LPR ? (LPR / G > 0 ? LPR / G : 1) : RT1;  // rows per lane group per tile:
                                                                                  // its logits fit the group's lanes
    static constexpr int TROWS = RPW * RT;             // rows per warp tile
    static constexpr int STAGES = TROWS <= 4 ? 3 : 2;  // cp.async pipeline depth per warp
    static constexpr int CPR = D / 8;                  // 16-byte chunks per K (or V) row
    // per warp: STAGES buffers x TROWS rows x (K, V) x D bf16
    static constexpr size_t STAGE_BYTES = (size_t)NWARP * STAGES * TROWS * 2 * D * 2;
    static constexpr int V = RT * G;                   // logits of a lane group's tile (<= LPR)
    static constexpr size_t SMEM = STAGE_BYTES + (size_t)NST * G * (D + 2) * 4 + (size_t)NST * V * 4 + 16;
    // TIERED: per warp and stage, the exponent word of each tile row (after SMEM)
    static constexpr size_t EX_BYTES = (size_t)NWARP * STAGES * TROWS * 4;
};

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, int src_bytes) {
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }


__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t x) { return make_float2(bf16_lo(x), bf16_hi(x)); }

// 2^x on the SFU (approximate, flushes denormal results to zero: weights below
// 2^-126 of the running maximum vanish, far inside the fp32 accumulation error).
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <int D, int G, bool TIERED = false>
__global__ void __launch_bounds__(kAttnThreads, 2)
sparse_decode_kernel(KV kv, const __nv_bfloat16 *__restrict__ q, int Hq,
                     const int32_t *__restrict__ sel_idx, const int32_t *__restrict__ sel_cnt, int cap_sel,
                     float *__restrict__ out, float *__restrict__ lse, AttnWS ws, int splits, float scale_log2,
                     const int32_t *__restrict__ seq_lens, int n_sink, int n_window, int topk, int wy, int nw,
                     Tiers tiers) {
    using S = DecodeShape<D, G>;
    constexpr int DPL = S::DPL, LPR = S::LPR, RPW = S::RPW, NST = S::NST, RT = S::RT;
    constexpr int TROWS = S::TROWS, CPR = S::CPR, NWARP = S::NWARP, STAGES = S::STAGES, V = S::V;
    static_assert((V & (V - 1)) == 0 && V <= LPR, "a lane group's logits fit its lanes");
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __nv_bfloat16 *stage = reinterpret_cast<__nv_bfloat16 *>(smem_raw);               // [NWARP][STAGES][TROWS][2][D]
    float *s_acc = reinterpret_cast<float *>(smem_raw + S::STAGE_BYTES);              // [NST][G][D]
    float *s_m = s_acc + NST * G * D;                                                  // [NST][G]
    float *s_l = s_m + NST * G;                                                        // [NST][G]
    float *s_p = s_l + NST * G;                                                        // [NST][V] weights
    __shared__ int s_last;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int sub = lane / LPR, li = lane % LPR;
    // The V = RT G logits of a lane group's tile are summed over its LPR lanes
    // by a transpose butterfly: at the level that pairs lanes across bit k every
    // lane sends the upper half of its values and keeps the lower half, and
    // after it lane li holds the logit of (row lv / G, head lv % G), lv = li &
    // (V - 1).  The halves line up because a lane keeps its slots in an order
    // XOR-ed with lv: slot (j, g) holds row j ^ jperm and head g ^ gperm.
    const int lv = li & (V - 1);
    const int gperm = lv % G, jperm = lv / G;
    // Roles.  With wy > 0 the first wy rows of the grid hold nw window CTAs per
    // (b, h): between them they attend over the sinks and the window, which
    // every selection contains, straight from the token range, so they do not
    // wait for the selection and run while the scorer still streams (on the SMs
    // the scorer leaves free).  The other CTAs take the top-k (middle) part of
    // the list, split `splits` ways.  With wy = 0 they take the whole list.
    const int BH = (int)gridDim.y - wy;
    const bool win = (int)blockIdx.y < wy;
    const int wid = win ? (int)(blockIdx.y * splits + blockIdx.x) : 0;  // window CTA number
    const int bh = win ? wid / nw : (int)blockIdx.y - wy;
    if (bh >= BH) return;  // spare window slots
    const int piece = wid % nw;  // this window CTA's share of the sinks + window
    const int split = win ? splits + piece : (int)blockIdx.x;  // partial slot
    const int nparts = splits + (wy > 0 ? nw : 0);
    const int b = bh / kv.Hkv, h = bh % kv.Hkv;
    const int64_t cap_tokens = kv.capacity();

    // this lane's slice of every query head of the group (slot g: head g ^ gperm)
    float qf[G][DPL];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const __nv_bfloat16 *qr = q + ((int64_t)b * Hq + h * G + (g ^ gperm)) * D + li * DPL;
#pragma unroll
        for (int e = 0; e < DPL; e += 2) {
            const uint32_t w = *reinterpret_cast<const uint32_t *>(qr + e);
            qf[g][e] = bf16_lo(w);
            qf[g][e + 1] = bf16_hi(w);
        }
    }
    float m = -INFINITY, lsum = 0.0f;  // of head lv % G (the same in all its lanes)
    float acc[G][DPL];                 // every head (in order) at this lane's dims
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[g][e] = 0.0f;

    // q is an input of the step; the selection comes from the preceding kernel
    // (the window CTAs need none of it: the lengths and rows they read were
    // written before the selection started)
    if (!win) griddep_wait();
    griddep_trigger();
    // The splits divide the capacity of their part of the list (not its count),
    // so the first ids load together with the count instead of after it; rows
    // past the count are masked.
    int64_t n = 0;
    if (wy > 0) {
        n = __ldcg(seq_lens + b);
        n = n < 0 ? 0 : (n > cap_tokens ? cap_tokens : n);
    }
    const int s_end = (int)(n_sink < n ? n_sink : n);
    const int w_beg = (int)(n - n_window > s_end ? n - n_window : s_end);
    const int nwin = (int)n - w_beg;
    const int cnt = win ? 0 : sel_cnt[bh];
    int r0, r1, rend;  // rows [r0, r1) of this CTA, valid below rend
    if (win) {  // the pieces divide the capacity n_sink + n_window of this part
        const int per = (n_sink + n_window + nw - 1) / nw;
        r0 = piece * per;
        r1 = r0 + per;
        rend = s_end + nwin;
    } else if (wy > 0) {  // the middle: list positions [n_sink, n_sink + topk), valid below cnt - nwin
        const int per = (topk + splits - 1) / splits;
        r0 = n_sink + split * per;
        r1 = min(r0 + per, n_sink + topk);
        rend = cnt - nwin;
    } else {
        const int per = (cap_sel + splits - 1) / splits;
        r0 = split * per;
        r1 = min(r0 + per, cap_sel);
        rend = cnt;
    }

    const int32_t *ids = sel_idx + (int64_t)bh * cap_sel;
    __nv_bfloat16 *wstage = stage + (size_t)warp * STAGES * TROWS * 2 * D;
    // Token of row `base + lane` of a tile (lanes < TROWS), -1 when the row is
    // outside the slice or past the count, or its id lies outside the cache.
    auto tile_token = [&](int base) -> int {
        const int r = base + lane;
        if (lane >= TROWS || r >= r1) return -1;
        const int t = win ? (r < s_end ? r : w_beg + (r - s_end)) : __ldg(ids + r);
        if (r >= rend) return -1;
        if (t < 0 || t >= cap_tokens) {
            raise_error(kErrCapacity);
            return -1;
        }
        if (kv.page_size && kv.page_of(b, t) < 0) return -1;
        return t;
    };
    // Tier of the row of token t (from tile_token: -1 or a valid token) of
    // a tile staged in buffer buf: 1 | (row & 1) << 1 for an FP8 row, 0
    // otherwise.  For an FP8 row the aligned exponent word holding the row's
    // pair is copied to word (warp * STAGES + buf) * TROWS + lane after SMEM,
    // committed with the row's copies.
    auto tile_meta = [&](int t, int buf) -> uint32_t {
        if constexpr (!TIERED) {
            return 0u;
        } else {
            if (t < 0) return 0u;
            const int64_t p = kv.page_of(b, t);
            const int64_t row = (p * kv.page_size + t % kv.page_size) * kv.Hkv + h;
            if (!__ldg(tiers.tier + p)) return 0u;
            const unsigned dst = (unsigned)__cvta_generic_to_shared(smem_raw + S::SMEM) +
                                 4u * (unsigned)((warp * STAGES + buf) * TROWS + lane);
            const int8_t *src = tiers.exps + (row & ~(int64_t)1) * 2;
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(dst), "l"(src) : "memory");
            return 1u | (uint32_t)(row & 1) << 1;
        }
    };
    // Gather a tile's K and V rows into buffer `buf` (zero-filled when invalid);
    // tok: this lane's tile_token() of the tile.
    // Lane l copies row l / LPT of the tile: chunks l % LPT, l % LPT + LPT, ...
    // of its K and V rows (so each lane computes one row address per tile).
    constexpr int LPT = 32 / TROWS;               // lanes per tile row
    constexpr int CPL = 2 * CPR / LPT;            // 16-byte chunks per lane (K then V)
    auto prefetch = [&](int tok, uint32_t meta, int buf) {
        __nv_bfloat16 *dst0 = wstage + (size_t)buf * TROWS * 2 * D;
        const int j = lane / LPT, c0 = lane % LPT;
        const int t = __shfl_sync(0xffffffffu, tok, j);
        const bool f8 = TIERED && (__shfl_sync(0xffffffffu, meta, j) & 1u);
        const int64_t off = t >= 0 ? kv.row(b, h, t) : 0;
        const int nbytes = t >= 0 ? 16 : 0;
        __nv_bfloat16 *dst = dst0 + (size_t)j * 2 * D;
#pragma unroll
        for (int m = 0; m < CPL; ++m) {
            const int c = c0 + m * LPT;       // chunk of the (K, V) pair of rows
            const bool isv = c >= CPR;        // compile-time per m when LPT divides CPR
            const int cc = isv ? c - CPR : c;
            if (TIERED && f8) {  // the FP8 row: its CPR / 2 chunks into the slot's first half
                const bool in = cc < CPR / 2 && t >= 0;
                const uint8_t *src = in ? (isv ? tiers.v8 : tiers.k8) + off + cc * 16 : tiers.k8;
                cp_async16(dst + (isv ? D : 0) + cc * 8, src, in ? 16 : 0);
            } else {
                const __nv_bfloat16 *src = (isv ? kv.v : kv.k) + off + cc * 8;
                cp_async16(dst + (isv ? D : 0) + cc * 8, src, nbytes);
            }
        }
        cp_async_commit();
    };

    constexpr int WSTEP = NWARP * TROWS;  // rows per CTA tile round
    int base = r0 + warp * TROWS;
    int tok[STAGES];
    uint32_t meta[STAGES];
#pragma unroll
    for (int s = 0; s < STAGES; ++s) meta[s] = 0u;
#pragma unroll
    for (int s = 0; s < STAGES - 1; ++s) {
        tok[s] = -1;
        if (base + s * WSTEP < r1) {
            tok[s] = tile_token(base + s * WSTEP);
            meta[s] = tile_meta(tok[s], s);
            prefetch(tok[s], meta[s], s);
        } else {
            cp_async_commit();
        }
    }
    for (int k = 0; base < r1; base += WSTEP, ++k) {
        const int buf = k % STAGES;
        const int ahead = base + (STAGES - 1) * WSTEP;
        const int abuf = (k + STAGES - 1) % STAGES;
        if (ahead < r1) {
            tok[abuf] = tile_token(ahead);
            meta[abuf] = tile_meta(tok[abuf], abuf);
            prefetch(tok[abuf], meta[abuf], abuf);
        } else {
            cp_async_commit();
        }
        cp_async_wait<STAGES - 1>();
        __syncwarp();
        const __nv_bfloat16 *tile = wstage + (size_t)buf * TROWS * 2 * D;

        // partial q . k of slot (j, g): row j ^ jperm, head g ^ gperm
        float x[V];
#pragma unroll
        for (int j = 0; j < RT; ++j) {
            const int jr = (j ^ jperm) * RPW + sub;  // row within the tile
            const __nv_bfloat16 *kr = tile + (size_t)jr * 2 * D + li * DPL;
            float kf[DPL];
            bool f8 = false;
            if constexpr (TIERED) {
                const uint32_t mk = __shfl_sync(0xffffffffu, meta[buf], jr);
                if (mk & 1u) {
                    const uint32_t ew = reinterpret_cast<const uint32_t *>(smem_raw + S::SMEM)
                                            [(warp * STAGES + buf) * TROWS + jr] >> ((mk & 2u) ? 16 : 0);
                    e4m3_row<DPL>(reinterpret_cast<const uint8_t *>(tile + (size_t)jr * 2 * D) + li * DPL,
                                  pow2_neg((int)(int8_t)ew), kf);
                    f8 = true;
                }
            }
            if (f8) {
            } else if constexpr (DPL >= 8) {
#pragma unroll
                for (int e = 0; e < DPL; e += 8) {
                    const uint4 w = *reinterpret_cast<const uint4 *>(kr + e);
                    kf[e + 0] = bf16_lo(w.x); kf[e + 1] = bf16_hi(w.x); kf[e + 2] = bf16_lo(w.y); kf[e + 3] = bf16_hi(w.y);
                    kf[e + 4] = bf16_lo(w.z); kf[e + 5] = bf16_hi(w.z); kf[e + 6] = bf16_lo(w.w); kf[e + 7] = bf16_hi(w.w);
                }
            } else {
                const uint2 w = *reinterpret_cast<const uint2 *>(kr);
                kf[0] = bf16_lo(w.x); kf[1] = bf16_hi(w.x); kf[2] = bf16_lo(w.y); kf[3] = bf16_hi(w.y);
            }
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float2 d2 = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int e = 0; e < DPL; e += 2)
                    d2 = ffma2(make_float2(qf[g][e], qf[g][e + 1]), make_float2(kf[e], kf[e + 1]), d2);
                x[j * G + g] = d2.x + d2.y;
            }
        }
#pragma unroll
        for (int half = V / 2; half >= 1; half >>= 1)
#pragma unroll
            for (int i = 0; i < half; ++i) x[i] += __shfl_xor_sync(0xffffffffu, x[i + half], half);
#pragma unroll
        for (int o = LPR / 2; o >= V; o >>= 1) x[0] += __shfl_xor_sync(0xffffffffu, x[0], o);
        // online softmax of head lv % G over its RT rows (lanes lv, lv + G, ...)
        const bool okl = __shfl_sync(0xffffffffu, tok[buf], (lv / G) * RPW + sub) >= 0;
        const float sc = okl ? x[0] * scale_log2 : -INFINITY;
        float tmax = sc;
#pragma unroll
        for (int o = G; o < V; o <<= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
        const float mn = fmaxf(m, tmax);
        const float c = mn == -INFINITY ? 1.0f : fast_exp2(m - mn);  // 0 while m = -inf
        const float pw = okl ? fast_exp2(sc - mn) : 0.0f;
        float ps = pw;
#pragma unroll
        for (int o = G; o < V; o <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
        lsum = fmaf(lsum, c, ps);
        m = mn;
        // the weights to the whole lane group through shared memory, each head's
        // rescale factor by shuffle
        float *sp = s_p + (warp * RPW + sub) * V;  // [RT][G]
        if (li < V) sp[li] = pw;
        float ch[G];
#pragma unroll
        for (int g = 0; g < G; ++g) ch[g] = __shfl_sync(0xffffffffu, c, sub * LPR + g);
        __syncwarp();
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < DPL; ++e) acc[g][e] *= ch[g];
        // P.V for the tile (rows that are not valid are zero-filled, weight 0)
#pragma unroll
        for (int j = 0; j < RT; ++j) {
            const int jr = j * RPW + sub;
            const __nv_bfloat16 *vrow = tile + ((size_t)jr * 2 + 1) * D + li * DPL;
            float vf[DPL];
            bool f8v = false;
            if constexpr (TIERED) {
                const uint32_t mv = __shfl_sync(0xffffffffu, meta[buf], jr);
                if (mv & 1u) {
                    const uint32_t ew = reinterpret_cast<const uint32_t *>(smem_raw + S::SMEM)
                                            [(warp * STAGES + buf) * TROWS + jr] >> ((mv & 2u) ? 16 : 0);
                    e4m3_row<DPL>(reinterpret_cast<const uint8_t *>(tile + ((size_t)jr * 2 + 1) * D) + li * DPL,
                                  pow2_neg((int)(int8_t)(ew >> 8)), vf);
                    f8v = true;
                }
            }
            if (f8v) {
            } else if constexpr (DPL >= 8) {
#pragma unroll
                for (int e = 0; e < DPL; e += 8) {
                    const uint4 w = *reinterpret_cast<const uint4 *>(vrow + e);
                    vf[e + 0] = bf16_lo(w.x); vf[e + 1] = bf16_hi(w.x); vf[e + 2] = bf16_lo(w.y); vf[e + 3] = bf16_hi(w.y);
                    vf[e + 4] = bf16_lo(w.z); vf[e + 5] = bf16_hi(w.z); vf[e + 6] = bf16_lo(w.w); vf[e + 7] = bf16_hi(w.w);
                }
            } else {
                const uint2 w = *reinterpret_cast<const uint2 *>(vrow);
                vf[0] = bf16_lo(w.x); vf[1] = bf16_hi(w.x); vf[2] = bf16_lo(w.y); vf[3] = bf16_hi(w.y);
            }
            float pj[G];
            if constexpr (G >= 4) {
#pragma unroll
                for (int g = 0; g < G; g += 4) {
                    const float4 p4 = *reinterpret_cast<const float4 *>(sp + j * G + g);
                    pj[g] = p4.x; pj[g + 1] = p4.y; pj[g + 2] = p4.z; pj[g + 3] = p4.w;
                }
            } else {
#pragma unroll
                for (int g = 0; g < G; ++g) pj[g] = sp[j * G + g];
            }
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float2 p2 = make_float2(pj[g], pj[g]);
#pragma unroll
                for (int e = 0; e < DPL; e += 2) {
                    const float2 a2 = ffma2(p2, make_float2(vf[e], vf[e + 1]), make_float2(acc[g][e], acc[g][e + 1]));
                    acc[g][e] = a2.x;
                    acc[g][e + 1] = a2.y;
                }
            }
        }
        __syncwarp();  // the buffer is refilled by a later prefetch
    }
    cp_async_wait<0>();

    // merge the NST running states of this CTA
    const int st = warp * RPW + sub;
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const float mg = __shfl_sync(0xffffffffu, m, sub * LPR + g);
        const float lg = __shfl_sync(0xffffffffu, lsum, sub * LPR + g);
        if (li == 0) { s_m[st * G + g] = mg; s_l[st * G + g] = lg; }
#pragma unroll
        for (int e = 0; e < DPL; ++e) s_acc[(st * G + g) * D + li * DPL + e] = acc[g][e];
    }
    __syncthreads();
    float *part = ws.part + ((int64_t)bh * kMaxSplits + split) * G * (D + 2);
    for (int x = tid; x < G * D; x += kAttnThreads) {
        const int g = x / D, i = x % D;
        float M = -INFINITY;
#pragma unroll 8
        for (int s = 0; s < NST; ++s) M = fmaxf(M, s_m[s * G + g]);
        float L = 0.0f, Acc = 0.0f;
        if (M != -INFINITY) {
#pragma unroll 8
            for (int s = 0; s < NST; ++s) {
                const float c = fast_exp2(s_m[s * G + g] - M);
                L = fmaf(s_l[s * G + g], c, L);
                Acc = fmaf(s_acc[(s * G + g) * D + i], c, Acc);
            }
        }
        part[g * (D + 2) + i] = Acc;
        if (i == 0) { part[g * (D + 2) + D] = M; part[g * (D + 2) + D + 1] = L; }
    }

    // the last CTA of this (b, h) merges the splits
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(ws.arrive + (int64_t)kSyncStride * bh, 1u) == (unsigned)(nparts - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const float *pbase = ws.part + (int64_t)bh * kMaxSplits * G * (D + 2);
    // each output element: every part's (m, l, acc) loaded at once -- for all
    // the elements of this thread (EPT) in one round trip -- then the
    // log-sum-exp merge in registers
    constexpr int MS = 16;  // parts merged per pass (all loads of a pass in flight)
    constexpr int EPT0 = (G * D + kAttnThreads - 1) / kAttnThreads;  // elements per thread
    constexpr int EPT = EPT0 < 2 ? EPT0 : 2;                           // of them per round trip
    for (int x0 = tid; x0 < G * D; x0 += EPT * kAttnThreads) {
        float M[EPT], L[EPT], Acc[EPT];
#pragma unroll
        for (int e = 0; e < EPT; ++e) { M[e] = -INFINITY; L[e] = 0.0f; Acc[e] = 0.0f; }
        for (int s0 = 0; s0 < nparts; s0 += MS) {
            float pm[EPT][MS], pl[EPT][MS], pa[EPT][MS];
#pragma unroll
            for (int e = 0; e < EPT; ++e) {
                const int x = x0 + e * kAttnThreads;
                const int g = x / D, i = x % D;
#pragma unroll
                for (int u = 0; u < MS; ++u) {
                    const float *ps = pbase + ((s0 + u) * G + g) * (D + 2);
                    const bool in = x < G * D && s0 + u < nparts;
                    pm[e][u] = in ? __ldcg(ps + D) : -INFINITY;
                    pl[e][u] = in ? __ldcg(ps + D + 1) : 0.0f;
                    pa[e][u] = in ? __ldcg(ps + i) : 0.0f;
                }
            }
#pragma unroll
            for (int e = 0; e < EPT; ++e) {
                float Mn = M[e];
#pragma unroll
                for (int u = 0; u < MS; ++u) Mn = fmaxf(Mn, pm[e][u]);
                if (Mn == -INFINITY) continue;
                const float cM = fast_exp2(M[e] - Mn);  // 0 when M = -inf
                L[e] *= cM;
                Acc[e] *= cM;
#pragma unroll
                for (int u = 0; u < MS; ++u) {
                    const float c = fast_exp2(pm[e][u] - Mn);  // 0 for empty parts (m = -inf)
                    L[e] = fmaf(pl[e][u], c, L[e]);
                    Acc[e] = fmaf(pa[e][u], c, Acc[e]);
                }
                M[e] = Mn;
            }
        }
#pragma unroll
        for (int e = 0; e < EPT; ++e) {
            const int x = x0 + e * kAttnThreads;
            if (x >= G * D) continue;
            const int g = x / D, i = x % D;
            const int64_t oq = (int64_t)b * Hq + h * G + g;
            out[oq * D + i] = L[e] > 0.0f ? Acc[e] / L[e] : 0.0f;
            if (i == 0 && lse) lse[oq] = L[e] > 0.0f ? (M[e] + log2f(L[e])) * 0.6931471805599453f : -INFINITY;
        }
    }
    if (tid == 0) ws.arrive[(int64_t)kSyncStride * bh] = 0;
}

}  // namespace dkv
