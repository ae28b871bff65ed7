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
constexpr int kCandSmem = 2048;  // in-bin candidates resolved in shared memory

enum : int { kStateNormal = 0, kStateAll = 1, kStateEmpty = 2 };

struct SelState {
    int32_t T1;       // threshold bin
    int32_t above1;   // tokens in bins > T1
    int32_t cnt_T1;   // tokens in bin T1
    int32_t flags;
    float A;          // score bound used for binning
    float inv_w;      // bins per unit score
    int32_t kk;       // min(topk, N)
    int32_t n;        // N (clamped)
};

struct SelWS {
    float *scores;       // [BH][ld]
    int64_t ld;          // row length (cache capacity in tokens)
    int32_t *cand;       // [BH][ld]
    uint32_t *hist;      // [BH][kBins]        zero between calls
    SelState *state;     // [BH]
    uint32_t *arrive;    // [2][BH]            zero between calls
    int32_t *seg_cnt;    // [BH][kMaxSelCtas]
};

__device__ __forceinline__ int score_bin(float s, float A, float inv_w) {
    int bin = (int)((s + A) * inv_w);
    return bin < 0 ? 0 : (bin > kBins - 1 ? kBins - 1 : bin);
}

// Token range [t0, t1) of CTA `c` of `nctas` over a length-n sequence; ranges
// are 64-aligned so a warp's 32 tokens never straddle a page.
__device__ __forceinline__ void cta_range(int64_t n, int c, int nctas, int64_t &t0, int64_t &t1) {
    int64_t per = ceil_div(ceil_div(n, nctas), 64) * 64;
    t0 = (int64_t)c * per;
    t1 = t0 + per < n ? t0 + per : n;
    if (t0 > n) t0 = n;
}

// Block-wide exclusive scan of one int per thread (blockDim = kSelThreads).
// Returns the exclusive prefix; *total gets the block sum.  All threads must call.
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
        int w = lane < kSelThreads / 32 ? s_warp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < kSelThreads / 32) s_warp[lane] = w;  // inclusive warp prefix
    }
    __syncthreads();
    int before = warp ? s_warp[warp - 1] : 0;
    *total = s_warp[kSelThreads / 32 - 1];
    __syncthreads();  // s_warp may be reused right after
    return before + x - v;
}

// ---------------------------------------------------------------------------
// Score + histogram.
template <int BITS>
struct ScoreShape {
    static constexpr int T = BITS / 8;         // byte tables
    static constexpr int COPIES = 32 / T;      // interleaved copies: lanes hit distinct banks
    static constexpr int NW = BITS / 32;       // 32-bit code words per token
    static constexpr size_t LUT_BYTES = 256 * 256;  // 256 byte values x 256-byte rows
    static constexpr size_t SMEM = LUT_BYTES + kBins * 4 + (kMaxDim + kMaxBits + 64) * 4;
};

// Rotate the token's code bytes by rho (byte r of the result = byte (r + rho)
// mod 4*NW of the input), so every lane reads its tables in a staggered order.
template <int NW>
__device__ __forceinline__ void rotate_bytes(uint32_t (&w)[NW], int rho) {
    if (NW == 4) {
        if (rho & 8) { uint32_t a = w[0], c = w[1]; w[0] = w[2]; w[1] = w[3]; w[2] = a; w[3] = c; }
        if (rho & 4) { uint32_t a = w[0]; w[0] = w[1]; w[1] = w[2]; w[2] = w[3]; w[3] = a; }
    } else if (NW == 2) {
        if (rho & 4) { uint32_t a = w[0]; w[0] = w[1]; w[1] = a; }
    }
    const int sh = 8 * (rho & 3);
    uint32_t o[NW];
#pragma unroll
    for (int k = 0; k < NW; ++k) o[k] = __funnelshift_r(w[k], w[(k + 1) % NW], sh);
#pragma unroll
    for (int k = 0; k < NW; ++k) w[k] = o[k];
}

template <int BITS>
__device__ __forceinline__ void load_code(const uint64_t *p, uint32_t (&w)[BITS / 32]) {
    if (BITS == 128) {
        uint4 x = __ldcs(reinterpret_cast<const uint4 *>(p));
        w[0] = x.x; w[1] = x.y; w[2 % (BITS / 32)] = x.z; w[3 % (BITS / 32)] = x.w;
    } else {
        uint2 x = __ldcs(reinterpret_cast<const uint2 *>(p));
        w[0] = x.x;
        if (BITS == 64) w[1 % (BITS / 32)] = x.y;
    }
}

template <int BITS, int D>
__global__ void __launch_bounds__(kSelThreads, 2)
score_hist_kernel(KV kv, const __nv_bfloat16 *__restrict__ q, int Hq, int G,
                  const int32_t *__restrict__ seq_lens, const RBits R, SelWS ws, int topk, int nctas) {
    using S = ScoreShape<BITS>;
    constexpr int T = S::T, NW = S::NW;
    extern __shared__ __align__(1024) unsigned char smem[];
    unsigned char *lut = smem;                                            // [256][256 B]
    uint32_t *hist = reinterpret_cast<uint32_t *>(smem + S::LUT_BYTES);   // [kBins]
    float *qsum = reinterpret_cast<float *>(hist + kBins);                // [D]
    float *Qp = qsum + kMaxDim;                                           // [BITS]
    float *red = Qp + kMaxBits;                                           // [64]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bh = blockIdx.y, b = bh / kv.Hkv, h = bh % kv.Hkv;
    const int64_t n = clamp_len(kv, seq_lens, b);

    for (int i = tid; i < kBins; i += kSelThreads) hist[i] = 0;
    for (int i = tid; i < D; i += kSelThreads) {
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
        if (lane == 0) {
            red[0] = a;
            red[1] = a > 0.0f ? (float)kBins / (2.0f * a) : 0.0f;
        }
    }
    // LUT_c[v] for the T byte tables, replicated COPIES times per 256-byte row:
    // word (v * 64 + copy * T + c).
    {
        const int v = tid & 255;
        for (int c = tid >> 8; c < T; c += kSelThreads / 256) {
            float val = 0.0f;
#pragma unroll
            for (int u = 0; u < 8; ++u) val += ((v >> u) & 1) ? Qp[8 * c + u] : -Qp[8 * c + u];
            float *row = reinterpret_cast<float *>(lut + v * 256);
#pragma unroll
            for (int cp = 0; cp < S::COPIES; ++cp) row[cp * T + c] = val;
        }
    }
    __syncthreads();
    const float A = red[0], inv_w = red[1];

    int64_t t0, t1;
    cta_range(n, blockIdx.x, nctas, t0, t1);
    const int rho = lane % T, copy = lane / T;
    uint32_t off[T];
#pragma unroll
    for (int r = 0; r < T; ++r) off[r] = 4u * (uint32_t)(copy * T + (rho + r) % T);

    float *srow = ws.scores + (int64_t)bh * ws.ld;
    constexpr int U = 4;
    constexpr int NWARPS = kSelThreads / 32;
    for (int64_t g0 = t0 + warp * 32; g0 < t1; g0 += (int64_t)NWARPS * 32 * U) {
        uint32_t w[U][NW];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t t = g0 + (int64_t)u * NWARPS * 32 + lane;
#pragma unroll
            for (int k = 0; k < NW; ++k) w[u][k] = 0;
            if (t < t1) {
                int64_t c = kv.code(b, h, t);
                if (c >= 0) load_code<BITS>(kv.codes + c, w[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t t = g0 + (int64_t)u * NWARPS * 32 + lane;
            rotate_bytes<NW>(w[u], rho);
            float s = 0.0f;
#pragma unroll
            for (int r = 0; r < T; ++r) {
                uint32_t addr = __byte_perm(w[u][r >> 2], off[r], 0x7604u | ((uint32_t)(r & 3) << 4));
                s += *reinterpret_cast<const float *>(lut + addr);
            }
            s += 0.0f;
            if (t < t1) {
                srow[t] = s;
                atomicAdd(&hist[score_bin(s, A, inv_w)], 1u);
            }
        }
    }
    __syncthreads();
    uint32_t *ghist = ws.hist + (int64_t)bh * kBins;
    for (int i = tid; i < kBins; i += kSelThreads)
        if (hist[i]) atomicAdd(ghist + i, hist[i]);

    // ---- last CTA of this (b, h): locate the threshold bin
    __shared__ int s_last;
    __shared__ int s_warp[32];
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(ws.arrive + bh, 1u) == (unsigned)(nctas - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int i = tid; i < kBins; i += kSelThreads) {
        hist[i] = __ldcg(ghist + i);
        ghist[i] = 0;
    }
    __syncthreads();
    const int64_t kk = topk < n ? topk : n;
    constexpr int PER = kBins / kSelThreads;  // bins per thread, thread 0 owns the top
    int local = 0;
    const int top = kBins - 1 - tid * PER;
#pragma unroll
    for (int e = 0; e < PER; ++e) local += hist[top - e];
    int total;
    const int before = block_excl_scan(local, s_warp, &total);
    if (tid == 0) {
        SelState st;
        st.A = A; st.inv_w = inv_w; st.kk = (int32_t)kk; st.n = (int32_t)n;
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
// Resolve helpers (run by the last CTA of a (b, h) in collect_kernel).

// Visit the concatenated segments (ascending token order) in tiles of
// kSelThreads; f(e_valid, t) is called by every thread for every tile.
template <class F>
__device__ __forceinline__ void for_list_tiles(const SelWS &ws, int bh, int nctas, int n,
                                               const int *s_seg_cnt, F &&f) {
    const int32_t *cand = ws.cand + (int64_t)bh * ws.ld;
    for (int c = 0; c < nctas; ++c) {
        int64_t t0, t1;
        cta_range(n, c, nctas, t0, t1);
        const int cnt = s_seg_cnt[c];
        for (int base = 0; base < cnt; base += kSelThreads) {
            const int e = base + threadIdx.x;
            const bool valid = e < cnt;
            const int t = valid ? __ldcg(cand + t0 + e) : 0;
            f(valid, t);
        }
    }
}

__device__ __forceinline__ void write_selection(const SelWS &ws, int bh, int nctas, const SelState &st,
                                                int S, int W, int cap_sel, int32_t *sel_idx,
                                                int32_t *sel_cnt, const int *s_seg_cnt, uint32_t Tkey,
                                                int IT, int *s_warp) {
    const int n = st.n;
    int32_t *out = sel_idx + (int64_t)bh * cap_sel;
    const float *srow = ws.scores + (int64_t)bh * ws.ld;
    const int s_end = S < n ? S : n;                  // sinks [0, s_end)
    const int w_beg = n - W > s_end ? n - W : s_end;  // window [w_beg, n)
    int pos;
    if (st.flags == kStateAll) {
        for (int t = threadIdx.x; t < n; t += kSelThreads) out[t] = t;
        pos = n;
    } else if (st.flags == kStateEmpty) {
        pos = 0;
    } else {
        for (int t = threadIdx.x; t < s_end; t += kSelThreads) out[t] = t;
        pos = s_end;
        for_list_tiles(ws, bh, nctas, n, s_seg_cnt, [&](bool valid, int t) {
            bool keep = false;
            if (valid && t >= s_end && t < w_beg) {
                const float s = __ldcg(srow + t);
                const int bin = score_bin(s, st.A, st.inv_w);
                const uint32_t key = float_key(s);
                keep = bin > st.T1 || (bin == st.T1 && (key > Tkey || (key == Tkey && t <= IT)));
            }
            int tot;
            const int p = block_excl_scan(keep ? 1 : 0, s_warp, &tot);
            if (keep && pos + p < cap_sel) out[pos + p] = t;
            pos += tot;
        });
        for (int t = w_beg + threadIdx.x; t < n; t += kSelThreads)
            if (pos + (t - w_beg) < cap_sel) out[pos + (t - w_beg)] = t;
        pos += n - w_beg;
        if (pos > cap_sel) pos = cap_sel;  // unreachable when the threshold is consistent
    }
    for (int r = pos + threadIdx.x; r < cap_sel; r += kSelThreads) out[r] = -1;
    if (threadIdx.x == 0) sel_cnt[bh] = pos;
}

// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kSelThreads)
collect_kernel(const int32_t *__restrict__ seq_lens_unused, SelWS ws, int nctas, int S, int W, int cap_sel,
               int32_t *sel_idx, int32_t *sel_cnt) {
    __shared__ int s_warp[32];
    __shared__ int s_last;
    __shared__ int s_seg_cnt[kMaxSelCtas];
    __shared__ uint32_t s_ck[kCandSmem];
    __shared__ int s_ci[kCandSmem];
    __shared__ uint32_t s_h[2048];
    __shared__ int s_misc[8];
    (void)seq_lens_unused;

    const int tid = threadIdx.x;
    const int bh = blockIdx.y;
    const SelState st = ws.state[bh];
    const int n = st.n;
    int32_t *cand = ws.cand + (int64_t)bh * ws.ld;
    const float *srow = ws.scores + (int64_t)bh * ws.ld;

    int count = 0;
    if (st.flags == kStateNormal) {
        int64_t t0, t1;
        cta_range(n, blockIdx.x, nctas, t0, t1);
        for (int64_t base = t0; base < t1; base += kSelThreads) {
            const int64_t t = base + tid;
            bool f = false;
            if (t < t1) f = score_bin(__ldcg(srow + t), st.A, st.inv_w) >= st.T1;
            int tot;
            const int p = block_excl_scan(f ? 1 : 0, s_warp, &tot);
            if (f) cand[t0 + count + p] = (int32_t)t;
            count += tot;
        }
    }
    if (tid == 0) ws.seg_cnt[(int64_t)bh * kMaxSelCtas + blockIdx.x] = count;
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(ws.arrive + gridDim.y + bh, 1u) == (unsigned)(nctas - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    // ---- resolve the exact threshold (Tkey, IT) inside bin T1
    for (int c = tid; c < nctas; c += kSelThreads) s_seg_cnt[c] = __ldcg(ws.seg_cnt + (int64_t)bh * kMaxSelCtas + c);
    __syncthreads();
    uint32_t Tkey = 0;
    int IT = 0x7fffffff;
    if (st.flags == kStateNormal) {
        const int need1 = st.kk - st.above1;  // 1 <= need1 <= cnt_T1
        if (need1 < st.cnt_T1 && st.cnt_T1 <= kCandSmem) {
            if (tid == 0) s_misc[0] = 0;
            __syncthreads();
            for_list_tiles(ws, bh, nctas, n, s_seg_cnt, [&](bool valid, int t) {
                if (valid) {
                    const float s = __ldcg(srow + t);
                    if (score_bin(s, st.A, st.inv_w) == st.T1) {
                        const int slot = atomicAdd(&s_misc[0], 1);
                        s_ck[slot] = float_key(s);
                        s_ci[slot] = t;
                    }
                }
            });
            __syncthreads();
            const int c1 = s_misc[0];
            for (int e = tid; e < c1; e += kSelThreads) {
                const uint32_t ke = s_ck[e];
                const int ie = s_ci[e];
                int rank = 0;
                for (int f = 0; f < c1; ++f) {
                    const uint32_t kf = s_ck[f];
                    rank += (kf > ke) || (kf == ke && s_ci[f] < ie);
                }
                if (rank == need1 - 1) { s_misc[1] = (int)ke; s_misc[2] = ie; }
            }
            __syncthreads();
            Tkey = (uint32_t)s_misc[1];
            IT = s_misc[2];
        } else if (need1 < st.cnt_T1) {
            // Large tie-heavy bin: radix-select the key over the in-bin tokens
            // (11/11/10 bits), then the need-th tied token in index order.
            uint32_t prefix = 0, mask = 0;
            int need = need1;
            const int shifts[3] = {21, 10, 0};
            const int widths[3] = {11, 11, 10};
            for (int p = 0; p < 3; ++p) {
                const int sh = shifts[p], nb = 1 << widths[p];
                for (int i = tid; i < 2048; i += kSelThreads) s_h[i] = 0;
                __syncthreads();
                for_list_tiles(ws, bh, nctas, n, s_seg_cnt, [&](bool valid, int t) {
                    if (valid) {
                        const float s = __ldcg(srow + t);
                        const uint32_t key = float_key(s);
                        if (score_bin(s, st.A, st.inv_w) == st.T1 && (key & mask) == prefix)
                            atomicAdd(&s_h[(key >> sh) & (nb - 1)], 1u);
                    }
                });
                __syncthreads();
                if (tid == 0) {
                    int run = 0, dd = nb - 1;
                    for (; dd >= 0; --dd) {
                        if (run + (int)s_h[dd] >= need) break;
                        run += s_h[dd];
                    }
                    s_misc[3] = dd;
                    s_misc[4] = need - run;
                }
                __syncthreads();
                prefix |= (uint32_t)s_misc[3] << sh;
                mask |= (uint32_t)(nb - 1) << sh;
                need = s_misc[4];
                __syncthreads();
            }
            Tkey = prefix;
            // the need-th token (index order) among bin == T1 and key == Tkey
            int run = 0;
            if (tid == 0) s_misc[5] = 0x7fffffff;
            __syncthreads();
            for_list_tiles(ws, bh, nctas, n, s_seg_cnt, [&](bool valid, int t) {
                bool m = false;
                if (valid) {
                    const float s = __ldcg(srow + t);
                    m = score_bin(s, st.A, st.inv_w) == st.T1 && float_key(s) == Tkey;
                }
                int tot;
                const int p = block_excl_scan(m ? 1 : 0, s_warp, &tot);
                if (m && run + p + 1 == need) s_misc[5] = t;
                run += tot;
            });
            __syncthreads();
            IT = s_misc[5];
        }
    }
    write_selection(ws, bh, nctas, st, S, W, cap_sel, sel_idx, sel_cnt, s_seg_cnt, Tkey, IT, s_warp);
    if (tid == 0) ws.arrive[gridDim.y + bh] = 0;
}

}  // namespace dkv
