// blocks.cuh -- block summaries: a CSA-style two-level index over the cache.
//
// DeepSeek DSA->CSA/HCA page, section CSA: every m history tokens are
// compressed into one summary entry and the top-k is taken over the
// summaries, while a sliding window keeps the recent tokens exact; section on
// the compressed versus the state cache: tokens of a block that is not yet
// complete wait in the state cache until m have arrived.
//
// The pages' compressor is learned; this library has none.  The summary of
// block i (tokens [i m, (i + 1) m)) is the hash code of the block's summed key
// -- the sign of a projection of the mean key is that of the sum -- stored in
// a dense array of block codes that the ordinary scorer and selector read as a
// cache of N / m "tokens" (KV::len_shift = log2 m).  Attention stays exact:
// expand_blocks_kernel turns the selected blocks into their tokens, united
// with the sinks and the window (which holds the incomplete tail), in the list
// format of the token selection, and the ordinary sparse decode reads it.
//
// Exactness: on keys of the 1/64 grid the fp32 block sums and projections are
// exact multiples of 1/64 (far below 2^24 units), so every code equals the one
// computed in any order or precision.
#pragma once
#include "common.cuh"
#include "encode.cuh"
#include "select.cuh"  // block_excl_scan

namespace dkv {

constexpr int kExpandThreads = 256;

// Sum over rows [t0, t0 + m) of (b, h) of their 16-byte chunk `part` (8 bf16
// values), in token order (a row whose page is invalid adds nothing; the error
// word is set).
__device__ __forceinline__ void block_chunk_sum(const KV &kv, int b, int h, int64_t t0, int m, int part,
                                                float (&s)[8]) {
#pragma unroll
    for (int e = 0; e < 8; ++e) s[e] = 0.0f;
    for (int u = 0; u < m; ++u) {
        const int64_t r = kv.row(b, h, t0 + u);
        if (r < 0) continue;
        const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(kv.k + r) + part);
        s[0] += bf16_lo(raw.x);
        s[1] += bf16_hi(raw.x);
        s[2] += bf16_lo(raw.y);
        s[3] += bf16_hi(raw.y);
        s[4] += bf16_lo(raw.z);
        s[5] += bf16_hi(raw.z);
        s[6] += bf16_lo(raw.w);
        s[7] += bf16_hi(raw.w);
    }
}

// ---------------------------------------------------------------------------
// Whole-cache block encoder: the tiling of encode_keys_kernel (tiles of KT
// blocks of one (b, kv head), thread (block, group) owns JPT hyperplanes), with
// each tile row the sum of a block's m key rows.
template <int BITS, int D>
__global__ void __launch_bounds__(128)
encode_blocks_kernel(KV kv, KV blk, const int32_t *__restrict__ seq_lens, const RBits R, int64_t tiles_per_seq) {
    using S = EncodeShape<BITS, D>;
    extern __shared__ float4 smem_f4[];
    float *Rf = reinterpret_cast<float *>(smem_f4);  // [D][BITS]
    float *ks = Rf + D * BITS;                       // [D][KS_LD]
    uint64_t *words = reinterpret_cast<uint64_t *>(ks + D * S::KS_LD);  // [KT][NG]

    const int bh = blockIdx.y;
    const int b = bh / kv.Hkv, h = bh % kv.Hkv;
    const int tid = threadIdx.x;
    const int m = 1 << blk.len_shift;
    // complete blocks inside both capacities
    const int64_t n_tok = clamp_len(kv, seq_lens, b);
    int64_t nb = clamp_len(blk, seq_lens, b);
    if (nb > (n_tok >> blk.len_shift)) nb = n_tok >> blk.len_shift;

    for (int e = tid; e < D * BITS; e += S::THREADS) {
        int i = e / BITS, j = e % BITS;
        uint32_t w = R.w[j * (D / 32) + i / 32];
        Rf[e] = ((w >> (i % 32)) & 1u) ? -1.0f : 1.0f;
    }

    const int key = tid % S::KT;
    const int grp = tid / S::KT;
    for (int64_t tile = blockIdx.x; tile < tiles_per_seq; tile += gridDim.x) {
        const int64_t i0 = tile * S::KT;
        if (i0 >= nb) break;
        __syncthreads();
        constexpr int CPR = D / 8;
        for (int c = tid; c < S::KT * CPR; c += S::THREADS) {
            const int kk = c / CPR, part = c % CPR;
            const int64_t i = i0 + kk;
            float s[8];
            if (i < nb) {
                block_chunk_sum(kv, b, h, i * m, m, part, s);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) s[e] = 0.0f;
            }
            float *col = ks + (part * 8) * S::KS_LD + kk;
#pragma unroll
            for (int e = 0; e < 8; ++e) col[e * S::KS_LD] = s[e];
        }
        __syncthreads();

        float acc[S::JPT];
#pragma unroll
        for (int jj = 0; jj < S::JPT; ++jj) acc[jj] = 0.0f;
        const float *rrow = Rf + grp * S::JPT;
#pragma unroll 2
        for (int i = 0; i < D; ++i) {
            const float kx = ks[i * S::KS_LD + key];
            const float4 *r4 = reinterpret_cast<const float4 *>(rrow + i * BITS);
#pragma unroll
            for (int q = 0; q < S::JPT / 4; ++q) {
                float4 r = r4[q];
                acc[4 * q + 0] = fmaf(r.x, kx, acc[4 * q + 0]);
                acc[4 * q + 1] = fmaf(r.y, kx, acc[4 * q + 1]);
                acc[4 * q + 2] = fmaf(r.z, kx, acc[4 * q + 2]);
                acc[4 * q + 3] = fmaf(r.w, kx, acc[4 * q + 3]);
            }
        }
        uint64_t word = 0;
#pragma unroll
        for (int jj = 0; jj < S::JPT; ++jj) word |= (uint64_t)(acc[jj] >= 0.0f) << jj;
        words[key * S::NG + grp] = word;
        __syncthreads();
        const int64_t i = i0 + key;
        if (grp == 0 && i < nb) {
            uint32_t w32[BITS / 32];
#pragma unroll
            for (int k = 0; k < BITS / 32; ++k) w32[k] = (uint32_t)(words[key * S::NG + k / 2] >> (32 * (k % 2)));
            store_code_rotated<BITS>(blk.codes + blk.code(b, h, i), w32, i);
        }
    }
}

// ---------------------------------------------------------------------------
// Decode-step block update, after the append: when seq_lens[b] is a multiple
// of m, the append just completed block seq_lens[b] / m - 1; its summary is
// encoded for every kv head.  CTA (c, b) takes hpc consecutive kv heads with
// one thread per (head, hyperplane), as the append does; the block's rows are
// summed into shared memory first.
template <int BITS, int D>
__global__ void __launch_bounds__(1024)
append_blocks_kernel(KV kv, KV blk, const int32_t *__restrict__ seq_lens, const RBits R, int hpc) {
    constexpr int WPR = D / 32;
    constexpr int CPR = D / 8;
    extern __shared__ float4 kf4[];                                        // [hpc][D / 4]
    uint32_t *code32 = reinterpret_cast<uint32_t *>(kf4 + hpc * (D / 4));  // [hpc][BITS / 32]
    const int b = blockIdx.y, c = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31;
    const int h0 = c * hpc, nh = min(hpc, kv.Hkv - h0);
    const int hl = tid / BITS, j = tid % BITS;
    uint32_t rw[WPR];
#pragma unroll
    for (int w = 0; w < WPR; ++w) rw[w] = R.w[j * WPR + w];

    griddep_wait();  // the append and its length update are complete
    griddep_trigger();
    const int64_t n = clamp_len(kv, seq_lens, b);
    const int m = 1 << blk.len_shift;
    if (nh <= 0 || n == 0 || (n & (m - 1))) return;  // uniform over the CTA
    const int64_t i = (n >> blk.len_shift) - 1;
    if (i >= blk.n_cap) {
        if (c == 0 && tid == 0) raise_error(kErrCapacity);
        return;
    }
    for (int e = tid; e < nh * CPR; e += blockDim.x) {
        const int hh = e / CPR, part = e % CPR;
        float s[8];
        block_chunk_sum(kv, b, h0 + hh, i * m, m, part, s);
        kf4[hh * (D / 4) + 2 * part] = make_float4(s[0], s[1], s[2], s[3]);
        kf4[hh * (D / 4) + 2 * part + 1] = make_float4(s[4], s[5], s[6], s[7]);
    }
    __syncthreads();
    if (hl < nh) {  // whole warps: a warp is 32 hyperplanes of one head
        const float4 *kh = kf4 + hl * (D / 4);
        float acc = 0.0f;
#pragma unroll
        for (int i4 = 0; i4 < D / 4; ++i4) {
            const float4 k4 = kh[i4];
            const uint32_t wbits = rw[i4 / 8] >> (4 * (i4 % 8));
            acc = fmaf((wbits & 1u) ? -1.0f : 1.0f, k4.x, acc);
            acc = fmaf((wbits & 2u) ? -1.0f : 1.0f, k4.y, acc);
            acc = fmaf((wbits & 4u) ? -1.0f : 1.0f, k4.z, acc);
            acc = fmaf((wbits & 8u) ? -1.0f : 1.0f, k4.w, acc);
        }
        const uint32_t word = __ballot_sync(0xffffffffu, acc >= 0.0f);
        if (lane == 0) code32[hl * (BITS / 32) + j / 32] = word;
    }
    __syncthreads();
    if (tid < nh) {
        uint32_t w32[BITS / 32];
#pragma unroll
        for (int k = 0; k < BITS / 32; ++k) w32[k] = code32[tid * (BITS / 32) + k];
        store_code_rotated<BITS>(blk.codes + blk.code(b, h0 + tid, i), w32, i);
    }
}

// ---------------------------------------------------------------------------
// Block ids -> token list.  One CTA per (b, kv head).  The selected blocks come
// ascending (the selector's output); the list written is ascending and
// duplicate-free, laid out as the token selection lays out its own: the sinks
// [0, s_end), then the tokens of the selected blocks inside [s_end, w_beg),
// then the window [w_beg, n) -- which holds the incomplete tail, as window >=
// m - 1 -- and -1 up to cap_sel.  Thread r takes consecutive blocks; one block
// scan places their tokens.
__global__ void __launch_bounds__(kExpandThreads)
expand_blocks_kernel(const int32_t *__restrict__ blk_idx, const int32_t *__restrict__ blk_cnt, int kb,
                     const int32_t *__restrict__ seq_lens, int64_t cap_tokens, int Hkv, int len_shift, int S, int W,
                     int cap_sel, int32_t *__restrict__ sel_idx, int32_t *__restrict__ sel_cnt) {
    __shared__ int s_warp[32];
    // The decode may launch now: its window CTAs read only what the append
    // wrote (complete before the selection, which this kernel follows, began),
    // its other CTAs wait for this kernel to complete.
    griddep_trigger();
    griddep_wait();  // the block selection is complete
    const int bh = blockIdx.x, b = bh / Hkv, tid = threadIdx.x;
    int64_t n = seq_lens[b];
    n = n < 0 ? 0 : (n > cap_tokens ? cap_tokens : n);
    const int m = 1 << len_shift;
    const int s_end = (int)(S < n ? S : n);
    const int w_beg = (int)(n - W > s_end ? n - W : s_end);
    int cb = blk_cnt[bh];
    cb = cb < 0 ? 0 : (cb > kb ? kb : cb);
    const int32_t *ids = blk_idx + (int64_t)bh * kb;
    const int per = (cb + kExpandThreads - 1) / kExpandThreads;
    const int r0 = min(cb, tid * per), r1 = min(cb, r0 + per);
    // tokens of block id in [s_end, w_beg)
    auto span = [&](int id, int &lo, int &hi) {
        lo = max(id * m, s_end);
        hi = min(id * m + m, w_beg);
    };
    int mine = 0;
    for (int r = r0; r < r1; ++r) {
        int lo, hi;
        span(ids[r], lo, hi);
        mine += hi > lo ? hi - lo : 0;
    }
    int mid;
    int pos = s_end + block_excl_scan<kExpandThreads>(mine, s_warp, &mid);
    int32_t *out = sel_idx + (int64_t)bh * cap_sel;
    for (int r = r0; r < r1; ++r) {
        int lo, hi;
        span(ids[r], lo, hi);
        for (int t = lo; t < hi; ++t) out[pos++] = t;
    }
    for (int t = tid; t < s_end; t += kExpandThreads) out[t] = t;
    const int nwin = (int)n - w_beg;
    for (int t = tid; t < nwin; t += kExpandThreads) out[s_end + mid + t] = w_beg + t;
    const int cnt = s_end + mid + nwin;
    for (int t = cnt + tid; t < cap_sel; t += kExpandThreads) out[t] = -1;
    if (tid == 0) sel_cnt[bh] = cnt;
}

}  // namespace dkv
