// decode.cuh -- stage 4: exact softmax attention over the selected rows only
// (DeepSeek DSA->CSA/HCA page, section "从 DSA 说起": real attention runs on the
// top-k the indexer picked; DASH-KV page, section "技术架构：动态混合精度机制":
// the tokens that matter are attended in full precision).
//
// Gathered split-K flash-decode: grid = (splits, B * Hkv).  Each CTA takes a
// contiguous slice of one (b, kv head)'s selected ids, gathers each K/V row
// once (16-byte loads, LPR = d/8 lanes per row) and serves all G query heads of
// the group from it, keeping a running (max, sum, acc) per head in fp32 with
// base-2 exponentials.  The per-CTA partials go to the workspace; the last CTA
// of the (b, h) (atomic arrival counter, no waiting) merges them with a
// log-sum-exp reduction and writes out / lse.
#pragma once
#include "common.cuh"

namespace dkv {

constexpr int kAttnThreads = 128;
constexpr int kMaxSplits = 256;

struct AttnWS {
    float *part;        // [BH][kMaxSplits][G][D + 2]  (acc[D], m, l)
    uint32_t *arrive;   // [BH]   zero between calls
};

template <int D, int G>
__global__ void __launch_bounds__(kAttnThreads)
sparse_decode_kernel(KV kv, const __nv_bfloat16 *__restrict__ q, int Hq,
                     const int32_t *__restrict__ sel_idx, const int32_t *__restrict__ sel_cnt, int cap_sel,
                     float *__restrict__ out, float *__restrict__ lse, AttnWS ws, int splits, float scale_log2) {
    constexpr int LPR = D / 8;        // lanes per row (8 bf16 = 16 B each)
    constexpr int RPW = 32 / LPR;     // rows per warp step
    constexpr int NWARP = kAttnThreads / 32;
    constexpr int NST = NWARP * RPW;  // independent running states per CTA
    constexpr int U = 4;              // rows in flight per lane group
    __shared__ float s_m[NST][G], s_l[NST][G];
    __shared__ float s_acc[NST][G][D];
    __shared__ int s_last;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int sub = lane / LPR, li = lane % LPR;
    const int bh = blockIdx.y, b = bh / kv.Hkv, h = bh % kv.Hkv;
    const int split = blockIdx.x;
    int cnt = sel_cnt[bh];
    if (cnt > cap_sel) cnt = cap_sel;
    if (cnt < 0) cnt = 0;
    const int64_t cap_tokens = kv.capacity();
    const int per = (cnt + splits - 1) / splits;
    const int r0 = split * per;
    const int r1 = r0 + per < cnt ? r0 + per : cnt;

    float qf[G][8];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(q + ((int64_t)b * Hq + h * G + g) * D) + li);
        qf[g][0] = bf16_lo(raw.x); qf[g][1] = bf16_hi(raw.x);
        qf[g][2] = bf16_lo(raw.y); qf[g][3] = bf16_hi(raw.y);
        qf[g][4] = bf16_lo(raw.z); qf[g][5] = bf16_hi(raw.z);
        qf[g][6] = bf16_lo(raw.w); qf[g][7] = bf16_hi(raw.w);
    }
    float m[G], l[G], acc[G][8];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m[g] = -INFINITY;
        l[g] = 0.0f;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[g][e] = 0.0f;
    }

    const int32_t *ids = sel_idx + (int64_t)bh * cap_sel;
    const int stride = NST;
    // warp-uniform loop (the dot-product reduction shuffles across the whole warp)
    for (int rw = r0 + warp * RPW; rw < r1; rw += stride * U) {
        uint4 kr[U], vr[U];
        bool ok[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int r = rw + sub + u * stride;
            ok[u] = false;
            kr[u] = make_uint4(0, 0, 0, 0);
            vr[u] = make_uint4(0, 0, 0, 0);
            if (r < r1) {
                const int t = __ldg(ids + r);
                int64_t off = -1;
                if (t >= 0 && t < cap_tokens) off = kv.row(b, h, t);
                else raise_error(kErrCapacity);
                if (off >= 0) {
                    ok[u] = true;
                    kr[u] = __ldg(reinterpret_cast<const uint4 *>(kv.k + off) + li);
                    vr[u] = __ldg(reinterpret_cast<const uint4 *>(kv.v + off) + li);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            // lanes of a row group share ok[u] (same row); groups differ only at the tail
            float kf[8] = {bf16_lo(kr[u].x), bf16_hi(kr[u].x), bf16_lo(kr[u].y), bf16_hi(kr[u].y),
                           bf16_lo(kr[u].z), bf16_hi(kr[u].z), bf16_lo(kr[u].w), bf16_hi(kr[u].w)};
            float vf[8] = {bf16_lo(vr[u].x), bf16_hi(vr[u].x), bf16_lo(vr[u].y), bf16_hi(vr[u].y),
                           bf16_lo(vr[u].z), bf16_hi(vr[u].z), bf16_lo(vr[u].w), bf16_hi(vr[u].w)};
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float dot = 0.0f;
#pragma unroll
                for (int e = 0; e < 8; ++e) dot = fmaf(qf[g][e], kf[e], dot);
#pragma unroll
                for (int o = LPR / 2; o; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
                if (ok[u]) {
                    const float x = dot * scale_log2;
                    const float mn = fmaxf(m[g], x);
                    const float c = exp2f(m[g] - mn);
                    const float p = exp2f(x - mn);
                    l[g] = fmaf(l[g], c, p);
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[g][e] = fmaf(acc[g][e], c, p * vf[e]);
                    m[g] = mn;
                }
            }
        }
    }

    // merge the NST running states of this CTA
    const int st = warp * RPW + sub;
#pragma unroll
    for (int g = 0; g < G; ++g) {
        if (li == 0) { s_m[st][g] = m[g]; s_l[st][g] = l[g]; }
#pragma unroll
        for (int e = 0; e < 8; ++e) s_acc[st][g][8 * li + e] = acc[g][e];
    }
    __syncthreads();
    float *part = ws.part + ((int64_t)bh * kMaxSplits + split) * G * (D + 2);
    for (int x = tid; x < G * D; x += kAttnThreads) {
        const int g = x / D, i = x % D;
        float M = -INFINITY;
#pragma unroll
        for (int s = 0; s < NST; ++s) M = fmaxf(M, s_m[s][g]);
        float L = 0.0f, Acc = 0.0f;
        if (M != -INFINITY) {
#pragma unroll
            for (int s = 0; s < NST; ++s) {
                const float c = exp2f(s_m[s][g] - M);
                L = fmaf(s_l[s][g], c, L);
                Acc = fmaf(s_acc[s][g][i], c, Acc);
            }
        }
        part[g * (D + 2) + i] = Acc;
        if (i == 0) { part[g * (D + 2) + D] = M; part[g * (D + 2) + D + 1] = L; }
    }

    // the last CTA of this (b, h) merges the splits
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(ws.arrive + bh, 1u) == (unsigned)(splits - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const float *base = ws.part + (int64_t)bh * kMaxSplits * G * (D + 2);
    for (int x = tid; x < G * D; x += kAttnThreads) {
        const int g = x / D, i = x % D;
        float M = -INFINITY;
        for (int s = 0; s < splits; ++s) M = fmaxf(M, __ldcg(base + (s * G + g) * (D + 2) + D));
        float L = 0.0f, Acc = 0.0f;
        if (M != -INFINITY) {
            for (int s = 0; s < splits; ++s) {
                const float *ps = base + (s * G + g) * (D + 2);
                const float c = exp2f(__ldcg(ps + D) - M);
                L = fmaf(__ldcg(ps + D + 1), c, L);
                Acc = fmaf(__ldcg(ps + i), c, Acc);
            }
        }
        const int64_t oq = (int64_t)b * Hq + h * G + g;
        out[oq * D + i] = L > 0.0f ? Acc / L : 0.0f;
        if (i == 0 && lse) lse[oq] = L > 0.0f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
    }
    if (tid == 0) ws.arrive[bh] = 0;
}

}  // namespace dkv
