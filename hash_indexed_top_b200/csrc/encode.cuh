// encode.cuh -- stage 1: sign-random-projection key codes.
//
// bit_j(k) = [ sum_i R[j][i] k[i] >= 0 ] against `bits` Rademacher hyperplanes
// (DASH-KV page, section "从平方到线性：复杂度降低的数学原理": LSH codes for the
// keys; section "技术架构：动态混合精度机制": a light key-side encoder).
//
// Both kernels accumulate every projection the same way -- fp32, dims in
// ascending order, acc = fma(R[j][i], k[i], acc) from 0 -- so a key appended
// during decode gets exactly the code a one-shot encode would give it.
#pragma once
#include "common.cuh"

namespace dkv {

// ---------------------------------------------------------------------------
// Whole-cache encoder.  One CTA of 128 threads works on tiles of KT keys of one
// (b, kv head); thread (key, group) owns JPT consecutive hyperplanes of one key.
// The tile is loaded with coalesced 16-byte loads and kept transposed in shared
// memory as fp32; R is expanded once per CTA into a +-1.0 table read as
// broadcast float4s.  ALU-bound: bits * d FMAs per key.
template <int BITS, int D>
struct EncodeShape {
    static constexpr int JPT = BITS < 64 ? BITS : 64;  // hyperplanes per thread
    static constexpr int NG = BITS / JPT;              // groups per key
    static constexpr int THREADS = 128;
    static constexpr int KT = THREADS / NG;            // keys per tile
    static constexpr int KS_LD = KT + 1;               // padded row of the transposed tile
    static constexpr size_t SMEM = sizeof(float) * ((size_t)D * BITS + (size_t)D * KS_LD) + 8 * KT * NG + 8;
};

template <int BITS, int D>
__global__ void __launch_bounds__(128)
encode_keys_kernel(KV kv, const int32_t *__restrict__ seq_lens, const RBits R, int64_t tiles_per_seq) {
    using S = EncodeShape<BITS, D>;
    extern __shared__ float4 smem_f4[];
    float *Rf = reinterpret_cast<float *>(smem_f4);  // [D][BITS]
    float *ks = Rf + D * BITS;                       // [D][KS_LD]
    uint64_t *words = reinterpret_cast<uint64_t *>(ks + D * S::KS_LD);  // [KT][NG] code words of the tile

    const int bh = blockIdx.y;
    const int b = bh / kv.Hkv, h = bh % kv.Hkv;
    const int tid = threadIdx.x;
    const int64_t n = clamp_len(kv, seq_lens, b);

    for (int e = tid; e < D * BITS; e += S::THREADS) {
        int i = e / BITS, j = e % BITS;
        uint32_t w = R.w[j * (D / 32) + i / 32];
        Rf[e] = ((w >> (i % 32)) & 1u) ? -1.0f : 1.0f;
    }

    const int key = tid % S::KT;
    const int grp = tid / S::KT;
    for (int64_t tile = blockIdx.x; tile < tiles_per_seq; tile += gridDim.x) {
        const int64_t t0 = tile * S::KT;
        if (t0 >= n) break;
        __syncthreads();  // previous tile's readers are done (and Rf is built)
        constexpr int CPR = D / 8;  // 16-byte chunks per row
        for (int c = tid; c < S::KT * CPR; c += S::THREADS) {
            int kk = c / CPR, part = c % CPR;
            int64_t t = t0 + kk;
            uint4 raw = make_uint4(0, 0, 0, 0);
            if (t < n) {
                int64_t r = kv.row(b, h, t);
                if (r >= 0) raw = __ldg(reinterpret_cast<const uint4 *>(kv.k + r) + part);
            }
            float *col = ks + (part * 8) * S::KS_LD + kk;
            col[0 * S::KS_LD] = bf16_lo(raw.x);
            col[1 * S::KS_LD] = bf16_hi(raw.x);
            col[2 * S::KS_LD] = bf16_lo(raw.y);
            col[3 * S::KS_LD] = bf16_hi(raw.y);
            col[4 * S::KS_LD] = bf16_lo(raw.z);
            col[5 * S::KS_LD] = bf16_hi(raw.z);
            col[6 * S::KS_LD] = bf16_lo(raw.w);
            col[7 * S::KS_LD] = bf16_hi(raw.w);
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
                // R is +-1: each product is exact, so a packed fma per two
                // hyperplanes rounds exactly like the add (or subtract) it is
                float4 r = r4[q];
                const float2 a01 = ffma2(make_float2(r.x, r.y), make_float2(kx, kx),
                                         make_float2(acc[4 * q + 0], acc[4 * q + 1]));
                const float2 a23 = ffma2(make_float2(r.z, r.w), make_float2(kx, kx),
                                         make_float2(acc[4 * q + 2], acc[4 * q + 3]));
                acc[4 * q + 0] = a01.x; acc[4 * q + 1] = a01.y;
                acc[4 * q + 2] = a23.x; acc[4 * q + 3] = a23.y;
            }
        }
        uint64_t word = 0;
#pragma unroll
        for (int jj = 0; jj < S::JPT; ++jj) word |= (uint64_t)(acc[jj] >= 0.0f) << jj;
        words[key * S::NG + grp] = word;
        __syncthreads();
        const int64_t t = t0 + key;
        if (grp == 0 && t < n) {
            uint32_t w32[BITS / 32];
#pragma unroll
            for (int k = 0; k < BITS / 32; ++k) w32[k] = (uint32_t)(words[key * S::NG + k / 2] >> (32 * (k % 2)));
            int64_t c = kv.code(b, h, t);
            if (c >= 0) store_code_rotated<BITS>(kv.codes + c, w32, t);
        }
    }
}

// ---------------------------------------------------------------------------
// Decode-step append.  One cluster of C CTAs per sequence (C = ceil(Hkv * bits
// / kAppendSpan)): CTA c handles hpc = ceil(Hkv / C) consecutive kv heads,
// with one thread per (head, hyperplane).  It copies the new K/V rows into
// slot seq_lens[b] and encodes the new keys (one sequential FMA chain over the
// dims per hyperplane, as in the whole-cache encoder; the sign bits of a warp,
// 32 hyperplanes of one head, are gathered with one ballot).  After a cluster
// barrier -- every CTA has read seq_lens[b] -- CTA 0 bumps it.  Few, wide
// CTAs: the append runs while the scorer's CTAs (one per SM) are being
// placed, and every SM it holds is one they cannot use until it ends.
constexpr int kAppendSpan = 512;     // (head, hyperplane) pairs per CTA
constexpr int kAppendCluster = 8;

template <int BITS, int D>
__global__ void __launch_bounds__(1024)
append_keys_kernel(KV kv, const __nv_bfloat16 *__restrict__ k_new, const __nv_bfloat16 *__restrict__ v_new,
                   int32_t *seq_lens, const RBits R, int hpc) {
    constexpr int WPR = D / 32;  // R words per hyperplane
    constexpr int CPR = D / 8;   // 16-byte chunks per row
    extern __shared__ float4 kf4[];                                    // [hpc][D / 4]
    uint32_t *code32 = reinterpret_cast<uint32_t *>(kf4 + hpc * (D / 4));  // [hpc][BITS / 32]
    const int b = blockIdx.y, c = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31;
    const int Hkv = kv.Hkv;
    const int h0 = c * hpc, nh = min(hpc, Hkv - h0);  // this CTA's heads [h0, h0 + nh)
    const int hl = tid / BITS, j = tid % BITS;       // this thread's (head, hyperplane)
    uint32_t rw[WPR];  // its hyperplane (depends on the context only)
#pragma unroll
    for (int w = 0; w < WPR; ++w) rw[w] = R.w[j * WPR + w];

    griddep_wait();
    griddep_trigger();  // the scorer may start building its LUT meanwhile
    // thread e < 2 nh CPR copies 16-byte chunk e of this CTA's new K (then V)
    // rows; its load does not depend on the position, so it is issued together
    // with the position's (2 * hpc * CPR <= hpc * BITS = blockDim.x)
    const int e = tid;
    const int isv = e >= nh * CPR;
    const int ee = isv ? e - nh * CPR : e;
    const int hh = ee / CPR, part = ee % CPR;
    const bool copies = e < 2 * nh * CPR;
    uint4 x = make_uint4(0u, 0u, 0u, 0u);
    if (copies)
        x = __ldg(reinterpret_cast<const uint4 *>((isv ? v_new : k_new) + ((int64_t)b * Hkv + h0 + hh) * D) + part);
    const int64_t pos = seq_lens[b];
    bool ok = pos >= 0 && pos < kv.capacity();
    if (ok && kv.page_size) {
        const int32_t p = __ldg(kv.page_table + (int64_t)b * kv.max_pages + pos / kv.page_size);
        ok = p >= 0 && p < kv.num_pages;
        if (!ok && c == 0 && tid == 0) raise_error(kErrPage);
    } else if (!ok && c == 0 && tid == 0) {
        raise_error(kErrCapacity);
    }
    if (ok && nh > 0) {
        if (copies) {
            const int64_t r = kv.row(b, h0 + hh, pos);
            reinterpret_cast<uint4 *>((isv ? kv.v : kv.k) + r)[part] = x;
            if (!isv) {
                kf4[hh * (D / 4) + 2 * part] = make_float4(bf16_lo(x.x), bf16_hi(x.x), bf16_lo(x.y), bf16_hi(x.y));
                kf4[hh * (D / 4) + 2 * part + 1] = make_float4(bf16_lo(x.z), bf16_hi(x.z), bf16_lo(x.w), bf16_hi(x.w));
            }
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
            store_code_rotated<BITS>(kv.codes + kv.code(b, h0 + tid, pos), w32, pos);
        }
    }
    cluster_sync();  // every CTA of this sequence has read seq_lens[b]
    if (c == 0 && tid == 0 && ok) seq_lens[b] = (int32_t)(pos + 1);
}

}  // namespace dkv
