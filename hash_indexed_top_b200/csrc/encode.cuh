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
// Decode-step append.  One cluster of C = min(Hkv, kAppendCluster) CTAs per
// sequence; CTA c handles kv heads c, c + C, ...: it copies the new K/V rows
// into slot seq_lens[b] and encodes the new key (thread j = hyperplane j, one
// sequential FMA chain over the dims as in the whole-cache encoder; the sign
// bits of a warp are gathered with one ballot).  After a cluster barrier --
// every CTA has read seq_lens[b] -- CTA 0 bumps it.
constexpr int kAppendThreads = 128;
constexpr int kAppendCluster = 8;

template <int BITS, int D>
__global__ void __launch_bounds__(kAppendThreads)
append_keys_kernel(KV kv, const __nv_bfloat16 *__restrict__ k_new, const __nv_bfloat16 *__restrict__ v_new,
                   int32_t *seq_lens, const RBits R) {
    constexpr int WPR = D / 32;  // R words per hyperplane
    constexpr int CPR = D / 8;   // 16-byte chunks per row
    __shared__ float4 kf4[D / 4];
    __shared__ uint32_t code32[BITS / 32];
    const int b = blockIdx.y, c = blockIdx.x, C = gridDim.x;
    const int tid = threadIdx.x, lane = tid & 31;
    const int Hkv = kv.Hkv;
    uint32_t rw[WPR];  // this thread's hyperplane (depends on the context only)
#pragma unroll
    for (int w = 0; w < WPR; ++w) rw[w] = tid < BITS ? R.w[tid * WPR + w] : 0u;

    griddep_wait();
    griddep_trigger();  // the scorer may start building its LUT meanwhile
    const int64_t pos = seq_lens[b];
    bool ok = pos >= 0 && pos < kv.capacity();
    if (ok && kv.page_size) {
        const int32_t p = __ldg(kv.page_table + (int64_t)b * kv.max_pages + pos / kv.page_size);
        ok = p >= 0 && p < kv.num_pages;
        if (!ok && c == 0 && tid == 0) raise_error(kErrPage);
    } else if (!ok && c == 0 && tid == 0) {
        raise_error(kErrCapacity);
    }
    if (ok) {
        for (int h = c; h < Hkv; h += C) {
            const int64_t r = kv.row(b, h, pos);
            for (int e = tid; e < 2 * CPR; e += kAppendThreads) {
                const int isv = e >= CPR;
                const int part = isv ? e - CPR : e;
                const uint4 *src = reinterpret_cast<const uint4 *>((isv ? v_new : k_new) + ((int64_t)b * Hkv + h) * D);
                const uint4 x = __ldg(src + part);
                reinterpret_cast<uint4 *>((isv ? kv.v : kv.k) + r)[part] = x;
                if (!isv) {
                    kf4[2 * part] = make_float4(bf16_lo(x.x), bf16_hi(x.x), bf16_lo(x.y), bf16_hi(x.y));
                    kf4[2 * part + 1] = make_float4(bf16_lo(x.z), bf16_hi(x.z), bf16_lo(x.w), bf16_hi(x.w));
                }
            }
            __syncthreads();
            if (tid < BITS) {  // whole warps (BITS is a multiple of 32)
                float acc = 0.0f;
#pragma unroll
                for (int i4 = 0; i4 < D / 4; ++i4) {
                    const float4 k4 = kf4[i4];
                    const float kx[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int i = 4 * i4 + u;
                        const float rf = ((rw[i / 32] >> (i % 32)) & 1u) ? -1.0f : 1.0f;
                        acc = fmaf(rf, kx[u], acc);
                    }
                }
                const uint32_t word = __ballot_sync(0xffffffffu, acc >= 0.0f);
                if (lane == 0) code32[tid >> 5] = word;
            }
            __syncthreads();
            if (tid == 0) {
                uint32_t w32[BITS / 32];
#pragma unroll
                for (int k = 0; k < BITS / 32; ++k) w32[k] = code32[k];
                store_code_rotated<BITS>(kv.codes + kv.code(b, h, pos), w32, pos);
            }
            __syncthreads();  // kf4 and code32 are reused by the next head
        }
    }
    cluster_sync();  // every CTA of this sequence has read seq_lens[b]
    if (c == 0 && tid == 0 && ok) seq_lens[b] = (int32_t)(pos + 1);
}

}  // namespace dkv
