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
    static constexpr size_t SMEM = sizeof(float) * ((size_t)D * BITS + (size_t)D * KS_LD);
};

template <int BITS, int D>
__global__ void __launch_bounds__(128)
encode_keys_kernel(KV kv, const int32_t *__restrict__ seq_lens, const RBits R, int64_t tiles_per_seq) {
    using S = EncodeShape<BITS, D>;
    extern __shared__ float4 smem_f4[];
    float *Rf = reinterpret_cast<float *>(smem_f4);  // [D][BITS]
    float *ks = Rf + D * BITS;                       // [D][KS_LD]

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
        const int64_t t = t0 + key;
        if (t < n) {
            uint64_t word = 0;
#pragma unroll
            for (int jj = 0; jj < S::JPT; ++jj) word |= (uint64_t)(acc[jj] >= 0.0f) << jj;
            int64_t c = kv.code(b, h, t);
            if (c >= 0) kv.codes[c + grp] = word;
        }
    }
}

// ---------------------------------------------------------------------------
// Decode-step append.  One CTA per sequence, one warp per kv head: copy the new
// K/V rows into slot seq_lens[b], encode the key (lane owns hyperplanes
// lane + 32 m; the sign bits are gathered with warp ballots), then bump
// seq_lens[b].
template <int BITS, int D>
__global__ void append_keys_kernel(KV kv, const __nv_bfloat16 *__restrict__ k_new,
                                   const __nv_bfloat16 *__restrict__ v_new, int32_t *seq_lens,
                                   const RBits R) {
    __shared__ uint32_t Rb[BITS * D / 32];
    __shared__ float kf[32][D];
    __shared__ int s_ok;
    const int b = blockIdx.x;
    const int h = threadIdx.x / 32, lane = threadIdx.x % 32;
    for (int e = threadIdx.x; e < BITS * D / 32; e += blockDim.x) Rb[e] = R.w[e];

    const int64_t pos = seq_lens[b];
    if (threadIdx.x == 0) {
        int ok = pos >= 0 && pos < kv.capacity();
        if (!ok) raise_error(kErrCapacity);
        if (ok && kv.page_size) ok = kv.page_of(b, pos) >= 0;
        s_ok = ok;
    }
    __syncthreads();
    const bool ok = s_ok != 0;
    if (ok && h < kv.Hkv) {
        const int64_t r = kv.row(b, h, pos);
        const uint4 *ksrc = reinterpret_cast<const uint4 *>(k_new + ((int64_t)b * kv.Hkv + h) * D);
        const uint4 *vsrc = reinterpret_cast<const uint4 *>(v_new + ((int64_t)b * kv.Hkv + h) * D);
        constexpr int CPR = D / 8;
        for (int c = lane; c < 2 * CPR; c += 32) {
            if (c < CPR) {
                uint4 x = __ldg(ksrc + c);
                reinterpret_cast<uint4 *>(kv.k + r)[c] = x;
                kf[h][8 * c + 0] = bf16_lo(x.x); kf[h][8 * c + 1] = bf16_hi(x.x);
                kf[h][8 * c + 2] = bf16_lo(x.y); kf[h][8 * c + 3] = bf16_hi(x.y);
                kf[h][8 * c + 4] = bf16_lo(x.z); kf[h][8 * c + 5] = bf16_hi(x.z);
                kf[h][8 * c + 6] = bf16_lo(x.w); kf[h][8 * c + 7] = bf16_hi(x.w);
            } else {
                reinterpret_cast<uint4 *>(kv.v + r)[c - CPR] = __ldg(vsrc + (c - CPR));
            }
        }
        __syncwarp();
        uint32_t words[BITS / 32];
#pragma unroll
        for (int m = 0; m < BITS / 32; ++m) {
            const int j = lane + 32 * m;
            float acc = 0.0f;
            for (int i = 0; i < D; ++i) {
                float rf = ((Rb[j * (D / 32) + i / 32] >> (i % 32)) & 1u) ? -1.0f : 1.0f;
                acc = fmaf(rf, kf[h][i], acc);
            }
            words[m] = __ballot_sync(0xffffffffu, acc >= 0.0f);
        }
        if (lane == 0) {
            int64_t c = kv.code(b, h, pos);
            if (BITS == 32) {
                kv.codes[c] = (uint64_t)words[0];
            } else {
#pragma unroll
                for (int w = 0; w < BITS / 64; ++w)
                    kv.codes[c + w] = (uint64_t)words[2 * w] | ((uint64_t)words[2 * w + 1] << 32);
            }
        }
    }
    __syncthreads();
    if (threadIdx.x == 0 && ok) seq_lens[b] = (int32_t)(pos + 1);
}

}  // namespace dkv
