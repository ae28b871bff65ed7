// radius.cuh -- 8-bit key-norm codes for radius-scaled scores.
//
// Spherical KV page, section 2.1 ADA: a compact key keeps a quantized radius
// r~ beside its angle code, and the logit is estimated as |q| r~ f_b(codes).
// Here the sign code's asymmetric score plays f_b and the selection ranks
// s' = r~ s (|q| is one constant per query).  The page fixes no quantizer; the
// one used is 8 bits, uniform in the norm with step 1/4:
//   c = min(255, floor(4 sqrt(sum_i k_i^2))),  r~ = (c + 1/2) / 4,
// with the sum taken in fp32 over i ascending and every operation rounded
// once (no fused multiply-add), so that any implementation decides c alike;
// on keys of the 1/64 grid the sum is exact.
#pragma once
#include "common.cuh"

namespace dkv {

constexpr int kRadiusThreads = 256;

// Radius code of one bf16 key row of D values.
template <int D>
__device__ __forceinline__ uint8_t radius_code(const __nv_bfloat16 *row) {
    float s = 0.0f;
#pragma unroll 4
    for (int c = 0; c < D / 8; ++c) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(row) + c);
        const float x[8] = {bf16_lo(raw.x), bf16_hi(raw.x), bf16_lo(raw.y), bf16_hi(raw.y),
                            bf16_lo(raw.z), bf16_hi(raw.z), bf16_lo(raw.w), bf16_hi(raw.w)};
#pragma unroll
        for (int e = 0; e < 8; ++e) s = __fadd_rn(s, __fmul_rn(x[e], x[e]));
    }
    const float v = floorf(4.0f * __fsqrt_rn(s));
    return v >= 255.0f ? (uint8_t)255 : (uint8_t)v;
}

// Codes of tokens [0, seq_lens[b]) of every (b, kv head): one thread per token.
template <int D>
__global__ void __launch_bounds__(kRadiusThreads)
radius_codes_kernel(KV kv, const int32_t *__restrict__ seq_lens, uint8_t *__restrict__ out) {
    const int bh = blockIdx.y, b = bh / kv.Hkv, h = bh % kv.Hkv;
    const int64_t n = clamp_len(kv, seq_lens, b);
    for (int64_t t = (int64_t)blockIdx.x * kRadiusThreads + threadIdx.x; t < n;
         t += (int64_t)gridDim.x * kRadiusThreads) {
        const int64_t r = kv.row(b, h, t);
        if (r < 0) continue;
        out[kv.radius_index(b, h, t)] = radius_code<D>(kv.k + r);
    }
}

// Decode step, after the append: the code of token seq_lens[b] - 1 (the one
// the append wrote) of every kv head; CTA b, thread h.
template <int D>
__global__ void __launch_bounds__(32)
append_radius_kernel(KV kv, const int32_t *__restrict__ seq_lens, uint8_t *__restrict__ out) {
    griddep_wait();  // the append and its length update are complete
    griddep_trigger();
    const int b = blockIdx.x, h = threadIdx.x;
    if (h >= kv.Hkv) return;
    const int64_t t = (int64_t)seq_lens[b] - 1;
    if (t < 0 || t >= kv.capacity()) return;
    const int64_t r = kv.row(b, h, t);
    if (r < 0) return;
    out[kv.radius_index(b, h, t)] = radius_code<D>(kv.k + r);
}

}  // namespace dkv
