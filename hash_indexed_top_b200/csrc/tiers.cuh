// tiers.cuh -- precision tiers of KV pages.
//
// Tier-homogeneous pages (Spherical KV page, section 2.2 RDR: each retained
// state gets a precision tier, protected states keep the highest, and states
// are grouped into pages of one tier so that the decode reads a page in one
// pass guided by its header; DASH-KV page, section
// "技术架构：动态混合精度机制", paras 2-3: the tokens that matter keep full
// floating-point precision, the rest a cheaper form; DeepSeek DSA->CSA/HCA
// page: the KV store itself is mixed-precision).
//
// Two tiers.  Tier 0: the bf16 rows.  Tier 1: FP8 E4M3 rows with one
// power-of-two scale per (token, kv head) row and tensor: s = the largest
// integer with amax * 2^s <= 448 (the largest finite E4M3), capped at 127, 0
// for a zero row; code_i = E4M3(x_i * 2^s) rounded to nearest even; the row
// reads back as value(code_i) * 2^-s, which bf16 and fp32 hold exactly.
// The page header is one tier byte per physical page.  The controller below
// demotes a page once all its tokens lie between the sinks and the window of
// their sequence, unless the caller protects it.  A demoted page's bf16 rows
// are no longer read by the tiered decode.
//
// Layouts (paged caches only): k8 / v8 [P][page][Hkv][d] uint8 (the K / V page
// layout, one byte per element), exps [P][page][Hkv][2] int8 (s of the K row,
// then of the V row), tier [P] uint8.
#pragma once
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"

namespace dkv {

struct Tiers {
    uint8_t *tier;        // [P]: 0 = bf16 rows, 1 = FP8 rows
    uint8_t *k8;          // [P][page][Hkv][d]
    uint8_t *v8;
    int8_t *exps;         // [P][page][Hkv][2]
};

constexpr int kDemoteThreads = 256;

// 2^-s for s in [-127, 127] (exact; 2^-127 is an fp32 subnormal).
__device__ __forceinline__ float pow2_neg(int s) {
    return s < 127 ? __int_as_float((127 - s) << 23) : __int_as_float(1 << 22);
}

// Two E4M3 codes (low byte first) as floats (exact).
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t two) {
    const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two & 0xffffu), __NV_E4M3);
    return __half22float2(__half2(hr));
}

// n (4, 8 or 16) codes at p (aligned to n bytes), times `scale`.
template <int N>
__device__ __forceinline__ void e4m3_row(const uint8_t *p, float scale, float *o) {
    uint32_t w[N / 4];
    if constexpr (N == 16) {
        const uint4 v = *reinterpret_cast<const uint4 *>(p);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if constexpr (N == 8) {
        const uint2 v = *reinterpret_cast<const uint2 *>(p);
        w[0] = v.x; w[1] = v.y;
    } else {
        static_assert(N == 4, "4, 8 or 16 codes");
        w[0] = *reinterpret_cast<const uint32_t *>(p);
    }
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
        const float2 lo = e4m3x2_to_float2(w[i]), hi = e4m3x2_to_float2(w[i] >> 16);
        o[4 * i + 0] = lo.x * scale;
        o[4 * i + 1] = lo.y * scale;
        o[4 * i + 2] = hi.x * scale;
        o[4 * i + 3] = hi.y * scale;
    }
}

// Scale exponent of a row whose largest magnitude is amax (see above).
__device__ __forceinline__ int tier_exponent(float amax) {
    if (amax == 0.0f) return 0;
    int E;
    const float f = frexpf(amax, &E);  // amax = f 2^E, f in [0.5, 1); 448 = 0.875 2^9
    const int s = f <= 0.875f ? 9 - E : 8 - E;
    return s > 127 ? 127 : s;
}

// One warp quantizes one row of D bf16 (DPL = D / 32 per lane).
template <int D>
__device__ __forceinline__ int8_t quantize_row(const __nv_bfloat16 *src, uint8_t *dst, int lane) {
    constexpr int DPL = D / 32;
    float x[DPL];
    if constexpr (DPL == 4) {
        const uint2 w = *reinterpret_cast<const uint2 *>(src + lane * 4);
        x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x); x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
    } else {
        static_assert(DPL == 2, "head dim 64 or 128");
        const uint32_t w = *reinterpret_cast<const uint32_t *>(src + lane * 2);
        x[0] = bf16_lo(w); x[1] = bf16_hi(w);
    }
    float amax = 0.0f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) amax = fmaxf(amax, fabsf(x[e]));
#pragma unroll
    for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const int s = tier_exponent(amax);
    // 2^s with s in [-120, 127] (amax is at most the largest bf16) is a normal
    // float; x 2^s is exact unless it falls below 2^-126, far under the
    // smallest E4M3 subnormal (2^-9), where both round to 0
    const float scale = __int_as_float((127 + s) << 23);
    uint32_t packed = 0;
#pragma unroll
    for (int e = 0; e < DPL; ++e) {
        const uint32_t c = __nv_cvt_float_to_fp8(x[e] * scale, __NV_SATFINITE, __NV_E4M3);
        packed |= c << (8 * e);
    }
    if constexpr (DPL == 4) *reinterpret_cast<uint32_t *>(dst + lane * 4) = packed;
    else *reinterpret_cast<uint16_t *>(dst + lane * 2) = (uint16_t)packed;
    return (int8_t)s;
}

// The controller: grid (max_pages, B).  CTA (p, b) demotes logical page p of
// sequence b when its tokens [p page, (p + 1) page) all lie in [S, n - W),
// its physical page is still tier 0 and not protected.  A page-table entry
// outside [0, num_pages) sets the error word and is skipped.
template <int D>
__global__ void __launch_bounds__(kDemoteThreads)
demote_pages_kernel(KV kv, Tiers tr, const uint8_t *__restrict__ protect, const int32_t *__restrict__ seq_lens,
                    int S, int W) {
    const int p = blockIdx.x, b = blockIdx.y;
    const int64_t n = seq_lens[b];
    const int64_t lo = (int64_t)p * kv.page_size, hi = lo + kv.page_size;
    if (lo < S || hi > n - W) return;
    const int32_t phys = __ldg(kv.page_table + (int64_t)b * kv.max_pages + p);
    if (phys < 0) return;
    if (phys >= kv.num_pages) {
        if (threadIdx.x == 0) raise_error(kErrPage);
        return;
    }
    if (tr.tier[phys] != 0 || (protect && protect[phys])) return;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int rows = kv.page_size * kv.Hkv;  // (slot, head) rows of the page
    for (int r = warp; r < 2 * rows; r += kDemoteThreads / 32) {
        const int isv = r >= rows;
        const int64_t row = (int64_t)phys * rows + (isv ? r - rows : r);
        const __nv_bfloat16 *src = (isv ? kv.v : kv.k) + row * D;
        uint8_t *dst = (isv ? tr.v8 : tr.k8) + row * D;
        const int8_t s = quantize_row<D>(src, dst, lane);
        if (lane == 0) tr.exps[row * 2 + isv] = s;
    }
    __syncthreads();
    if (threadIdx.x == 0) tr.tier[phys] = 1;
}

}  // namespace dkv
