// common.cuh -- layout addressing, hyperplane bits and the device error word
// shared by the kernels of libdashkv (one translation unit: dashkv.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dkv {

constexpr int kMaxBits = 128;
constexpr int kMaxDim = 128;
constexpr int kSmCountFallback = 148;
// One 128-byte line per (b, h) for every workspace word that CTAs update
// atomically, so that different (b, h) never serialise on one L2 line.
constexpr int kSyncStride = 32;

// Device error word (one per device that loads the library).  Bits:
// kErrTimeout: a bounded wait on a shared-memory barrier gave up (a bulk copy
// did not complete in time); the affected results are not valid.
enum : unsigned { kErrCapacity = 1u, kErrPage = 2u, kErrTimeout = 4u };
// Defined once, in dashkv.cu (the library is built with relocatable device code).
extern __device__ unsigned g_error_word;

__device__ __forceinline__ void raise_error(unsigned bit) { atomicOr(&g_error_word, bit); }

// Thread-block cluster barrier (every thread of every CTA of the cluster
// arrives; release / acquire order their memory accesses at cluster scope).
__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_sync() {
    cluster_arrive();
    cluster_wait();
}

// Address, in the cluster's shared window, of the object at `p` (this CTA's
// shared memory) in the CTA of cluster rank `rank`.
__device__ __forceinline__ uint32_t cluster_addr(const void *p, uint32_t rank) {
    const uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    return r;
}
__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
// Packed fp32 fused multiply-add (two lanes of fp32 per instruction on sm_100):
// (a.x * b.x + c.x, a.y * b.y + c.y), each rounded once like fmaf.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
// Hint: bring `bytes` (a multiple of 16, 16-byte aligned) at p into L2.
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
// L2 cache policy for data read once (evicted first).
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ uint4 ld_cluster_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

// ---- shared-memory barriers and bulk copies (global -> this CTA's shared
// memory only, completion counted in bytes on an mbarrier).
__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mbar), "r"(count) : "memory");
}
// Make barrier initialisation visible to the async proxy (bulk copies).
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t mbar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mbar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t mbar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(mbar) : "memory");
}
// Copy `bytes` (a multiple of 16; both addresses 16-byte aligned) from global
// memory into this CTA's shared memory; completion is signalled on `mbar`.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t mbar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(mbar)
                 : "memory");
}
// bulk_g2s with an L2 cache policy
__device__ __forceinline__ void bulk_g2s_hint(uint32_t dst, const void *src, uint32_t bytes, uint32_t mbar, uint64_t pol) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(mbar), "l"(pol)
                 : "memory");
}
// Bounded wait for the phase of parity `parity` of `mbar` to complete.  Each
// poll suspends the warp until the phase completes or kMbarSuspendNs pass (a
// suspended warp takes no issue slots from the warps that have work); after
// kMbarSpins polls (about a second at most) it gives up, sets the timeout bit
// of the error word and returns false.
constexpr int kMbarSpins = 1 << 12;
constexpr uint32_t kMbarSuspendNs = 250000;
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity) {
    for (int it = 0; it < kMbarSpins; ++it) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(mbar), "r"(parity), "r"(kMbarSuspendNs)
            : "memory");
        if (done) return true;
    }
    raise_error(kErrTimeout);
    return false;
}

// Hyperplanes as sign bits: bit (i % 32) of word [j * (d / 32) + i / 32] is set
// when R[j][i] = -1.  2 KB at bits = d = 128, passed by value as a kernel
// parameter (constant bank), so no device allocation is needed.
struct RBits {
    uint32_t w[kMaxBits * kMaxDim / 32];
};

// Cache addressing.  page_size == 0 selects the dense layout.
struct KV {
    __nv_bfloat16 *k;
    __nv_bfloat16 *v;
    uint64_t *codes;
    int64_t n_cap;             // dense rows per (b, h)
    const int32_t *page_table; // [B][max_pages]
    int32_t max_pages;
    int32_t num_pages;
    int32_t page_size;         // 0 = dense
    int32_t Hkv;
    int32_t d;
    int32_t W;                 // 64-bit code words per key
    int32_t len_shift;         // entries per sequence = seq_lens[b] >> len_shift (block summaries: log2 m)
    const uint8_t *radius;     // optional 8-bit key-norm codes (layout of radius_index), or null

    __host__ __device__ int64_t capacity() const {
        return page_size ? (int64_t)max_pages * page_size : n_cap;
    }
    // Physical page of token t of sequence b, or -1 (error word set) when the
    // page table entry is out of range.
    __device__ __forceinline__ int64_t page_of(int b, int64_t t) const {
        int32_t p = __ldg(page_table + (int64_t)b * max_pages + t / page_size);
        if (p < 0 || p >= num_pages) {
            raise_error(kErrPage);
            return -1;
        }
        return p;
    }
    // Element offset of row (b, h, t) in k / v, or -1.
    __device__ __forceinline__ int64_t row(int b, int h, int64_t t) const {
        if (!page_size) return (((int64_t)b * Hkv + h) * n_cap + t) * d;
        int64_t p = page_of(b, t);
        if (p < 0) return -1;
        return ((p * page_size + t % page_size) * Hkv + h) * (int64_t)d;
    }
    // Byte offset of the radius code of (b, h, t) -- dense [B][Hkv][n_cap], paged
    // [P][Hkv][page] (the codes' layout without the word axis) -- or -1.
    __device__ __forceinline__ int64_t radius_index(int b, int h, int64_t t) const {
        if (!page_size) return ((int64_t)b * Hkv + h) * n_cap + t;
        int64_t p = page_of(b, t);
        if (p < 0) return -1;
        return (p * Hkv + h) * page_size + t % page_size;
    }
    // Word offset of the code of (b, h, t), or -1.
    __device__ __forceinline__ int64_t code(int b, int h, int64_t t) const {
        if (!page_size) return (((int64_t)b * Hkv + h) * n_cap + t) * W;
        int64_t p = page_of(b, t);
        if (p < 0) return -1;
        return ((p * Hkv + h) * page_size + t % page_size) * (int64_t)W;
    }
};

// Entries of sequence b (tokens, or complete blocks of a block-summary view)
// clamped to the capacity (error word set when they exceed it).
__device__ __forceinline__ int64_t clamp_len(const KV &kv, const int32_t *seq_lens, int b) {
    int64_t n = __ldg(seq_lens + b) >> kv.len_shift;
    int64_t cap = kv.capacity();
    if (n > cap) {
        raise_error(kErrCapacity);
        n = cap;
    }
    return n < 0 ? 0 : n;
}

// Programmatic dependent launch.  wait(): block until the preceding kernel of
// the stream has completed and its writes are visible (a no-op when this kernel
// was launched without the programmatic-serialization attribute).  trigger():
// allow the following kernel to be scheduled early (it still waits in wait()).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_trigger() { asm volatile("griddepcontrol.launch_dependents;" :::); }

__device__ __forceinline__ float bf16_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t x) { return __uint_as_float(x & 0xFFFF0000u); }

// Order-preserving map from fp32 to uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t float_key(float f) {
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Rotate the token's code bytes by rho (byte r of the result = byte (r + rho)
// mod 4*NW of the input).
// Branch-free: word rotation by rho / 4 as two select stages, then a funnel
// shift by 8 (rho % 4) bits across neighbouring words.
template <int NW>
__device__ __forceinline__ void rotate_bytes(uint32_t (&w)[NW], bool by8, bool by4, uint32_t sh) {
    uint32_t a[NW], c[NW];
#pragma unroll
    for (int k = 0; k < NW; ++k) a[k] = (NW == 4 && by8) ? w[(k + 2) % NW] : w[k];
#pragma unroll
    for (int k = 0; k < NW; ++k) c[k] = (NW >= 2 && by4) ? a[(k + 1) % NW] : a[k];
#pragma unroll
    for (int k = 0; k < NW; ++k) w[k] = __funnelshift_r(c[k], c[(k + 1) % NW], sh);
}

// Code storage.  Token t's code (b bits = T = b/8 bytes, LSB-first, hyperplane j
// in byte j/8 bit j%8) is stored with its bytes rotated by t mod T: stored byte
// p holds code byte (p + t mod T) mod T.  The scorer's lane that handles token t
// reads its bytes in exactly that order, so the swizzle replaces a per-token
// register rotation.  w: the code as BITS/32 little-endian 32-bit words;
// rotate_code() turns them into the stored order in registers.
template <int BITS>
__device__ __forceinline__ void rotate_code(uint32_t (&w)[BITS / 32], int64_t t) {
    constexpr int NW = BITS / 32;
    const int rho = (int)(t % (BITS / 8));
    rotate_bytes<NW>(w, (rho & 8) != 0, (rho & 4) != 0, 8u * (uint32_t)(rho & 3));
}
template <int BITS>
__device__ __forceinline__ void store_code_rotated(uint64_t *dst, const uint32_t (&w)[BITS / 32], int64_t t) {
    constexpr int NW = BITS / 32;
    uint32_t r[NW];
#pragma unroll
    for (int k = 0; k < NW; ++k) r[k] = w[k];
    rotate_code<BITS>(r, t);
    if constexpr (NW == 1) {
        dst[0] = (uint64_t)r[0];
    } else {
#pragma unroll
        for (int k = 0; k < NW / 2; ++k) dst[k] = (uint64_t)r[2 * k] | ((uint64_t)r[2 * k + 1] << 32);
    }
}

__host__ __device__ __forceinline__ int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace dkv
