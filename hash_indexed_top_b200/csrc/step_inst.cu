// step_inst.cu -- the step kernel's instantiations for one (bits, head dim)
// pair, chosen with -DSTEP_BITS=... -DSTEP_D=... (the build compiles this file
// once per pair, in parallel, into relocatable device code).
#include "step.cuh"

#if !defined(STEP_BITS) || !defined(STEP_D)
#error "compile with -DSTEP_BITS=<32|64|128> -DSTEP_D=<64|128>"
#endif

#define DKV_CAT_(a, b, c) a##b##_##c
#define DKV_CAT(a, b, c) DKV_CAT_(a, b, c)

namespace dkv {

StepKern DKV_CAT(step_kern_, STEP_BITS, STEP_D)(int G, bool paged, bool radius) {
    constexpr int B = STEP_BITS, D = STEP_D;
    if (radius) return paged ? step_kernel<B, D, 0, true, true> : step_kernel<B, D, 0, false, true>;
    switch (G) {
        case 1: return paged ? step_kernel<B, D, 1, true, false> : step_kernel<B, D, 1, false, false>;
        case 2: return paged ? step_kernel<B, D, 2, true, false> : step_kernel<B, D, 2, false, false>;
        case 4: return paged ? step_kernel<B, D, 4, true, false> : step_kernel<B, D, 4, false, false>;
        case 8: return paged ? step_kernel<B, D, 8, true, false> : step_kernel<B, D, 8, false, false>;
        default: return paged ? step_kernel<B, D, 0, true, false> : step_kernel<B, D, 0, false, false>;
    }
}

}  // namespace dkv
