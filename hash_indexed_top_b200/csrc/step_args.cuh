// step_args.cuh -- shapes, shared-memory layout and launch arguments of the
// clustered step kernel (step.cuh), shared with the host code that launches it.
#pragma once
#include "common.cuh"
#include "select.cuh"

namespace dkv {

// 16 warps per CTA.  While the code stream runs, warps 0..14 consume it and
// warp 15 is its producer (it refills the ring); every other part of the step
// uses all 16 warps.
constexpr int kStepWarps = 16;
constexpr int kStepThreads = kStepWarps * 32;
constexpr int kStreamWarps = kStepWarps - 1;
constexpr int kRingStages = 5;

// The code stream runs in CTA-wide stages of STG_TOK consecutive tokens
// (15 KB of codes): consumer warp w takes the 32 TPL tokens [32 TPL w, 32 TPL (w + 1))
// of every stage, lane l those congruent to l mod 32 (TPL of them, so the
// per-stage bookkeeping of a warp is shared by several tokens per lane).
template <int BITS>
struct StepShape {
    static constexpr int CODE_B = BITS >= 64 ? BITS / 8 : 8;  // bytes of one token's code in memory
    static constexpr int TPL = BITS == 128 ? 2 : 4;            // tokens per lane per stage
    static constexpr int STG_TOK = kStreamWarps * 32 * TPL;    // tokens per stage
    static constexpr int STG_B = STG_TOK * CODE_B;             // bytes per stage (15 KB)
    static constexpr int RING_B = kRingStages * STG_B;
};

// The threshold estimate samples tokens into a histogram of kSampleBins bins
// (bin b of the selection histogram falls in sample bin b / kSampleDiv).
constexpr int kSampleDiv = 4;
constexpr int kSampleBins = kBins / kSampleDiv;
constexpr int kSampleStrata = 64;  // sampled 32-token blocks (at most)

// The attention's cluster merge: CTA c receives, for the elements x = g D + i
// with x mod C = c, every CTA's partial sum (slot [cta][x / C]) and every
// CTA's per-head (max, sum) pair, in a region just below the LUT that nothing
// else uses.
constexpr int kMaxG = 8;
constexpr int kRecvAccFloats = kMaxG * kMaxDim + kMaxCluster;
constexpr int kRecvBytes = (kRecvAccFloats + kMaxCluster * kMaxG * 2) * 4;

// Fixed part of the low shared region (byte offsets from the dynamic base).
struct StepLow {
    static constexpr int HIST = 0;                                 // u32[kBins]
    static constexpr int SUP = HIST + kBins * 4;                   // u32[64] super-bin counts
    static constexpr int SHIST = SUP + 64 * 4;                     // u32[kSampleBins] sample histogram
    static constexpr int SSUP = SHIST + kSampleBins * 4;           // u32[64] its super-bin counts
    static constexpr int QSUM = SSUP + 64 * 4;                     // f32[kMaxDim]
    static constexpr int QP = QSUM + kMaxDim * 4;                  // f32[kMaxBits]
    static constexpr int KNEW = QP + kMaxBits * 4;                 // f32[kMaxDim] appended key
    static constexpr int MISC = KNEW + kMaxDim * 4;                // int[64]
    static constexpr int NEWC = MISC + 64 * 4;                     // u32[4] appended key's code
    static constexpr int NEWR = NEWC + 16;                         // u32[4] the same in stored (rotated) order
    static constexpr int MBAR = NEWR + 16;                         // u64[kRingStages] full barriers of the ring
    static constexpr int MBAR_EMPTY = MBAR + kRingStages * 8;      // u64[kRingStages] slots released by every consumer
    static constexpr int WDEF = MBAR_EMPTY + kRingStages * 8;      // int[kStepWarps] definite tokens per warp
    static constexpr int CNT = WDEF + kStepWarps * 4;              // int[kMaxCluster][2]
    static constexpr int MID = CNT + kMaxCluster * 8;              // int[kMaxCluster]
    static constexpr int WARPSCAN = MID + kMaxCluster * 4;         // int[32] block-scan scratch
    static constexpr int END = (WARPSCAN + 128 + 255) / 256 * 256; // candidate lists start here
};
static_assert(StepLow::MBAR % 8 == 0 && StepLow::MBAR_EMPTY % 8 == 0, "mbarriers are 8-byte aligned");

// misc[] slots
enum : int {
    kMTloc = 0, kMIns = 1, kMNinb = 2, kMOvf = 3, kMT1 = 4, kMAbove = 5, kMCntT1 = 6,
    kMTkey = 8, kMIT = 9, kMBefore = 10, kMTotal = 11, kMAnyOvf = 12, kMKept = 13,
    kMSamp = 14, kMTmax = 15
};

struct StepArgs {
    KV kv;
    const __nv_bfloat16 *q;
    int Hq, G;
    int32_t *seq_lens;                   // read; incremented when appending
    const __nv_bfloat16 *k_new, *v_new;  // [B][Hkv][D] (null: no append)
    SelWS ws;                            // scores / cand / seg_cnt rows for the slow path
    int topk, S, W, cap_sel;
    int32_t *sel_idx, *sel_cnt;
    float *scores_out;                   // optional [B][Hkv][ld_out]
    int64_t ld_out;
    float *out, *lse;                    // attention outputs (G > 0)
    float scale_log2;                    // log2(e) / sqrt(d)
    uint32_t *seq_arrive;                // [B] x kSyncStride: clusters of a sequence done with its length
    int smem_bytes;                      // dynamic shared memory of the launch
};

using StepKern = void (*)(const StepArgs, const RBits);

// The step kernel for (bits, head dim, G, paged, radius); G = 0: selection
// only, G > 0: append + selection + attention for G query heads per kv head.
// One getter per (bits, head dim), each defined in its own translation unit
// (step_inst.cu compiled once per pair).
#define DKV_STEP_GETTER(BITS, D) StepKern step_kern_##BITS##_##D(int G, bool paged, bool radius);
DKV_STEP_GETTER(32, 64)
DKV_STEP_GETTER(32, 128)
DKV_STEP_GETTER(64, 64)
DKV_STEP_GETTER(64, 128)
DKV_STEP_GETTER(128, 64)
DKV_STEP_GETTER(128, 128)
#undef DKV_STEP_GETTER

}  // namespace dkv
