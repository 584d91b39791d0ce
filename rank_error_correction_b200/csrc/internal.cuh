// internal.cuh -- declarations shared by the translation units of libglowq.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "glowq.h"

namespace glowq {

// Host-side view of one module of a group (validated by api.cu).
struct ModuleView {
    const uint32_t* q;   // packed 4-bit codes [O][d/8]
    const void* s;       // INT4: fp16 scales [O][d/128]; MXFP4 / NVFP4: scale bytes
    const uint8_t* z;    // INT4 zeros (nullptr for FP4)
    const float* ts;     // NVFP4 tensor scale (device), else nullptr
    const uint16_t* A;   // nullptr: correction off for this module
    uint16_t* Y;
    int64_t ldY;
    int64_t O;
};

constexpr int kDecodeMaxTokens = 16;
// Tokens up to which the tcgen05 path uses 64-token pair tiles and may split k.
constexpr int kSmallBatchMaxTokens = 64;

// Workspace layout: [zero region][R partials][solo R][k-split slots].  The
// zero region holds the decode hand-off flags (bytes 0..255) and the k-split
// tickets (bytes 256..4095, one u32 per CTA of a split tile); it must be zero
// before a call and every call that completes leaves it zero.
constexpr size_t kWorkspaceZeroBytes = 4096;
constexpr size_t kTicketOffsetBytes = 256;
constexpr int kMaxTickets = (int)((kWorkspaceZeroBytes - kTicketOffsetBytes) / 4);
constexpr int kMaxSplit = 8;          // parts per tile
constexpr int kMinSplitBlocks = 8;    // k-blocks (of 64) per part, at least
// Costs of the small-batch work decomposition in k-blocks of streamed weights
// (fitted to a sweep of S = 1..8 over the LLaMA-2-7B / LLaMA-3.1-8B /
// LLaMA-2-13B units at T = 32 and 64 on B200, ~0.37 us per k-block): a work
// unit's fixed cost (ring fill, accumulator drain, stores), and a split tile's
// partial-sum traffic and reduction, a base plus a share per part.
constexpr int kUnitCost = 15;
constexpr int kSplitBaseCost = 6;
constexpr int kSplitPartCost = 3;

// Argument checks of glowq_solo_forward, without the workspace (api.cu).
glowq_status validate_solo_call(const glowq_module* mod, int64_t d, const uint16_t* B, int32_t r, const uint16_t* X,
                                int64_t T);

// Device address of this device's status word (bounded-wait timeouts).
unsigned int* device_status_ptr();

// decode.cu
// Corrected GEMV over the stacked rows (T <= 16), one launch.  With r > 0 it
// also computes R = X B^T (written to R) from fp32 partial sums in `partial`
// (decode_partial_bytes(T, r)); `flags` are the first 256 bytes of the
// workspace's zero region, which every completed call leaves zero.
cudaError_t launch_gemv_decode(const ModuleView* mods, int m, int d, int T, int r, const uint16_t* X,
                               const uint16_t* B, uint16_t* R, unsigned int* flags, float* partial, int num_sms,
                               cudaStream_t st, int fmt = GLOWQ_FMT_INT4, const float* tok_scale = nullptr);
size_t decode_partial_bytes(int64_t T, int r);
// pack.cu
cudaError_t launch_pack_int4(const float* W, int64_t O, int64_t d, uint32_t* q, uint16_t* s, uint8_t* z,
                             cudaStream_t st);
cudaError_t launch_dequant_int4(const uint32_t* q, const uint16_t* s, const uint8_t* z, int64_t O, int64_t d,
                                uint16_t* out, cudaStream_t st);
cudaError_t launch_error_norms(const float* W, const uint32_t* q, const uint16_t* s, const uint8_t* z,
                               int64_t O, int64_t d, double* out_rows, cudaStream_t st);
// fp4.cu
cudaError_t launch_quantize_act_e4m3(const uint16_t* X, int64_t T, int64_t d, uint8_t* codes, float* scales,
                                     uint16_t* Xq, cudaStream_t st);
cudaError_t launch_pack_fp4(int fmt, const float* W, int64_t O, int64_t d, uint32_t* codes, uint8_t* scales,
                            float* tensor_scale, cudaStream_t st);
cudaError_t launch_dequant_fp4(int fmt, const uint32_t* codes, const uint8_t* scales, const float* tensor_scale,
                               int64_t O, int64_t d, uint16_t* out, cudaStream_t st);
// solve.cu: the offline group solve (float64)
struct SolveModule {
    const float* W;      // O x d fp32 weights
    const uint32_t* q;   // INT4 packed codes
    const uint16_t* s;   // fp16 scales
    const uint8_t* z;    // zeros
    int64_t O;
};
size_t solve_workspace_bytes(int64_t M, int64_t d, int l);
glowq_status group_solve_impl(const SolveModule* mods, int m, int64_t d, const double* Sh, const double* Shp,
                              int r, int p, int qit, const double* Omega, double* A, double* B, double* sing,
                              double* gec, uint16_t* A16, uint16_t* B16, void* workspace, unsigned int* err,
                              cudaStream_t st);
// prefill.cu: TMA tensor maps (driver entry point resolved at run time)
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn();
// 2-D row-major tensor [outer][inner], row pitch `pitch` bytes, box {box_inner, box_outer}.
bool make_map(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
              uint64_t pitch, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw);
// `partial`: scratch of prefill_partial_bytes(T, r) for the split R projection
// (nullptr: one slice of d per CTA, R written directly).
// `tickets` (zeroed workspace words) and `slots` (max_slots fp32 partial
// tiles of prefill_slot_bytes) enable the k-split; nullptr / 0: whole tiles.
glowq_status prefill_group_forward(const ModuleView* mods, int m, int d, const uint16_t* B, int r,
                                   const uint16_t* X, int64_t T, uint16_t* R, float* partial, int num_sms,
                                   cudaStream_t st, int fmt = GLOWQ_FMT_INT4, const float* tok_scale = nullptr,
                                   uint16_t* R_scaled = nullptr, unsigned int* tickets = nullptr,
                                   float* slots = nullptr, int64_t max_slots = 0);
size_t prefill_partial_bytes(int64_t T, int r);
// Work decomposition of the tcgen05 GEMM: token width bn of the pair tiles,
// tiles [0, split_from) whole, the rest split into S parts of kbs k-blocks;
// slots = fp32 partial tiles the split needs.
struct SplitPlan {
    int bn;
    int64_t ntiles_n, ntiles, split_from;
    int S, kbs;
    int64_t slots;
};
SplitPlan plan_prefill_split(int64_t T, int d, int64_t mtiles, int pairs, int64_t max_slots);
int gemm_max_pairs(int num_sms);
int prefill_tile_n(int64_t T);
size_t prefill_slot_bytes(int bn);

}  // namespace glowq
