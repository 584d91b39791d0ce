// api.cu -- the extern "C" boundary of libglowq: argument validation, path
// dispatch (decode kernels for T <= 16, tcgen05 kernels above) and launches.
// Argument meaning, layouts and error behaviour are documented in glowq.h.
#include <cstdint>
#include <cstdio>
#include <cstring>

#include "common.cuh"
#include "internal.cuh"

namespace glowq {

__device__ unsigned int g_device_status = 0;

// Failure-path self-test: one thread waits, bounded, on a barrier that never
// completes (its only expected arrival never comes).
__global__ void selftest_wait_kernel(uint32_t polls, unsigned int* status) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        mbar_wait(&bar, 0, status, polls);
    }
}

unsigned int* device_status_ptr() {
    static unsigned int* cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return nullptr;
    if (dev < 64 && cached[dev]) return cached[dev];
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    if (dev < 64) cached[dev] = static_cast<unsigned int*>(p);
    return static_cast<unsigned int*>(p);
}


static inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int device_sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace layout: [zero region, 4 KB][R partials][solo R][k-split slots].
// The zero region holds the decode GEMV's hand-off flags (producers of R ->
// consumers) and the tcgen05 GEMM's k-split tickets; it sits at offset 0 for
// every T, so no other call sharing the workspace overwrites it.
static size_t workspace_flag_bytes(int32_t r) { return r > 0 ? kWorkspaceZeroBytes : 0; }

// fp32 partial sums of R = X B^T split along d: up to 16 slices for T <= 16
// (decode), up to 8 when the prefill token tiles alone would not fill the GPU.
static size_t workspace_partial_bytes(int64_t T, int32_t r) {
    if (r <= 0 || T <= 0) return 0;
    return align_up(T <= kDecodeMaxTokens ? decode_partial_bytes(T, r) : prefill_partial_bytes(T, r), 256);
}

static size_t workspace_solo_R_bytes(int64_t T, int32_t r) {
    if (r <= 0 || T <= 0) return 0;
    return align_up((size_t)T * (size_t)r * 2, 256);
}

// Shared validation for the forward calls.
static glowq_status validate_forward(const glowq_module* mods, int32_t m, int64_t d, const uint16_t* B, int32_t r,
                                     const uint16_t* X, int64_t T) {
    if (!mods || m < 1 || m > GLOWQ_MAX_MODULES || d <= 0 || T < 0 || r < 0) return GLOWQ_ERR_ARG;
    if (d % GLOWQ_GROUP_SIZE != 0 || d > (int64_t)1 << 20) return GLOWQ_ERR_SHAPE;
    if (r > GLOWQ_MAX_RANK || r % 8 != 0) return GLOWQ_ERR_SHAPE;
    if (r > 0 && !B) return GLOWQ_ERR_ARG;
    if (T > 0 && !X) return GLOWQ_ERR_ARG;
    if ((B && !aligned16(B)) || (X && !aligned16(X))) return GLOWQ_ERR_ALIGN;
    int64_t rows = 0;
    for (int i = 0; i < m; ++i) {
        const glowq_module& md = mods[i];
        if (!md.qweight || !md.scales || !md.zeros || !md.Y) return GLOWQ_ERR_ARG;
        if (md.out_features <= 0 || md.out_features % 16 != 0) return GLOWQ_ERR_SHAPE;
        if (md.ldY < md.out_features || md.ldY % 8 != 0) return GLOWQ_ERR_ALIGN;
        if (!aligned16(md.qweight) || !aligned16(md.Y) || (md.A && !aligned16(md.A))) return GLOWQ_ERR_ALIGN;
        if ((reinterpret_cast<uintptr_t>(md.scales) & 1u) != 0) return GLOWQ_ERR_ALIGN;
        rows += md.out_features;
    }
    if (rows > ((int64_t)1 << 30) || T > ((int64_t)1 << 30)) return GLOWQ_ERR_SHAPE;
    return GLOWQ_OK;
}

// Host-side validation of a solo call (exported to the other translation units).
glowq_status validate_solo_call(const glowq_module* mod, int64_t d, const uint16_t* B, int32_t r, const uint16_t* X,
                                int64_t T) {
    return validate_forward(mod, 1, d, B, r, X, T);
}

// R: the projection the kernels write and read; W4A8 (tok_scale != nullptr):
// the decode kernels write R = fp16(s_t X' B^T) there, the prefill kernels
// write the unscaled fp16(X' B^T) there for the GEMM and fp16(s_t X' B^T) to
// R_scaled (when not null).
// Offset of the k-split slots: behind everything else the call may use.
static size_t split_base_bytes(int64_t T, int32_t r) {
    return kWorkspaceZeroBytes + workspace_partial_bytes(T, r) + workspace_solo_R_bytes(T, r);
}

// split_bytes: the workspace's size when the bytes behind split_base_bytes(T, r)
// may hold k-split slots (0: no split).
static glowq_status forward_views(const ModuleView* hm, int32_t m, int64_t d, const uint16_t* B, int32_t r,
                                  const uint16_t* X, int64_t T, uint16_t* R, void* workspace, size_t split_bytes,
                                  cudaStream_t st, int fmt, const float* tok_scale = nullptr,
                                  uint16_t* R_scaled = nullptr) {
    if (T == 0) return GLOWQ_OK;
    const bool use_r = r > 0;
    float* partial = (use_r && workspace_partial_bytes(T, r) > 0)
                         ? reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) + workspace_flag_bytes(r))
                         : nullptr;
    if (T <= kDecodeMaxTokens) {
        unsigned int* flags = use_r ? reinterpret_cast<unsigned int*>(workspace) : nullptr;
        cudaError_t e = launch_gemv_decode(hm, m, (int)d, (int)T, use_r ? r : 0, X, use_r ? B : nullptr, R, flags,
                                           partial, device_sm_count(), st, fmt, tok_scale);
        return e == cudaSuccess ? GLOWQ_OK : GLOWQ_ERR_CUDA;
    }
    unsigned int* tickets = nullptr;
    float* slots = nullptr;
    int64_t max_slots = 0;
    const size_t base = split_base_bytes(T, r);
    if (workspace && split_bytes > base) {
        tickets = reinterpret_cast<unsigned int*>(static_cast<char*>(workspace) + kTicketOffsetBytes);
        slots = reinterpret_cast<float*>(static_cast<char*>(workspace) + base);
        max_slots = (int64_t)((split_bytes - base) / prefill_slot_bytes(prefill_tile_n(T)));
    }
    return prefill_group_forward(hm, m, (int)d, use_r ? B : nullptr, use_r ? r : 0, X, T, R, partial,
                                 device_sm_count(), st, fmt, tok_scale, use_r ? R_scaled : nullptr, tickets, slots,
                                 max_slots);
}

static glowq_status forward_impl(const glowq_module* mods, int32_t m, int64_t d, const uint16_t* B, int32_t r,
                                 const uint16_t* X, int64_t T, uint16_t* R, void* workspace, size_t ws_bytes,
                                 cudaStream_t st) {
    ModuleView hm[GLOWQ_MAX_MODULES];
    for (int i = 0; i < m; ++i)
        hm[i] = {mods[i].qweight, mods[i].scales, mods[i].zeros, nullptr, (r > 0) ? mods[i].A : nullptr,
                 mods[i].Y, mods[i].ldY, mods[i].out_features};
    return forward_views(hm, m, d, B, r, X, T, R, workspace, ws_bytes, st, GLOWQ_FMT_INT4);
}

// Validation of MXFP4 / NVFP4 modules and their conversion to module views.
static glowq_status fp4_views(glowq_format fmt, const glowq_fp4_module* mods, int32_t m, int64_t d,
                              const uint16_t* B, int32_t r, const uint16_t* X, int64_t T, ModuleView* hm) {
    if (fmt != GLOWQ_FMT_MXFP4 && fmt != GLOWQ_FMT_NVFP4) return GLOWQ_ERR_ARG;
    if (!mods || m < 1 || m > GLOWQ_MAX_MODULES) return GLOWQ_ERR_ARG;
    glowq_module tmp[GLOWQ_MAX_MODULES];
    for (int i = 0; i < m; ++i) {
        const glowq_fp4_module& f = mods[i];
        if (!f.scales || (fmt == GLOWQ_FMT_NVFP4 && !f.tensor_scale)) return GLOWQ_ERR_ARG;
        const uintptr_t sa = reinterpret_cast<uintptr_t>(f.scales);
        if ((fmt == GLOWQ_FMT_MXFP4 && (sa & 3u)) || (fmt == GLOWQ_FMT_NVFP4 && (sa & 7u)) ||
            (f.tensor_scale && (reinterpret_cast<uintptr_t>(f.tensor_scale) & 3u)))
            return GLOWQ_ERR_ALIGN;
        // the shared checks of the INT4 path (zeros are not used: any non-null value)
        tmp[i] = {f.codes, reinterpret_cast<const uint16_t*>(f.scales), f.scales, f.A, f.out_features, f.Y, f.ldY};
    }
    glowq_status v = validate_forward(tmp, m, d, B, r, X, T);
    if (v != GLOWQ_OK) return v;
    for (int i = 0; i < m; ++i)
        hm[i] = {mods[i].codes, mods[i].scales, nullptr, fmt == GLOWQ_FMT_NVFP4 ? mods[i].tensor_scale : nullptr,
                 (r > 0) ? mods[i].A : nullptr, mods[i].Y, mods[i].ldY, mods[i].out_features};
    return GLOWQ_OK;
}

}  // namespace glowq

using namespace glowq;

extern "C" {

const char* glowq_version(void) { return "0.1.0"; }

const char* glowq_status_string(glowq_status s) {
    switch (s) {
        case GLOWQ_OK: return "ok";
        case GLOWQ_ERR_ARG: return "invalid argument (null pointer or negative size)";
        case GLOWQ_ERR_SHAPE: return "unsupported shape (d % 128, out_features % 16, r % 8, r <= 256)";
        case GLOWQ_ERR_ALIGN: return "misaligned pointer or leading dimension";
        case GLOWQ_ERR_CUDA: return "CUDA error while enqueueing work";
        case GLOWQ_ERR_TIMEOUT: return "a device-side bounded wait ran out";
        case GLOWQ_ERR_UNSUPPORTED: return "request outside this build's scope";
        case GLOWQ_ERR_NUMERIC: return "a factorisation met a non-positive pivot";
    }
    return "unknown status";
}

glowq_status glowq_pack_int4(const float* W, int64_t O, int64_t d, int32_t group_size, uint32_t* qweight,
                             uint16_t* scales, uint8_t* zeros, void* stream) {
    if (O < 0 || d < 0) return GLOWQ_ERR_ARG;
    if (group_size != GLOWQ_GROUP_SIZE) return GLOWQ_ERR_UNSUPPORTED;
    if (d % GLOWQ_GROUP_SIZE != 0 || O % 16 != 0) return GLOWQ_ERR_SHAPE;   // 16-row blocks
    if (O == 0 || d == 0) return GLOWQ_OK;
    if (!W || !qweight || !scales || !zeros) return GLOWQ_ERR_ARG;
    if (!aligned16(W) || (reinterpret_cast<uintptr_t>(qweight) & 3u) || (reinterpret_cast<uintptr_t>(scales) & 1u))
        return GLOWQ_ERR_ALIGN;
    return launch_pack_int4(W, O, d, qweight, scales, zeros, (cudaStream_t)stream) == cudaSuccess ? GLOWQ_OK
                                                                                                : GLOWQ_ERR_CUDA;
}

glowq_status glowq_dequant_int4(const uint32_t* qweight, const uint16_t* scales, const uint8_t* zeros, int64_t O,
                                int64_t d, int32_t group_size, uint16_t* W_deq, void* stream) {
    if (O < 0 || d < 0) return GLOWQ_ERR_ARG;
    if (group_size != GLOWQ_GROUP_SIZE) return GLOWQ_ERR_UNSUPPORTED;
    if (d % GLOWQ_GROUP_SIZE != 0 || O % 16 != 0) return GLOWQ_ERR_SHAPE;
    if (O == 0 || d == 0) return GLOWQ_OK;
    if (!qweight || !scales || !zeros || !W_deq) return GLOWQ_ERR_ARG;
    if (!aligned16(W_deq) || (reinterpret_cast<uintptr_t>(qweight) & 3u) || (reinterpret_cast<uintptr_t>(scales) & 1u))
        return GLOWQ_ERR_ALIGN;
    return launch_dequant_int4(qweight, scales, zeros, O, d, W_deq, (cudaStream_t)stream) == cudaSuccess
               ? GLOWQ_OK
               : GLOWQ_ERR_CUDA;
}

glowq_status glowq_error_norms(const float* W, const uint32_t* qweight, const uint16_t* scales,
                               const uint8_t* zeros, int64_t O, int64_t d, double* row_norms, void* stream) {
    if (O < 0 || d < 0) return GLOWQ_ERR_ARG;
    if (d % GLOWQ_GROUP_SIZE != 0 || O % 16 != 0) return GLOWQ_ERR_SHAPE;
    if (O == 0 || d == 0) return GLOWQ_OK;
    if (!W || !qweight || !scales || !zeros || !row_norms) return GLOWQ_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(row_norms) & 7u) || (reinterpret_cast<uintptr_t>(scales) & 1u) ||
        (reinterpret_cast<uintptr_t>(qweight) & 3u) || (reinterpret_cast<uintptr_t>(W) & 3u))
        return GLOWQ_ERR_ALIGN;
    return launch_error_norms(W, qweight, scales, zeros, O, d, row_norms, (cudaStream_t)stream) == cudaSuccess
               ? GLOWQ_OK
               : GLOWQ_ERR_CUDA;
}

glowq_status glowq_pack_fp4(glowq_format fmt, const float* W, int64_t O, int64_t d, uint32_t* codes,
                            uint8_t* scales, float* tensor_scale, void* stream) {
    if (O < 0 || d < 0) return GLOWQ_ERR_ARG;
    if (fmt != GLOWQ_FMT_MXFP4 && fmt != GLOWQ_FMT_NVFP4) return GLOWQ_ERR_ARG;
    if (d % GLOWQ_GROUP_SIZE != 0) return GLOWQ_ERR_SHAPE;
    if (O == 0 || d == 0) return GLOWQ_OK;
    if (!W || !codes || !scales || (fmt == GLOWQ_FMT_NVFP4 && !tensor_scale)) return GLOWQ_ERR_ARG;
    if (!aligned16(W) || (reinterpret_cast<uintptr_t>(codes) & 3u) ||
        (tensor_scale && (reinterpret_cast<uintptr_t>(tensor_scale) & 3u)))
        return GLOWQ_ERR_ALIGN;
    return launch_pack_fp4((int)fmt, W, O, d, codes, scales, tensor_scale, (cudaStream_t)stream) == cudaSuccess
               ? GLOWQ_OK
               : GLOWQ_ERR_CUDA;
}

glowq_status glowq_dequant_fp4(glowq_format fmt, const uint32_t* codes, const uint8_t* scales,
                               const float* tensor_scale, int64_t O, int64_t d, uint16_t* W_deq, void* stream) {
    if (O < 0 || d < 0) return GLOWQ_ERR_ARG;
    if (fmt != GLOWQ_FMT_MXFP4 && fmt != GLOWQ_FMT_NVFP4) return GLOWQ_ERR_ARG;
    if (d % GLOWQ_GROUP_SIZE != 0) return GLOWQ_ERR_SHAPE;
    if (O == 0 || d == 0) return GLOWQ_OK;
    if (!codes || !scales || !W_deq || (fmt == GLOWQ_FMT_NVFP4 && !tensor_scale)) return GLOWQ_ERR_ARG;
    if (!aligned16(W_deq) || (reinterpret_cast<uintptr_t>(codes) & 3u)) return GLOWQ_ERR_ALIGN;
    return launch_dequant_fp4((int)fmt, codes, scales, tensor_scale, O, d, W_deq, (cudaStream_t)stream) ==
                   cudaSuccess
               ? GLOWQ_OK
               : GLOWQ_ERR_CUDA;
}

size_t glowq_workspace_bytes(int64_t T, int32_t r) {
    if (T <= 0 || r <= 0) return 0;
    return workspace_flag_bytes(r) + workspace_partial_bytes(T, r) + workspace_solo_R_bytes(T, r);
}

size_t glowq_workspace_bytes_for(int64_t T, int32_t r, int64_t d, const int64_t* out_features, int32_t m) {
    const size_t need = (r >= 0) ? glowq_workspace_bytes(T, r) : 0;
    if (T <= kDecodeMaxTokens || T > ((int64_t)1 << 30) || r < 0 || d <= 0 || d % GLOWQ_GROUP_SIZE != 0 ||
        d > ((int64_t)1 << 20) || !out_features || m < 1 || m > GLOWQ_MAX_MODULES)
        return need;
    int64_t mtiles = 0;
    for (int i = 0; i < m; ++i) {
        if (out_features[i] <= 0 || out_features[i] > ((int64_t)1 << 30)) return need;
        mtiles += (out_features[i] + 255) / 256;
    }
    const SplitPlan p = plan_prefill_split(T, (int)d, mtiles, gemm_max_pairs(device_sm_count()), INT64_MAX);
    if (p.S <= 1) return need;
    return split_base_bytes(T, r) + (size_t)p.slots * prefill_slot_bytes(p.bn);
}

glowq_status glowq_group_forward(const glowq_module* mods, int32_t m, int64_t d, const uint16_t* B, int32_t r,
                                 const uint16_t* X, int64_t T, uint16_t* R_out, void* workspace,
                                 size_t workspace_bytes, void* stream) {
    glowq_status v = validate_forward(mods, m, d, B, r, X, T);
    if (v != GLOWQ_OK) return v;
    if (T == 0) return GLOWQ_OK;
    if (workspace && !aligned16(workspace)) return GLOWQ_ERR_ALIGN;
    if (r > 0) {
        if (!R_out) return GLOWQ_ERR_ARG;
        if (!aligned16(R_out)) return GLOWQ_ERR_ALIGN;
        const size_t need = workspace_flag_bytes(r) + workspace_partial_bytes(T, r);
        if (!workspace || workspace_bytes < need) return GLOWQ_ERR_ARG;
        if (!aligned16(workspace)) return GLOWQ_ERR_ALIGN;
    }
    return forward_impl(mods, m, d, B, r, X, T, R_out, workspace, workspace_bytes, (cudaStream_t)stream);
}

glowq_status glowq_solo_forward(const glowq_module* mod, int64_t d, const uint16_t* B, int32_t r, const uint16_t* X,
                                int64_t T, void* workspace, size_t workspace_bytes, void* stream) {
    glowq_status v = validate_forward(mod, 1, d, B, r, X, T);
    if (v != GLOWQ_OK) return v;
    if (T == 0) return GLOWQ_OK;
    if (workspace && !aligned16(workspace)) return GLOWQ_ERR_ALIGN;
    uint16_t* R = nullptr;
    if (r > 0) {
        const size_t need = glowq_workspace_bytes(T, r);
        if (!workspace || workspace_bytes < need) return GLOWQ_ERR_ARG;
        if (!aligned16(workspace)) return GLOWQ_ERR_ALIGN;
        R = reinterpret_cast<uint16_t*>(reinterpret_cast<char*>(workspace) + workspace_flag_bytes(r) +
                                        workspace_partial_bytes(T, r));
    }
    return forward_impl(mod, 1, d, B, r, X, T, R, workspace, workspace_bytes, (cudaStream_t)stream);
}

glowq_status glowq_group_forward_fp4(glowq_format fmt, const glowq_fp4_module* mods, int32_t m, int64_t d,
                                     const uint16_t* B, int32_t r, const uint16_t* X, int64_t T, uint16_t* R_out,
                                     void* workspace, size_t workspace_bytes, void* stream) {
    ModuleView hm[GLOWQ_MAX_MODULES];
    glowq_status v = fp4_views(fmt, mods, m, d, B, r, X, T, hm);
    if (v != GLOWQ_OK) return v;
    if (T == 0) return GLOWQ_OK;
    if (workspace && !aligned16(workspace)) return GLOWQ_ERR_ALIGN;
    if (r > 0) {
        if (!R_out) return GLOWQ_ERR_ARG;
        if (!aligned16(R_out)) return GLOWQ_ERR_ALIGN;
        const size_t need = workspace_flag_bytes(r) + workspace_partial_bytes(T, r);
        if (!workspace || workspace_bytes < need) return GLOWQ_ERR_ARG;
        if (!aligned16(workspace)) return GLOWQ_ERR_ALIGN;
    }
    return forward_views(hm, m, d, B, r, X, T, R_out, workspace, workspace_bytes, (cudaStream_t)stream, (int)fmt);
}

glowq_status glowq_solo_forward_fp4(glowq_format fmt, const glowq_fp4_module* mod, int64_t d, const uint16_t* B,
                                    int32_t r, const uint16_t* X, int64_t T, void* workspace, size_t workspace_bytes,
                                    void* stream) {
    ModuleView hm[1];
    glowq_status v = fp4_views(fmt, mod, 1, d, B, r, X, T, hm);
    if (v != GLOWQ_OK) return v;
    if (T == 0) return GLOWQ_OK;
    if (workspace && !aligned16(workspace)) return GLOWQ_ERR_ALIGN;
    uint16_t* R = nullptr;
    if (r > 0) {
        const size_t need = glowq_workspace_bytes(T, r);
        if (!workspace || workspace_bytes < need) return GLOWQ_ERR_ARG;
        if (!aligned16(workspace)) return GLOWQ_ERR_ALIGN;
        R = reinterpret_cast<uint16_t*>(reinterpret_cast<char*>(workspace) + workspace_flag_bytes(r) +
                                        workspace_partial_bytes(T, r));
    }
    return forward_views(hm, 1, d, B, r, X, T, R, workspace, workspace_bytes, (cudaStream_t)stream, (int)fmt);
}

size_t glowq_solve_workspace_bytes(int64_t rows, int64_t d, int32_t r, int32_t p) {
    if (rows <= 0 || d <= 0 || r <= 0 || p < 0) return 0;
    return solve_workspace_bytes(rows, d, r + p);
}

glowq_status glowq_group_solve(const glowq_solve_module* mods, int32_t m, int64_t d, const double* Sx_half,
                               const double* Sx_half_pinv, int32_t r, int32_t p, int32_t q, const double* Omega,
                               double* A, double* B, double* sing, double* g_ec, uint16_t* A16, uint16_t* B16,
                               void* workspace, size_t workspace_bytes, void* stream) {
    if (!mods || m < 1 || m > GLOWQ_MAX_MODULES || d <= 0 || r < 1 || p < 0 || q < 0 || q > 16) return GLOWQ_ERR_ARG;
    if (!Sx_half || !Sx_half_pinv || !Omega || !A || !B || !workspace) return GLOWQ_ERR_ARG;
    if (d % GLOWQ_GROUP_SIZE != 0 || r % 8 != 0 || p % 2 != 0 || r + p > 112) return GLOWQ_ERR_SHAPE;
    SolveModule sm[GLOWQ_MAX_MODULES];
    int64_t M = 0;
    for (int i = 0; i < m; ++i) {
        const glowq_solve_module& md = mods[i];
        if (!md.W || !md.qweight || !md.scales || !md.zeros || md.out_features <= 0) return GLOWQ_ERR_ARG;
        if (md.out_features % 16 != 0) return GLOWQ_ERR_SHAPE;   // 16-row code blocks
        if ((reinterpret_cast<uintptr_t>(md.qweight) & 3u) || (reinterpret_cast<uintptr_t>(md.scales) & 1u) ||
            (reinterpret_cast<uintptr_t>(md.W) & 3u))
            return GLOWQ_ERR_ALIGN;
        sm[i] = {md.W, md.qweight, md.scales, md.zeros, md.out_features};
        M += md.out_features;
    }
    if (r + p > M || r + p > d) return GLOWQ_ERR_SHAPE;
    const uintptr_t al8 = 7u;
    if ((reinterpret_cast<uintptr_t>(Sx_half) & al8) || (reinterpret_cast<uintptr_t>(Sx_half_pinv) & al8) ||
        (reinterpret_cast<uintptr_t>(Omega) & al8) || (reinterpret_cast<uintptr_t>(A) & al8) ||
        (reinterpret_cast<uintptr_t>(B) & al8) || (sing && (reinterpret_cast<uintptr_t>(sing) & al8)) ||
        (g_ec && (reinterpret_cast<uintptr_t>(g_ec) & al8)) || (A16 && (reinterpret_cast<uintptr_t>(A16) & 1u)) ||
        (B16 && (reinterpret_cast<uintptr_t>(B16) & 1u)) || !aligned16(workspace))
        return GLOWQ_ERR_ALIGN;
    if (workspace_bytes < solve_workspace_bytes(M, d, r + p)) return GLOWQ_ERR_ARG;
    return group_solve_impl(sm, m, d, Sx_half, Sx_half_pinv, r, p, q, Omega, A, B, sing, g_ec, A16, B16,
                            workspace, device_status_ptr(), (cudaStream_t)stream);
}

glowq_status glowq_quantize_act_e4m3(const uint16_t* X, int64_t T, int64_t d, uint8_t* codes, float* scales,
                                     uint16_t* X_q, void* stream) {
    if (T < 0 || d < 0) return GLOWQ_ERR_ARG;
    if (T == 0 || d == 0) return GLOWQ_OK;
    if (!X || !scales || !X_q) return GLOWQ_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(X) & 1u) || (reinterpret_cast<uintptr_t>(X_q) & 1u) ||
        (reinterpret_cast<uintptr_t>(scales) & 3u))
        return GLOWQ_ERR_ALIGN;
    return launch_quantize_act_e4m3(X, T, d, codes, scales, X_q, (cudaStream_t)stream) == cudaSuccess
               ? GLOWQ_OK
               : GLOWQ_ERR_CUDA;
}

// W4A8 workspace: [forward workspace][X' T x d fp16][s_t T floats][R' T x r fp16]
static size_t w4a8_xq_offset(int64_t T, int32_t r) { return align_up(glowq_workspace_bytes(T, r) + 16, 256); }
static size_t w4a8_scale_offset(int64_t T, int64_t d, int32_t r) {
    return w4a8_xq_offset(T, r) + align_up((size_t)T * d * 2, 256);
}
static size_t w4a8_rprime_offset(int64_t T, int64_t d, int32_t r) {
    return w4a8_scale_offset(T, d, r) + align_up((size_t)T * 4, 256);
}

size_t glowq_w4a8_workspace_bytes(int64_t T, int64_t d, int32_t r) {
    if (T <= 0 || d <= 0 || r < 0) return 0;
    return w4a8_rprime_offset(T, d, r) + align_up((size_t)T * (size_t)r * 2, 256);
}

static glowq_status w4a8_impl(const glowq_module* mods, int32_t m, int64_t d, const uint16_t* B, int32_t r,
                              const uint16_t* X, int64_t T, uint16_t* R_out, void* workspace, size_t workspace_bytes,
                              cudaStream_t st, bool solo) {
    glowq_status v = validate_forward(mods, m, d, B, r, X, T);
    if (v != GLOWQ_OK) return v;
    if (T == 0) return GLOWQ_OK;
    if (!solo && r > 0) {
        if (!R_out) return GLOWQ_ERR_ARG;
        if (!aligned16(R_out)) return GLOWQ_ERR_ALIGN;
    }
    if (!workspace || workspace_bytes < glowq_w4a8_workspace_bytes(T, d, r)) return GLOWQ_ERR_ARG;
    if (!aligned16(workspace)) return GLOWQ_ERR_ALIGN;
    char* ws = static_cast<char*>(workspace);
    uint16_t* Xq = reinterpret_cast<uint16_t*>(ws + w4a8_xq_offset(T, r));
    float* ts = reinterpret_cast<float*>(ws + w4a8_scale_offset(T, d, r));
    uint16_t* Rp = reinterpret_cast<uint16_t*>(ws + w4a8_rprime_offset(T, d, r));
    if (launch_quantize_act_e4m3(X, T, d, nullptr, ts, Xq, st) != cudaSuccess) return GLOWQ_ERR_CUDA;
    ModuleView hm[GLOWQ_MAX_MODULES];
    for (int i = 0; i < m; ++i)
        hm[i] = {mods[i].qweight, mods[i].scales, mods[i].zeros, nullptr, (r > 0) ? mods[i].A : nullptr,
                 mods[i].Y, mods[i].ldY, mods[i].out_features};
    uint16_t* Rsolo = r > 0 ? reinterpret_cast<uint16_t*>(ws + workspace_flag_bytes(r) + workspace_partial_bytes(T, r))
                            : nullptr;
    uint16_t* R;
    uint16_t* Rs = nullptr;
    if (T <= kDecodeMaxTokens) {
        R = solo ? Rsolo : R_out;          // the decode kernels write the scaled R
    } else {
        R = solo ? Rsolo : Rp;             // the GEMM reads the unscaled R'
        Rs = solo ? nullptr : R_out;
    }
    return forward_views(hm, m, d, B, r, Xq, T, R, workspace, 0, st, GLOWQ_FMT_INT4, ts, Rs);
}

glowq_status glowq_group_forward_w4a8(const glowq_module* mods, int32_t m, int64_t d, const uint16_t* B, int32_t r,
                                      const uint16_t* X, int64_t T, uint16_t* R_out, void* workspace,
                                      size_t workspace_bytes, void* stream) {
    return w4a8_impl(mods, m, d, B, r, X, T, R_out, workspace, workspace_bytes, (cudaStream_t)stream, false);
}

glowq_status glowq_solo_forward_w4a8(const glowq_module* mod, int64_t d, const uint16_t* B, int32_t r,
                                     const uint16_t* X, int64_t T, void* workspace, size_t workspace_bytes,
                                     void* stream) {
    return w4a8_impl(mod, 1, d, B, r, X, T, nullptr, workspace, workspace_bytes, (cudaStream_t)stream, true);
}

glowq_status glowq_selftest_wait_timeout(uint32_t polls, void* stream) {
    if (polls < 1 || polls > 65536) return GLOWQ_ERR_ARG;
    unsigned int* status = device_status_ptr();
    if (!status) return GLOWQ_ERR_CUDA;
    selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(polls, status);
    return cudaGetLastError() == cudaSuccess ? GLOWQ_OK : GLOWQ_ERR_CUDA;
}

glowq_status glowq_get_device_status(void* stream) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return GLOWQ_ERR_CUDA;
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v)) != cudaSuccess) return GLOWQ_ERR_CUDA;
    if (v != 0 && cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)) != cudaSuccess) return GLOWQ_ERR_CUDA;
    return (glowq_status)v;
}

}  // extern "C"
