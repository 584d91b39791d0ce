// noalloc.cu -- a solo-module forward that allocates nothing.
//
// glowq_solo_forward needs a scratch workspace (the projection R = X B^T, the
// decode hand-off flags, for T > 16 the split-d partial sums of R, and for
// small batches the k-split's tickets and partial tiles).
// Normally the caller allocates it.  Some callers cannot allocate device
// memory when they call us: a custom op or plugin running inside another
// runtime's enqueue step, where that runtime owns every device allocation and
// forbids cudaMalloc/cudaFree on its hot path.  For them,
// glowq_solo_forward_noalloc uses a fixed scratch array compiled into the
// library instead, so the call allocates nothing.
#include <atomic>

#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.cuh"

namespace {

constexpr size_t kNoallocScratchBytes = (size_t)1 << 20;   // 1 MiB per device
// The first 4 KB of any workspace (the decode kernels' hand-off flags and the
// tensor-core GEMM's k-split tickets) must read zero when a call starts.
constexpr size_t kZeroBytes = 4096;

// Lives in every device that loads the library, for the life of the process.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
// Device address of the array per device, looked up once.  Two host threads
// making their first call together both store the same value.  The cache
// holds for the life of the CUDA context: it is not refreshed after a
// cudaDeviceReset.
static std::atomic<void*> g_scratch_ptr[kMaxDevices];

// Device address of the scratch array on the current device.  In host code the
// symbol g_noalloc_scratch is only a host-side stand-in; the kernels need the
// address the runtime reports for this device.
static void* scratch_for_current_device(glowq_status* err) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        *err = GLOWQ_ERR_CUDA;
        return nullptr;
    }
    void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
    if (!p) {
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            *err = GLOWQ_ERR_CUDA;
            return nullptr;
        }
        g_scratch_ptr[dev].store(p, std::memory_order_release);
    }
    return p;
}

}  // namespace

extern "C" {

size_t glowq_noalloc_scratch_bytes(void) { return kNoallocScratchBytes; }

glowq_status glowq_solo_forward_noalloc(const glowq_module* mod, int64_t d, const uint16_t* B, int32_t r,
                                        const uint16_t* X, int64_t T, void* stream) {
    // every host-side check runs before anything is enqueued
    const glowq_status v = glowq::validate_solo_call(mod, d, B, r, X, T);
    if (v != GLOWQ_OK) return v;
    if (glowq_workspace_bytes(T, r) > kNoallocScratchBytes) return GLOWQ_ERR_SHAPE;
    if (T == 0) return GLOWQ_OK;
    glowq_status err = GLOWQ_OK;
    void* scratch = scratch_for_current_device(&err);
    if (!scratch) return err;
    // The array keeps whatever the previous call left, including flags or
    // tickets a failed or timed-out call may have left non-zero: clear them,
    // ordered on the caller's stream before this call's kernels (no allocation).
    if (cudaMemsetAsync(scratch, 0, kZeroBytes, (cudaStream_t)stream) != cudaSuccess) return GLOWQ_ERR_CUDA;
    return glowq_solo_forward(mod, d, B, r, X, T, scratch, kNoallocScratchBytes, stream);
}

}  // extern "C"
