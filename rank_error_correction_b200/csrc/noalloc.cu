// noalloc.cu -- a solo-module forward that allocates nothing.
//
// glowq_solo_forward needs a scratch workspace (the projection R = X B^T and,
// for small T, its split-d partial sums).  Normally the caller allocates it.
// Some callers cannot allocate device memory when they call us: a custom op or
// plugin running inside another runtime's enqueue step, where that runtime
// owns every device allocation and forbids cudaMalloc/cudaFree on its hot
// path.  For them, glowq_solo_forward_noalloc uses a fixed scratch array
// compiled into the library instead, so the call allocates nothing.
#include <cuda_runtime.h>

#include "common.cuh"

namespace {

constexpr size_t kNoallocScratchBytes = (size_t)1 << 20;   // 1 MiB per device

// Lives in every device that loads the library, for the life of the process.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
static void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  The host-side
// symbol is only a stand-in; the kernels need the address the runtime reports.
static void* scratch_for_current_device(glowq_status* err) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        *err = GLOWQ_ERR_CUDA;
        return nullptr;
    }
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            *err = GLOWQ_ERR_CUDA;
            return nullptr;
        }
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" {

size_t glowq_noalloc_scratch_bytes(void) { return kNoallocScratchBytes; }

glowq_status glowq_solo_forward_noalloc(const glowq_module* mod, int64_t d, const uint16_t* B, int32_t r,
                                        const uint16_t* X, int64_t T, void* stream) {
    if (T < 0 || r < 0) return GLOWQ_ERR_ARG;
    if (glowq_workspace_bytes(T, r) > kNoallocScratchBytes) return GLOWQ_ERR_SHAPE;
    glowq_status err = GLOWQ_OK;
    void* scratch = scratch_for_current_device(&err);
    if (!scratch) return err;
    return glowq_solo_forward(mod, d, B, r, X, T, scratch, kNoallocScratchBytes, stream);
}

}  // extern "C"
