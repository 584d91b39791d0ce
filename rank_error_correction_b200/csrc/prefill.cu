// prefill.cu -- large-T path (tcgen05 tensor-core kernels); placeholder until
// the tcgen05 kernels land: large T is reported as unsupported.
#include "common.cuh"
#include "internal.cuh"

namespace glowq {


glowq_status prefill_group_forward(const ModuleView*, int, int, const uint16_t*, int, const uint16_t*, int64_t,
                                   uint16_t*, int, cudaStream_t) {
    return GLOWQ_ERR_UNSUPPORTED;
}

}  // namespace glowq
