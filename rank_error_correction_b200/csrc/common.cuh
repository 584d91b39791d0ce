// common.cuh -- shared device helpers for libglowq (sm_100a).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "glowq.h"

namespace glowq {

constexpr int kGroup = GLOWQ_GROUP_SIZE;   // INT4 quantisation group along d

// INT4 packed weights are stored in blocks of 16 rows x 64 k (8 words of 8
// codes per row, 512 B), blocks ordered along k within a 16-row tile and tiles
// in row order: word kw of row o (codes of k = 8 kw .. 8 kw + 7) sits at this
// index.  A decode ring stage (16 rows x two 128-groups) is then 2 KB of
// contiguous memory, and a prefill k-block (128 rows x 64 k) eight
// contiguous 512-byte blocks.
__host__ __device__ __forceinline__ int64_t qword_index(int64_t o, int64_t kw, int64_t d) {
    return ((((o >> 4) * (d >> 6) + (kw >> 3)) << 7) | ((o & 15) << 3) | (kw & 7));
}

// Bounded waits that run out record a code in the per-device status word
// (defined in api.cu; kernels receive its device address as an argument).
__device__ __forceinline__ void record_status(unsigned int* status, unsigned int code) {
    if (status) atomicCAS(status, 0u, code);
}

// ---- programmatic dependent launch (PDL) ----------------------------------
// griddepcontrol.wait: block until the grids this one depends on completed
// and their writes are visible; a no-op when launched without the attribute.
__device__ __forceinline__ void pdl_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
// Allow the next PDL-launched grid in the stream to be scheduled.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- loads ----------------------------------------------------------------
// Streaming 128-bit load that does not allocate in L1 (weights are read once).
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}
__device__ __forceinline__ uint4 ldg_128(const void* p) {
    return __ldg(reinterpret_cast<const uint4*>(p));
}
// Loads served by L2 (never by a possibly stale L1 line) for data that a kernel
// overlapping this one may have written: activations produced before a
// programmatic launch, R produced by a concurrently running kernel.
__device__ __forceinline__ uint4 ldcg_128(const void* p) {
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p)
                 : "memory");
    return v;
}
__device__ __forceinline__ float ldcg_f32(const float* p) {
    float v;
    asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint2 ldcg_64(const void* p) {
    uint2 v;
    asm volatile("ld.global.cg.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p) : "memory");
    return v;
}

// ---- flags in global memory between concurrently running kernels ----------
// Release: this thread's earlier writes (and those it has observed) become
// visible to any thread that acquires the incremented value.
__device__ __forceinline__ void flag_release_add(unsigned int* f, unsigned int v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(f), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned int flag_acquire_load(const unsigned int* f) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
    return v;
}
// Bounded wait until *f >= target.  Returns false (and records
// GLOWQ_ERR_TIMEOUT) if the value was not reached within `limit` polls.
__device__ __forceinline__ bool flag_wait_geq(const unsigned int* f, unsigned int target, unsigned int* status,
                                              uint32_t limit = (1u << 22)) {
    for (uint32_t it = 0; it < limit; ++it) {
        if (flag_acquire_load(f) >= target) return true;
        if (it >= 64) __nanosleep(64);
    }
    record_status(status, GLOWQ_ERR_TIMEOUT);
    return false;
}

// ---- mbarriers and bulk (TMA) copies --------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
// Make barrier initialisation visible to the async proxy (bulk copies).
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
// Arrive (release, CTA scope) on an mbarrier.
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Bounded wait for the phase with the given parity to complete.  Returns false
// (and records GLOWQ_ERR_TIMEOUT) if it did not complete within `limit` polls.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned int* status,
                                          uint32_t limit = (1u << 20)) {
    const uint32_t a = smem_u32(bar);
    for (uint32_t it = 0; it < limit; ++it) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(a), "r"(parity)
            : "memory");
        if (done) return true;
    }
    record_status(status, GLOWQ_ERR_TIMEOUT);
    return false;
}
// Contiguous global -> shared bulk copy completing on an mbarrier
// (16-byte aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_g2s(uint32_t dst_smem, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst_smem), "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
// 2-D tiled TMA load (tensor map in parameter/constant space) completing on an mbarrier.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* map, uint64_t* bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const void* map, uint64_t* bar, int c0, int c1, int c2,
                                            int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
        : "memory");
}
// L2 policy for data read exactly once per call (decode weight streams): its
// lines are the first evicted, so activations, flags and R stay resident.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
// 2-D tiled TMA load with an L2 cache policy.
__device__ __forceinline__ void tma_load_2d_hint(uint32_t dst, const void* map, uint64_t* bar, int x, int y,
                                                 uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}
// Order this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (bulk copy) accesses.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- half2 packing -------------------------------------------------------
__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) {
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) {
    return *reinterpret_cast<__half2*>(&u);
}

// INT4 -> fp16 dequantisation of one packed word (8 codes, low nibble first).
// Produces four half2 values holding codes (0,4), (1,5), (2,6), (3,7): the
// nibble n is placed in the mantissa of 1024.0 (0x6400 | n == 1024 + n), the
// biased zero (1024 + z) is subtracted exactly, and the exact integer q - z is
// multiplied by the scale with a single fp16 rounding -- bit-identical to
// fp16_RN((q - z) * s).
__device__ __forceinline__ void dequant_word(uint32_t w, __half2 bias_z, __half2 scale,
                                             __half2 out[4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t v = ((w >> (4 * i)) & 0x000F000Fu) | 0x64006400u;   // one LOP3 (+ shift)
        out[i] = __hmul2(__hsub2(u32_as_h2(v), bias_z), scale);
    }
}

// Same unpacking without the scale: four half2 holding the exact integers
// (q - z) of codes (0,4), (1,5), (2,6), (3,7); the caller applies the group
// scale after the dot product.
__device__ __forceinline__ void unpack_sub_word(uint32_t w, __half2 bias_z, __half2 out[4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t v = ((w >> (4 * i)) & 0x000F000Fu) | 0x64006400u;   // one LOP3 (+ shift)
        out[i] = __hsub2(u32_as_h2(v), bias_z);
    }
}

// ---- warp-level MMA (register operands) ---------------------------------
// D(16x8 fp32) += A(16x16 fp16) * B(16x8 fp16)
__device__ __forceinline__ void mma_16816(float c[4], const uint32_t a[4], const uint32_t b[2]) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// byte_perm helpers to pair halves: lo halves of (x, y) and hi halves of (x, y)
__device__ __forceinline__ uint32_t pair_lo(uint32_t x, uint32_t y) { return __byte_perm(x, y, 0x5410); }
__device__ __forceinline__ uint32_t pair_hi(uint32_t x, uint32_t y) { return __byte_perm(x, y, 0x7632); }

}  // namespace glowq
