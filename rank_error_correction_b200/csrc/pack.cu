// pack.cu -- INT4 g128 asymmetric quantisation/packing, dequantisation and the
// quantisation-error norms used by GlowQ-S.
//
// GlowQ pages, papernotes.org summary, experimental set-up paragraph: W4A16
// with INT4 weights in groups of 128.  The quantiser's exact arithmetic is this
// library's reading (asymmetric round-to-nearest with zero kept exactly
// representable), stated in glowq.h beside glowq_pack_int4.
#include "common.cuh"

namespace glowq {

__device__ __forceinline__ float clamp_code(float v) {
    if (!(v >= 0.0f)) v = 0.0f;  // also NaN -> 0
    if (v > 15.0f) v = 15.0f;
    return v;
}

// One warp per (row, 128-group).  Lane l owns elements 4l .. 4l+3 (one float4),
// i.e. half of packed word l/2.
__global__ void __launch_bounds__(256) pack_int4_kernel(const float* __restrict__ W, int64_t O,
                                                         int64_t d, uint32_t* __restrict__ q,
                                                         __half* __restrict__ s, uint8_t* __restrict__ z) {
    const int lane = threadIdx.x & 31;
    const int64_t ng = d / kGroup;
    const int64_t unit = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (unit >= O * ng) return;
    const int64_t o = unit / ng, g = unit % ng;
    const float4 w4 = __ldg(reinterpret_cast<const float4*>(W + o * d + g * kGroup) + lane);
    const float w[4] = {w4.x, w4.y, w4.z, w4.w};
    float mn = 0.0f, mx = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        mn = (w[i] < mn) ? w[i] : mn;
        mx = (w[i] > mx) ? w[i] : mx;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float omn = __shfl_xor_sync(0xffffffffu, mn, off);
        const float omx = __shfl_xor_sync(0xffffffffu, mx, off);
        mn = (omn < mn) ? omn : mn;
        mx = (omx > mx) ? omx : mx;
    }
    const float range = __fsub_rn(mx, mn);
    const float s32 = __fdiv_rn(range, 15.0f);
    __half sh = __float2half_rn(s32);
    unsigned short sb = __half_as_ushort(sh);
    if ((sb & 0x7fffu) == 0u) sb = 0x3c00u;        // 1.0
    if ((sb & 0x7fffu) == 0x7c00u) sb = 0x7bffu;   // 65504
    sh = __ushort_as_half(sb);
    const float sf = __half2float(sh);
    const float zf = clamp_code(rintf(__fdiv_rn(-mn, sf)));
    uint32_t nib = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float c = clamp_code(__fadd_rn(rintf(__fdiv_rn(w[i], sf)), zf));
        nib |= ((uint32_t)c & 0xfu) << (4 * i);
    }
    const uint32_t hi = __shfl_down_sync(0xffffffffu, nib, 1);
    if ((lane & 1) == 0) q[qword_index(o, g * (kGroup / 8) + lane / 2, d)] = nib | (hi << 16);
    if (lane == 0) {
        s[o * ng + g] = sh;
        z[o * ng + g] = (uint8_t)zf;
    }
}

// One thread per packed word (row-major order of the output): 8 fp16 outputs
// (one 16-byte store).
__global__ void __launch_bounds__(256) dequant_int4_kernel(const uint32_t* __restrict__ q,
                                                            const __half* __restrict__ s,
                                                            const uint8_t* __restrict__ z, int64_t O,
                                                            int64_t d, __half* __restrict__ out) {
    const int64_t words = O * (d / 8);
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= words) return;
    const int64_t o = i / (d / 8), kw = i % (d / 8);
    const int64_t g = (kw * 8) / kGroup;
    const int64_t ng = d / kGroup;
    const uint32_t w = q[qword_index(o, kw, d)];
    const float sf = __half2float(s[o * ng + g]);
    const int zz = z[o * ng + g];
    __align__(16) __half v[8];
#pragma unroll
    for (int n = 0; n < 8; ++n) {
        const int c = (w >> (4 * n)) & 0xf;
        // (c - z) * s is exact in fp32 (<= 4 x 11 significant bits); one rounding to fp16
        v[n] = __float2half_rn(__fmul_rn((float)(c - zz), sf));
    }
    *reinterpret_cast<uint4*>(out + o * d + kw * 8) = *reinterpret_cast<uint4*>(v);
}

// Per-row ||W - w_hat||^2 and ||W||^2 in fp64, one warp per row (fixed
// reduction order, so the result is deterministic).  out: [O][2].
__global__ void __launch_bounds__(256) error_norms_kernel(const float* __restrict__ W,
                                                           const uint32_t* __restrict__ q,
                                                           const __half* __restrict__ s,
                                                           const uint8_t* __restrict__ z, int64_t O,
                                                           int64_t d, double* __restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int64_t o = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (o >= O) return;
    const int64_t ng = d / kGroup;
    double se = 0.0, sw = 0.0;
    for (int64_t kw = lane; kw < d / 8; kw += 32) {
        const int64_t g = (kw * 8) / kGroup;
        const uint32_t w = q[qword_index(o, kw, d)];
        const float sf = __half2float(s[o * ng + g]);
        const int zz = z[o * ng + g];
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            const int c = (w >> (4 * n)) & 0xf;
            const double wh = (double)__half2float(__float2half_rn(__fmul_rn((float)(c - zz), sf)));
            const double wv = (double)W[o * d + kw * 8 + n];
            se += (wv - wh) * (wv - wh);
            sw += wv * wv;
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        se += __shfl_xor_sync(0xffffffffu, se, off);
        sw += __shfl_xor_sync(0xffffffffu, sw, off);
    }
    if (lane == 0) {
        out[2 * o] = se;
        out[2 * o + 1] = sw;
    }
}

cudaError_t launch_pack_int4(const float* W, int64_t O, int64_t d, uint32_t* q, uint16_t* s, uint8_t* z,
                             cudaStream_t st) {
    const int64_t units = O * (d / kGroup);
    if (units == 0) return cudaSuccess;
    const int warps = 8;
    const int64_t blocks = (units + warps - 1) / warps;
    pack_int4_kernel<<<(unsigned)blocks, warps * 32, 0, st>>>(W, O, d, q, reinterpret_cast<__half*>(s), z);
    return cudaGetLastError();
}

cudaError_t launch_dequant_int4(const uint32_t* q, const uint16_t* s, const uint8_t* z, int64_t O, int64_t d,
                                uint16_t* out, cudaStream_t st) {
    const int64_t words = O * (d / 8);
    if (words == 0) return cudaSuccess;
    dequant_int4_kernel<<<(unsigned)((words + 255) / 256), 256, 0, st>>>(
        q, reinterpret_cast<const __half*>(s), z, O, d, reinterpret_cast<__half*>(out));
    return cudaGetLastError();
}

cudaError_t launch_error_norms(const float* W, const uint32_t* q, const uint16_t* s, const uint8_t* z,
                               int64_t O, int64_t d, double* out_rows, cudaStream_t st) {
    if (O == 0) return cudaSuccess;
    error_norms_kernel<<<(unsigned)((O + 7) / 8), 256, 0, st>>>(W, q, reinterpret_cast<const __half*>(s), z,
                                                                O, d, out_rows);
    return cudaGetLastError();
}

}  // namespace glowq
