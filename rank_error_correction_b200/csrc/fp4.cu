// fp4.cu -- MXFP4 and NVFP4 base weights: quantisation/packing and
// dequantisation (thelatestinai.com GlowQ page, Table 13: GlowQ's correction
// on top of MXFP4 and NVFP4 base weights).
//
// The pages name the datatypes without defining them; the definitions used
// here are their public ones, each a reading stated in glowq.h:
//   E2M1 element: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0;
//     magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6; nearest, ties to the even
//     mantissa, saturating at 6; zero and NaN encode as 0.
//   MXFP4: blocks of 32 k, one E8M0 scale 2^(floor(log2 amax) - 2).
//   NVFP4: blocks of 16 k, one E4M3 scale of amax / (6 s_t), one fp32 tensor
//     scale s_t = amax_tensor / (6 * 448).
// Codes are packed like INT4: code k of a row is nibble (k % 8) of word k / 8.
#include "common.cuh"
#include "internal.cuh"

namespace glowq {

// E2M1 code of v (sign applied, zero and NaN -> 0).
__device__ __forceinline__ uint32_t e2m1_encode(float v) {
    const float a = fabsf(v);
    if (!(a > 0.0f)) return 0u;   // zero or NaN
    uint32_t c;
    if (a <= 0.25f) c = 0;        // tie at 0.25 -> 0 (even mantissa)
    else if (a < 0.75f) c = 1;    // 0.5
    else if (a <= 1.25f) c = 2;   // 1.0 (ties at 0.75 and 1.25 go to it)
    else if (a < 1.75f) c = 3;    // 1.5
    else if (a <= 2.5f) c = 4;    // 2.0
    else if (a < 3.5f) c = 5;     // 3.0
    else if (a <= 5.0f) c = 6;    // 4.0
    else c = 7;                   // 6.0, saturating
    if (c == 0) return 0u;
    return c | (v < 0.0f ? 8u : 0u);
}

// Exact value of an E2M1 code.
__device__ __forceinline__ float e2m1_value(uint32_t c) {
    const uint32_t e = (c >> 1) & 3u, m = c & 1u;
    const float mag = (e == 0) ? 0.5f * (float)m : ldexpf(1.0f + 0.5f * (float)m, (int)e - 1);
    return (c & 8u) ? -mag : mag;
}

// E4M3 (no infinities, largest finite 448) code of a >= 0: nearest, ties to
// the even mantissa, saturating at 448; NaN -> 0x7f.
__device__ __forceinline__ uint32_t e4m3_encode_nonneg(float a) {
    if (!(a == a)) return 0x7fu;
    if (a >= 448.0f) return 0x7eu;
    if (a < 0.015625f) {                        // below 2^-6: subnormal grid m * 2^-9
        const float m = rintf(a * 512.0f);      // exact scaling, round half to even
        return (uint32_t)m;                     // m == 8 is the smallest normal, code 0x08
    }
    const int E = (int)((__float_as_uint(a) >> 23) & 0xffu) - 127;   // floor(log2 a), a normal
    const float r = ldexpf(a, -E);                                     // in [1, 2), exact
    float m = rintf((r - 1.0f) * 8.0f);                                // exact, ties to even
    int e = E + 7;
    if (m == 8.0f) {
        m = 0.0f;
        ++e;
    }
    const uint32_t code = ((uint32_t)e << 3) | (uint32_t)m;
    return code > 0x7eu ? 0x7eu : code;
}

__device__ __forceinline__ float e4m3_value(uint32_t c) {
    const uint32_t e = (c >> 3) & 15u, m = c & 7u;
    const float mag = (e == 0) ? ldexpf((float)m, -9) : ldexpf(1.0f + (float)m / 8.0f, (int)e - 7);
    return (c & 0x80u) ? -mag : mag;
}

// One warp per (row, 128 k): lane l owns k = 4l .. 4l+3 (one float4), eight
// lanes per MXFP4 block; two lanes form a packed word.
__global__ void __launch_bounds__(256) pack_mxfp4_kernel(const float* __restrict__ W, int64_t O, int64_t d,
                                                          uint32_t* __restrict__ codes, uint8_t* __restrict__ scales) {
    const int lane = threadIdx.x & 31;
    const int64_t nc = d / 128;
    const int64_t unit = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (unit >= O * nc) return;
    const int64_t o = unit / nc, c = unit % nc;
    const float4 w4 = __ldg(reinterpret_cast<const float4*>(W + o * d + c * 128) + lane);
    const float w[4] = {w4.x, w4.y, w4.z, w4.w};
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        if (fabsf(w[i]) > amax) amax = fabsf(w[i]);   // NaN never compares greater
#pragma unroll
    for (int off = 4; off > 0; off >>= 1) {          // the 8 lanes of this block
        const float oa = __shfl_xor_sync(0xffffffffu, amax, off);
        if (oa > amax) amax = oa;
    }
    // E8M0 code: floor(log2 amax) - 2, biased by 127, clamped to 0..254
    int e = 0;
    if (amax > 0.0f) {
        const int be = (int)((__float_as_uint(amax) >> 23) & 0xffu);
        e = (be == 255) ? 124 : be - 2;   // an infinite amax takes frexp's exponent 0
        e = e < 0 ? 0 : (e > 254 ? 254 : e);
    }
    // 2^(e - 127): normal for e >= 1, the subnormal 2^-127 for e == 0
    const float X = (e >= 1) ? __uint_as_float((uint32_t)e << 23) : __uint_as_float(0x00400000u);
    uint32_t nib = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) nib |= e2m1_encode(__fdiv_rn(w[i], X)) << (4 * i);
    const uint32_t hi = __shfl_down_sync(0xffffffffu, nib, 1);
    if ((lane & 1) == 0) codes[o * (d / 8) + c * 16 + lane / 2] = nib | (hi << 16);
    if ((lane & 7) == 0) scales[o * (d / 32) + c * 4 + lane / 8] = (uint8_t)e;
}

// Largest |w| of the tensor (NaN ignored) as float bits, by atomicMax on the
// bits of non-negative floats (their order is the integer order).
__global__ void __launch_bounds__(256) absmax_kernel(const float* __restrict__ W, int64_t n,
                                                      unsigned int* __restrict__ out) {
    float m = 0.0f;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const float a = fabsf(W[i]);
        if (a > m) m = a;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float o = __shfl_xor_sync(0xffffffffu, m, off);
        if (o > m) m = o;
    }
    if ((threadIdx.x & 31) == 0) atomicMax(out, __float_as_uint(m));
}

// Tensor scale s_t = amax / (6 * 448) (1 for an all-zero tensor), in place.
__global__ void nvfp4_tensor_scale_kernel(float* st) {
    const float amax = *st;   // written as float bits by absmax_kernel
    float s = __fdiv_rn(amax, 2688.0f);
    if (!(s > 0.0f)) s = 1.0f;
    *st = s;
}

// One warp per (row, 128 k): lane l owns k = 4l .. 4l+3, four lanes per
// NVFP4 block.
__global__ void __launch_bounds__(256) pack_nvfp4_kernel(const float* __restrict__ W, int64_t O, int64_t d,
                                                          const float* __restrict__ st_p,
                                                          uint32_t* __restrict__ codes, uint8_t* __restrict__ scales) {
    const int lane = threadIdx.x & 31;
    const int64_t nc = d / 128;
    const int64_t unit = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (unit >= O * nc) return;
    const int64_t o = unit / nc, c = unit % nc;
    const float st = *st_p;
    const float4 w4 = __ldg(reinterpret_cast<const float4*>(W + o * d + c * 128) + lane);
    const float w[4] = {w4.x, w4.y, w4.z, w4.w};
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        if (fabsf(w[i]) > amax) amax = fabsf(w[i]);
#pragma unroll
    for (int off = 2; off > 0; off >>= 1) {          // the 4 lanes of this block
        const float oa = __shfl_xor_sync(0xffffffffu, amax, off);
        if (oa > amax) amax = oa;
    }
    const float six_st = __fmul_rn(6.0f, st);
    const uint32_t S = e4m3_encode_nonneg(__fdiv_rn(amax, six_st));
    const float full = __fmul_rn(e4m3_value(S), st);
    uint32_t nib = 0;
    if (full > 0.0f) {
#pragma unroll
        for (int i = 0; i < 4; ++i) nib |= e2m1_encode(__fdiv_rn(w[i], full)) << (4 * i);
    }
    const uint32_t hi = __shfl_down_sync(0xffffffffu, nib, 1);
    if ((lane & 1) == 0) codes[o * (d / 8) + c * 16 + lane / 2] = nib | (hi << 16);
    if ((lane & 3) == 0) scales[o * (d / 16) + c * 8 + lane / 4] = (uint8_t)S;
}

// w_hat = fp16_RN(exact dequantised value): MXFP4 e2m1 * 2^(e - 127) is exact
// in fp32; NVFP4 e2m1 * e4m3 * s_t is formed exactly in fp64.
__global__ void __launch_bounds__(256) dequant_fp4_kernel(int fmt, const uint32_t* __restrict__ codes,
                                                           const uint8_t* __restrict__ scales,
                                                           const float* __restrict__ st_p, int64_t O, int64_t d,
                                                           __half* __restrict__ out) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;   // one packed word
    if (i >= O * (d / 8)) return;
    const int64_t o = i / (d / 8), k0 = (i % (d / 8)) * 8;
    const uint32_t w = codes[i];
    __align__(16) __half h[8];
    if (fmt == GLOWQ_FMT_MXFP4) {
        const uint32_t e = scales[o * (d / 32) + k0 / 32];
        const float X = (e >= 1) ? __uint_as_float(e << 23) : __uint_as_float(0x00400000u);
#pragma unroll
        for (int j = 0; j < 8; ++j) h[j] = __float2half_rn(e2m1_value((w >> (4 * j)) & 0xfu) * X);
    } else {
        const double f = (double)e4m3_value(scales[o * (d / 16) + k0 / 16]) * (double)(*st_p);
#pragma unroll
        for (int j = 0; j < 8; ++j) h[j] = __double2half((double)e2m1_value((w >> (4 * j)) & 0xfu) * f);
    }
    *reinterpret_cast<uint4*>(out + o * d + k0) = *reinterpret_cast<const uint4*>(h);
}

// ---------------------------------------------------------------------------
// W4A8 activations (thelatestinai.com GlowQ page, Tables 14-15: GlowQ with
// FP8 activations): per token t, s_t = amax_t / 448 (1 for an all-zero row)
// and codes E4M3(x / s_t), nearest, ties to even, saturating at 448, NaN ->
// 0x7f; a value that rounds to zero keeps code 0 whatever its sign.  One CTA
// per token.  Writes the codes (optional), s_t, and the exact code values as
// fp16 (X' = x_hat / s_t, so that x_hat = s_t X').
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t e4m3_encode(float v) {
    if (!(v == v)) return 0x7fu;
    const uint32_t c = e4m3_encode_nonneg(fabsf(v));
    return (c != 0u && v < 0.0f) ? (c | 0x80u) : c;
}

__global__ void __launch_bounds__(256) quantize_act_e4m3_kernel(const __half* __restrict__ X, int64_t d,
                                                                 uint8_t* __restrict__ codes, float* __restrict__ scales,
                                                                 __half* __restrict__ Xq) {
    __shared__ float wmax[8];
    const int64_t t = blockIdx.x;
    const __half* x = X + t * d;
    float amax = 0.0f;
    for (int64_t k = threadIdx.x; k < d; k += blockDim.x) {
        const float a = fabsf(__half2float(x[k]));
        if (a > amax) amax = a;                       // NaN never compares greater
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float b = __shfl_xor_sync(0xffffffffu, amax, o);
        if (b > amax) amax = b;
    }
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = 0.0f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w)
        if (wmax[w] > amax) amax = wmax[w];
    float s = __fdiv_rn(amax, 448.0f);
    if (!(s > 0.0f)) s = 1.0f;
    if (threadIdx.x == 0) scales[t] = s;
    for (int64_t k = threadIdx.x; k < d; k += blockDim.x) {
        const uint32_t c = e4m3_encode(__fdiv_rn(__half2float(x[k]), s));
        if (codes) codes[t * d + k] = (uint8_t)c;
        // exact: E4M3 values are fp16 values (the NaN codes stay NaN)
        Xq[t * d + k] = ((c & 0x7fu) == 0x7fu) ? __ushort_as_half((unsigned short)0x7e00u)
                                               : __float2half_rn(e4m3_value(c));
    }
}

cudaError_t launch_quantize_act_e4m3(const uint16_t* X, int64_t T, int64_t d, uint8_t* codes, float* scales,
                                     uint16_t* Xq, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    quantize_act_e4m3_kernel<<<(unsigned)T, 256, 0, st>>>(reinterpret_cast<const __half*>(X), d, codes, scales,
                                                           reinterpret_cast<__half*>(Xq));
    return cudaGetLastError();
}

cudaError_t launch_pack_fp4(int fmt, const float* W, int64_t O, int64_t d, uint32_t* codes, uint8_t* scales,
                            float* tensor_scale, cudaStream_t st) {
    const int64_t units = O * (d / 128);
    const unsigned blocks = (unsigned)((units + 7) / 8);
    if (fmt == GLOWQ_FMT_MXFP4) {
        pack_mxfp4_kernel<<<blocks, 256, 0, st>>>(W, O, d, codes, scales);
        return cudaGetLastError();
    }
    cudaError_t e = cudaMemsetAsync(tensor_scale, 0, sizeof(float), st);
    if (e != cudaSuccess) return e;
    const int64_t n = O * d;
    int64_t nb = (n + 255) / 256;
    if (nb > 4096) nb = 4096;
    absmax_kernel<<<(unsigned)nb, 256, 0, st>>>(W, n, reinterpret_cast<unsigned int*>(tensor_scale));
    nvfp4_tensor_scale_kernel<<<1, 1, 0, st>>>(tensor_scale);
    pack_nvfp4_kernel<<<blocks, 256, 0, st>>>(W, O, d, tensor_scale, codes, scales);
    return cudaGetLastError();
}

cudaError_t launch_dequant_fp4(int fmt, const uint32_t* codes, const uint8_t* scales, const float* tensor_scale,
                               int64_t O, int64_t d, uint16_t* out, cudaStream_t st) {
    const int64_t words = O * (d / 8);
    dequant_fp4_kernel<<<(unsigned)((words + 255) / 256), 256, 0, st>>>(fmt, codes, scales, tensor_scale, O, d,
                                                                         reinterpret_cast<__half*>(out));
    return cudaGetLastError();
}

}  // namespace glowq
