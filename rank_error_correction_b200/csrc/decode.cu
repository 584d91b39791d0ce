// decode.cu -- small-T (T <= 16) path of the GlowQ corrected linear layer.
//
// GlowQ pages, papernotes.org summary, key design 4: one shared projection
// R = X B^T per input-sharing group, then y_i = W_i^(q) X + A_i R for every
// module; solo modules compute their own R inline.
//
// At T <= 16 the layer is a weight-streaming GEMV: every INT4 weight byte is
// read once from HBM and meets at most 16 tokens, so the kernels are HBM-bound.
// One call is two launches chained with programmatic dependent launch:
//   * rproj_cluster: R = X B^T by one cluster of 8 CTAs splitting d; the
//     partial sums meet on chip in a fixed order (deterministic), R is rounded
//     to fp16 once and written to the caller's R buffer.  It lets the GEMV
//     launch once X is final and tells it through workspace flags when X is
//     final and when R is stored.
//   * corrected_gemv: one launch over the stacked rows of all modules of the
//     group.  Each warp streams its 16 rows of packed weights with 2-D TMA
//     boxes into a private ring of mbarrier-tracked stages; the stream and the
//     main loop run while the projection is still being computed (R is needed
//     only by the epilogue, and a control warp per CTA collects it into shared
//     memory meanwhile).  Nibbles become exact fp16 values
//     (16 + q/64 for even k, 64 + q for odd k) with one LOP3 per pair; the
//     multiply-accumulate runs on the tensor cores with register operands
//     (mma.sync m16n8k16, fp32 accumulate, one chain per parity) and each
//     128-group's dot product is finished in fp32 from the two chains and the
//     even/odd activation sums.  The k order inside an MMA is permuted
//     identically on both operands (a permutation of the contraction index
//     leaves the dot product unchanged) so packed words map straight onto
//     fragments.  d may be split inside the CTA or across a thread-block
//     cluster whose partial sums meet in distributed shared memory; the
//     rank-r correction A_i R is one more short MMA slab on the same fp32
//     accumulators.
//   * Numerics: the operand products are exact, sums are fp32; the
//     effective weight is the exact (q - z) s rather
//     than its fp16 rounding (at most 2^-12 relative per weight, far inside the
//     parity bar).
#include <cstdio>
#include <cstdlib>

#include "common.cuh"
#include "internal.cuh"

namespace glowq {



// ---------------------------------------------------------------------------
// R = X B^T for T <= 16 in one launch.  A cluster of kRcCtas CTAs splits d
// (CTA c takes the c-th slice of the 32-wide k steps).  Inside a CTA the work
// items (B row block of 16 rows, k-lane) are spread over the warps; a k-lane
// takes every kl-th k step of the slice, two steps' loads in flight.  Partial
// sums meet in a fixed order: k-lanes in shared memory, then the CTAs of the
// cluster through distributed shared memory (ascending rank), so R does not
// depend on timing.  R is rounded to fp16 once.
// The CTA is small enough to be resident next to a GEMV CTA, so it starts
// while the preceding GEMV still runs: B is static, so its slice is copied
// into shared memory (or, when it does not fit, pulled into L2) before the
// wait on the preceding kernel; after the wait only X is read from memory.
//
// Hand-off to the GEMV that follows (flags = three zeroed words):
//   flags[0]  each CTA adds 1 once its wait has returned (X is final), and only
//             then allows the GEMV to launch, so the GEMV streams weights and
//             runs its main loop while R is still being computed;
//   flags[1]  each CTA adds 1 after its part of R is stored; the GEMV reads R
//             in its epilogue only after seeing kRcCtas here;
//   flags[2]  counts GEMV CTAs past both waits; the last one zeroes all three.
// A GEMV launched without the programmatic attribute starts after this kernel
// has completed and finds both counts already reached.
// ---------------------------------------------------------------------------
constexpr int kRcCtas = 8;
constexpr int kRcWarps = 8;
constexpr int kRcStageB = 72 * 1024;         // largest B slice staged in shared memory

__host__ __device__ inline int rc_row_blocks(int r) { return (r + 15) / 16; }
__host__ __device__ inline int rc_klanes(int r) {
    const int kl = kRcWarps / rc_row_blocks(r);
    return kl > 0 ? kl : 1;
}
// B slice of one CTA: r rows x (steps of 32 k), row pitch padded by 16 B
__host__ __device__ inline int rc_b_pitch(int d) {
    const int nsteps = d / 32;
    return ((nsteps + kRcCtas - 1) / kRcCtas) * 64 + 16;
}
__host__ __device__ inline bool rc_stage_b(int r, int d) { return r * rc_b_pitch(d) <= kRcStageB; }
// shared memory: per-k-lane partials [kl][8*NT][r] + the CTA partial [8*NT][r]
// (fp32), the CTA's X slice [T][slice] (fp16), then the staged B slice and its
// mbarrier
__host__ __device__ inline int rc_part_bytes(int r, int nt) { return (rc_klanes(r) + 1) * 8 * nt * r * 4; }
__host__ __device__ inline int rc_x_bytes(int d, int nt) { return 8 * nt * (rc_b_pitch(d) - 16); }
// the X slice is staged when it fits in 32 KB (wider inputs read X in the loop)
__host__ __device__ inline bool rc_stage_x(int d, int nt) { return rc_x_bytes(d, nt) <= 32 * 1024; }
__host__ __device__ inline int rc_smem_bytes(int r, int d, int nt) {
    const int p = (rc_part_bytes(r, nt) + 15) / 16 * 16 + (rc_stage_x(d, nt) ? rc_x_bytes(d, nt) : 0);
    return rc_stage_b(r, d) ? p + r * rc_b_pitch(d) + 16 : p;
}

template <int NT>
__global__ void __cluster_dims__(kRcCtas, 1, 1) __launch_bounds__(kRcWarps * 32, 4)
    rproj_cluster_kernel(const __half* __restrict__ X, const __half* __restrict__ B, int T, int d, int r,
                         __half* __restrict__ R, unsigned int* flags, unsigned int* status) {
    extern __shared__ __align__(16) float rc_smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int nrb = rc_row_blocks(r), kl = rc_klanes(r);
    const int TP = 8 * NT;                       // padded token count
    float* part = rc_smem;                       // [kl][TP][r]
    float* cpart = rc_smem + kl * TP * r;        // [TP][r]
    uint32_t crank;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(crank));
    const int nsteps = d / 32;
    const int s0 = (int)((int64_t)crank * nsteps / kRcCtas), s1 = (int)((int64_t)(crank + 1) * nsteps / kRcCtas);
    const bool staged = rc_stage_b(r, d);
    const int pitch = rc_b_pitch(d);
    const bool staged_x = rc_stage_x(d, NT);
    unsigned char* xsl = reinterpret_cast<unsigned char*>(rc_smem) + (rc_part_bytes(r, NT) + 15) / 16 * 16;
    const int xpitch = pitch - 16;               // bytes of one token's slice
    unsigned char* bs = xsl + (staged_x ? rc_x_bytes(d, NT) : 0);
    uint64_t* bbar = reinterpret_cast<uint64_t*>(bs + r * pitch);
    // B is static: stage (or prefetch) this CTA's slice before the wait
    if (staged) {
        if (threadIdx.x == 0) {
            mbar_init(bbar, 1);
            fence_mbar_init();
            mbar_arrive_expect_tx(bbar, (uint32_t)(r * (s1 - s0) * 64));
        }
        __syncthreads();
        for (int j = threadIdx.x; j < r; j += blockDim.x)
            bulk_g2s(smem_u32(bs + j * pitch), B + (int64_t)j * d + s0 * 32, (uint32_t)((s1 - s0) * 64), bbar);
    } else {
        for (int j = threadIdx.x; j < r; j += blockDim.x)
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;"
                         ::"l"(B + (int64_t)j * d + s0 * 32), "r"((uint32_t)((s1 - s0) * 64))
                         : "memory");
    }
    pdl_wait();                 // X may come from the previous kernel in the stream
    if (flags && threadIdx.x == 0) flag_release_add(flags + 0, 1u);
    pdl_launch_dependents();    // the GEMV may start streaming weights now
    // the CTA's slice of X in one round trip (16-byte chunks), padding tokens 0
    if (staged_x) {
        const int chunks = xpitch / 16, n = TP * chunks;
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            const int tok = i / chunks, c = i - tok * chunks;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (tok < T && s0 * 32 + c * 8 < s1 * 32) v = ldcg_128(X + (int64_t)tok * d + s0 * 32 + c * 8);
            *reinterpret_cast<uint4*>(xsl + tok * xpitch + c * 16) = v;
        }
    }
    if (staged) mbar_wait(bbar, 0, status);
    __syncthreads();
    const uint4 zero4 = make_uint4(0, 0, 0, 0);
    for (int item = warp; item < nrb * kl; item += kRcWarps) {
        const int rb = item % nrb, kq = item / nrb;
        const int j0 = rb * 16 + g, j1 = j0 + 8;
        float acc[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[n][i] = 0.f;
        constexpr int U = 2;   // k steps per iteration, all loads issued before the MMAs
        for (int st = s0 + kq; st < s1; st += U * kl) {
            uint4 blo[U], bhi[U], xv[U][NT];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int su = st + u * kl;
                const bool in = su < s1;
                const int k = su * 32 + 8 * t;
                if (staged) {
                    const int off = (su - s0) * 64 + 16 * t;
                    blo[u] = (in && j0 < r) ? *reinterpret_cast<const uint4*>(bs + j0 * pitch + off) : zero4;
                    bhi[u] = (in && j1 < r) ? *reinterpret_cast<const uint4*>(bs + j1 * pitch + off) : zero4;
                } else {
                    blo[u] = (in && j0 < r) ? ldg_128(B + (int64_t)j0 * d + k) : zero4;
                    bhi[u] = (in && j1 < r) ? ldg_128(B + (int64_t)j1 * d + k) : zero4;
                }
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    const int tok = n * 8 + g;
                    if (staged_x)
                        xv[u][n] = in ? *reinterpret_cast<const uint4*>(xsl + tok * xpitch + (su - s0) * 64 + 16 * t)
                                      : zero4;
                    else
                        xv[u][n] = (in && tok < T) ? ldcg_128(X + (int64_t)tok * d + k) : zero4;
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint32_t a0[4] = {blo[u].x, bhi[u].x, blo[u].y, bhi[u].y};
                const uint32_t a1[4] = {blo[u].z, bhi[u].z, blo[u].w, bhi[u].w};
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    const uint32_t b0[2] = {xv[u][n].x, xv[u][n].y};
                    const uint32_t b1[2] = {xv[u][n].z, xv[u][n].w};
                    mma_16816(acc[n], a0, b0);
                    mma_16816(acc[n], a1, b1);
                }
            }
        }
        float* my = part + kq * TP * r;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            const int tk = n * 8 + 2 * t;
            if (j0 < r) {
                my[tk * r + j0] = acc[n][0];
                my[(tk + 1) * r + j0] = acc[n][1];
            }
            if (j1 < r) {
                my[tk * r + j1] = acc[n][2];
                my[(tk + 1) * r + j1] = acc[n][3];
            }
        }
    }
    __syncthreads();
    // this CTA's partial: k-lanes in ascending order
    for (int i = threadIdx.x; i < T * r; i += blockDim.x) {
        float v = part[i];
        for (int q = 1; q < kl; ++q) v += part[q * TP * r + i];
        cpart[i] = v;
    }
    // all CTAs' partials are complete and visible in the cluster
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
    const uint32_t cbase = (uint32_t)__cvta_generic_to_shared(cpart);
    for (int i = (int)crank * blockDim.x + threadIdx.x; i < T * r; i += kRcCtas * blockDim.x) {
        float v = 0.f;
#pragma unroll
        for (int c = 0; c < kRcCtas; ++c) {
            uint32_t ra;
            asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(cbase + 4u * (uint32_t)i), "r"(c));
            float pv;
            asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(pv) : "r"(ra) : "memory");
            v = (c == 0) ? pv : v + pv;
        }
        R[i] = __float2half_rn(v);
    }
    // no CTA leaves while another may still read its shared memory
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
    // this CTA's stores of R (ordered before thread 0 by the barrier) are published
    if (flags && threadIdx.x == 0) flag_release_add(flags + 1, 1u);
}

// ---------------------------------------------------------------------------
// Corrected GEMV over the stacked rows of a group.
//
// Work shape (chosen on the host from the occupancy calculator so that every
// CTA is resident in one wave, with up to kMaxWarps compute warps per CTA):
//   * a CTA holds `rt` row tiles of 16 rows x `kw` in-CTA splits of its slice
//     of d (rt * kw warps; warp w owns tile w % rt and split w / rt);
//   * optionally a thread-block cluster of `kc` CTAs splits d further (then
//     kw == 1); partial sums meet in distributed shared memory.
//
// Arithmetic of one 128-group (row o, tokens t, codes q, zero z, scale s), with
// E / O the even / odd k of the group:
//   sum_k (q_k - z) s x_k = s * (64 D_E + D_O - (1024 + z) S_E - (64 + z) S_O),
//   D_E = sum_{k in E} (16 + q_k / 64) x_k,  D_O = sum_{k in O} (64 + q_k) x_k
//   (two tensor-core chains, fp32 accumulate),  S_E / S_O = sums of x over E / O.
// Both operand forms are exact fp16 values built without subtracting anything
// per weight: the nibble lands in mantissa bits 0..3 of 16.0 or 4..7 of 64.0,
// one shift and four LOP3 per 8 codes.  S_E and S_O are computed once per CTA,
// while the activation slice is staged.
//
// Shared memory (dynamic), in this order:
//   ring [warps][S][16][32] u32      packed-weight stream: a stage is one 2-D TMA
//                                    box of the warp's 16 rows x 2 groups (2 KB)
//   bars [warps][S] u64              mbarriers of the weight stream
//   xs   [T+1][wpt_max] uint4        the CTA's activation slice (row T all zero,
//                                    read by the lanes of padding tokens); each
//                                    8-element word stored as the half2 pairs
//                                    (x0,x4) (x2,x6) (x1,x5) (x3,x7) of the MMA B
//                                    fragment, word index XOR-swizzled
//   xsum [ncta_max][8*NT] f32        per-group activation sums S (0 for padding)
//   sz   [warps][16][nsub_max+1] f32x2  (s, 64 + z) of the warp's rows and groups
//   red  [nslots][NT*4][32] f32      partial sums sent to the finalising warp
//   as   [fin_slots][16][r+8] f16    A rows of the tiles this CTA finalises
//   rs   [8*NT][r+8] f16             R of the call (rows of padding tokens zero)
//   rbar u64                         completes when rs holds R
//
// Besides its rt * kw compute warps a CTA has one control warp.  It waits until
// X is final (the R kernel's flags[0], or the preceding grid), then, while the
// compute warps run the main loop, until R is stored (flags[1]); it copies R
// into shared memory for the epilogue and, as the last CTA to get there,
// returns the flags to zero.  The hand-off latency thus stays off the weight
// stream and out of the epilogue.
// ---------------------------------------------------------------------------
constexpr int kMaxWarps = 11;   // compute warps; with the control warp 12 x 32 x 128 registers
                                // leave room for an R CTA on the SM
// Pipeline stages per warp (one 2-D TMA box of 16 rows x 2 groups of 128,
// 2 KB) are a template parameter S in {4, 8}: the host trades ring depth
// against resident warps.

struct GemvModule {
    const uint32_t* q;
    const __half* s;
    const uint8_t* z;
    const __half* A;   // nullptr: correction off for this module
    __half* Y;
    int64_t ldY;
    int O;
    int tile_begin;    // first 16-row tile of this module in the stacked order
};

struct GemvArgs {
    CUtensorMap tmq[GLOWQ_MAX_MODULES];   // qweight [O][d/8] u32, box {32 words, 16 rows}
    GemvModule mod[GLOWQ_MAX_MODULES];
    int m;
    int d;
    int T;
    int r;
    int num_tiles;
    int rt;            // row tiles per CTA
    int kw;            // in-CTA splits of d
    int kc;            // CTAs per cluster splitting d (kw == 1 when kc > 1)
    const __half* X;   // T x d
    const __half* R;   // T x r (read after the wait)
    unsigned int* flags;    // hand-off words of the R kernel (nullptr: wait for the preceding grid)
    int nflag;              // count each flag reaches (CTAs of the R kernel)
    unsigned int* status;   // device status word (bounded-wait timeouts)
};

struct GemvLayout {    // byte offsets into dynamic shared memory
    int xs, xsum, sz, red, as, rs, rbar, total;
    int wpt_max, ncta_max, nsub_max, fin_slots;
};

// Launch-time constants computed on the host (no divisions in the kernel).
struct GemvPlan {
    GemvLayout L;
    int gsplit[17];    // group boundaries of split j = crank * kw + ks, j in [0, kc * kw] (kc * kw <= 16)
};

__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

__host__ __device__ inline GemvLayout gemv_layout(int T, int d, int r, int rt, int kw, int kc, int nt, int stages) {
    GemvLayout L;
    const int warps = rt * kw;
    const int ngroups = d / 128;
    L.ncta_max = ceil_div(ngroups, kc);
    L.nsub_max = ceil_div(L.ncta_max, kw);
    L.wpt_max = L.ncta_max * 16;
    L.fin_slots = (kc > 1) ? ceil_div(rt, kc) : rt;
    const int nslots = (kc > 1) ? kc * L.fin_slots : (kw > 1 ? kw * rt : 0);
    int off = warps * stages * 2048;          // TMA ring (offset 0, 1024-aligned base)
    off += warps * stages * 8;                // mbarriers
    off = (off + 15) / 16 * 16;
    L.xs = off;
    off += (T + 1) * L.wpt_max * 16;
    L.xsum = off;
    off += L.ncta_max * 2 * 8 * nt * 4;
    off = (off + 15) / 16 * 16;
    L.sz = off;
    off += warps * 16 * (L.nsub_max + 1) * 8;
    L.red = off;
    off += nslots * nt * 4 * 32 * 4;
    L.as = off;
    off += (r > 0) ? L.fin_slots * 16 * (r + 8) * 2 : 0;
    off = (off + 15) / 16 * 16;
    L.rs = off;
    off += (r > 0) ? 8 * nt * (r + 8) * 2 : 0;
    off = (off + 15) / 16 * 16;
    L.rbar = off;
    off += 16;
    L.total = off;
    return L;
}

__device__ __forceinline__ void cp_async16(uint32_t smem_addr, const void* gptr) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr), "l"(gptr) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// D = A * B with a zero accumulator (starts an independent chain)
__device__ __forceinline__ void mma_16816_zc(float c[4], const uint32_t a[4], const uint32_t b[2]) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
        : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]), "f"(0.0f));
}

// One packed word (8 codes, low nibble first) -> four half2 of exact values,
// one shift and four LOP3:
//   ev[0] = 16 + q/64 of codes (0,4)   nibble in mantissa bits 0..3 of 16.0
//   ev[1] = 16 + q/64 of codes (2,6)
//   od[0] = 64 + q    of codes (1,5)   nibble in mantissa bits 4..7 of 64.0
//   od[1] = 64 + q    of codes (3,7)
__device__ __forceinline__ void unpack_even_odd(uint32_t w, uint32_t ev[2], uint32_t od[2]) {
    const uint32_t w8 = w >> 8;
    ev[0] = (w & 0x000F000Fu) | 0x4C004C00u;
    od[0] = (w & 0x00F000F0u) | 0x54005400u;
    ev[1] = (w8 & 0x000F000Fu) | 0x4C004C00u;
    od[1] = (w8 & 0x00F000F0u) | 0x54005400u;
}

template <int NT, int S, bool ONE>
// (the bound of 512 threads caps registers at 128 per thread; launches use at
// most kMaxWarps compute warps and the control warp).  ONE: T == 1, so only the
// first column of each MMA tile (lanes t == 0, elements 0 and 2) is finished.
__global__ void __launch_bounds__(512, 1) corrected_gemv_kernel(const __grid_constant__ GemvArgs args,
                                                                           const __grid_constant__ GemvPlan plan) {
    pdl_launch_dependents();
    extern __shared__ __align__(1024) unsigned char smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // the weight streams' TMA descriptors into the descriptor cache
    if (threadIdx.x < GLOWQ_MAX_MODULES && (int)threadIdx.x < args.m)
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&args.tmq[threadIdx.x])) : "memory");
    const int g = lane >> 2, t = lane & 3;
    const int rt = args.rt, kw = args.kw, kc = args.kc;
    const int warps = rt * kw;
    const int d = args.d, T = args.T, r = args.r;
    const int ngroups = d / 128;
    const GemvLayout& L = plan.L;
    unsigned char* ring = smem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + warps * S * 2048);
    uint4* xs = reinterpret_cast<uint4*>(smem + L.xs);
    float* xsum = reinterpret_cast<float*>(smem + L.xsum);
    float2* szs = reinterpret_cast<float2*>(smem + L.sz);
    float* red = reinterpret_cast<float*>(smem + L.red);
    __half* as = reinterpret_cast<__half*>(smem + L.as);
    __half* rs = reinterpret_cast<__half*>(smem + L.rs);
    uint64_t* rbar = reinterpret_cast<uint64_t*>(smem + L.rbar);
    const bool control = warp == warps;         // the last warp: hand-off with the R kernel

    const int crank = blockIdx.x % kc;          // rank in the cluster (cluster dims (kc,1,1))
    const int block = blockIdx.x / kc;
    const int C0 = plan.gsplit[crank * kw], C1 = plan.gsplit[crank * kw + kw];
    const int ncta = C1 - C0;
    const int wpt = ncta * 16;                  // 8-element words per token in the CTA's slice
    const int tl = warp % rt, ks = warp / rt;   // tile within the CTA, split index
    const int G0 = control ? 0 : plan.gsplit[crank * kw + ks];
    const int G1 = control ? 0 : plan.gsplit[crank * kw + ks + 1];
    const int tile = block * rt + tl;
    const bool active = !control && tile < args.num_tiles;
    // The module of this warp's tile.  Kernel parameters are read through the
    // constant cache, cold at every launch: the lookup reads every module's
    // first tile and scale / zero pointers unconditionally (independent loads,
    // one round of misses) rather than a chain of dependent reads.
    int mi = 0, tb = 0;
    const __half* Ms = args.mod[0].s;
    const uint8_t* Mz = args.mod[0].z;
#pragma unroll
    for (int i = 1; i < GLOWQ_MAX_MODULES; ++i) {
        const int b = args.mod[i].tile_begin;
        const __half* si = args.mod[i].s;
        const uint8_t* zi = args.mod[i].z;
        if (i < args.m && tile >= b) {
            mi = i;
            tb = b;
            Ms = si;
            Mz = zi;
        }
    }
    const GemvModule& M = args.mod[mi];
    const int tile_row = (tile - tb) * 16;
    const int row_lo = tile_row + g, row_hi = row_lo + 8;
    // the warp that finalises this tile: split 0 of the owner CTA of the cluster
    const int owner = (kc > 1) ? tl % kc : 0;
    const int fslot = (kc > 1) ? tl / kc : tl;
    const bool finaliser = !control && ks == 0 && owner == crank;
    const bool has_corr = r > 0 && M.A != nullptr;

    // Prologue order (from per-CTA timelines of back-to-back calls): barriers,
    // scale/zero loads, weight stream, A prefetch, scale/zero staging, then X.
    // 1) the weight stream's ring: per warp, S mbarriers; lane 0 issues one 2-D
    //    TMA box (16 rows x 2 groups) per stage
    constexpr int kStages = S;
    uint64_t* my_bars = bars + warp * kStages;
    unsigned char* my_ring = ring + warp * kStages * 2048;
    const uint32_t ring_smem = smem_u32(my_ring);
    const CUtensorMap* tmq = &args.tmq[mi];
    const int nsub = G1 - G0;
    const int npairs = (nsub + 1) / 2;
    // the barriers are initialised and fenced while this thread has no memory
    // operation outstanding (the release fence would wait for it)
    if (active && lane == 0) {
        for (int i = 0; i < kStages; ++i) mbar_init(my_bars + i, 1);
        fence_mbar_init();
    }
    // 2) this warp's scales and zeros are the longest-latency reads of the
    //    prologue (scattered, cold): a split of at most 32 groups is loaded in
    //    one batch ahead of the weight stream (behind it, they would queue
    //    after every stage in flight), and staged in step 5
    const int sz_stride = L.nsub_max + 1;
    float2* my_sz = szs + warp * 16 * sz_stride;
    const int rr = lane & 15;   // lane -> row (lane & 15) and every other group starting at lane >> 4
    const int64_t sz_base = (int64_t)(tile_row + rr) * ngroups + G0;
    const int nsub0 = G1 - G0;
    const bool one_batch = active && nsub0 <= 32;
    unsigned short sv[16];
    unsigned char zv[16];
    if (one_batch) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int gg = (lane >> 4) + 2 * j;
            if (gg < nsub0) {
                sv[j] = __half_as_ushort(Ms[sz_base + gg]);
                zv[j] = Mz[sz_base + gg];
            }
        }
    }

    // 3) start the weight stream (read once per call: evict-first in L2)
    const uint64_t wpol = l2_policy_evict_first();
    if (active) {
        if (lane == 0) {
            for (int i = 0; i < kStages && i < npairs; ++i) {
                mbar_arrive_expect_tx(my_bars + i, 2048u);
                tma_load_2d_hint(ring_smem + i * 2048, tmq, my_bars + i, (G0 + 2 * i) * 16, tile_row, wpol);
            }
        }
        __syncwarp();
    }
    // 4) the finalising warp prefetches its tile's rows of A
    if (active && has_corr && finaliser) {
        const uint32_t a_base = (uint32_t)__cvta_generic_to_shared(as + fslot * 16 * (r + 8));
        const int cpr = r / 8;   // 16-byte chunks per row
        for (int c = lane; c < 16 * cpr; c += 32) {
            const int rr = c / cpr, cc = c - rr * cpr;
            cp_async16(a_base + (uint32_t)((rr * (r + 8) + cc * 8) * 2), M.A + (int64_t)(tile_row + rr) * r + cc * 8);
        }
    }
    cp_async_commit();

    // 5) stage (s, 64 + z) of the warp's rows x groups [G0, G1); longer splits
    //    load in batches of 16 per lane, all issued before any is used
    if (one_batch) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int gg = (lane >> 4) + 2 * j;
            if (gg < nsub)
                my_sz[rr * sz_stride + gg] = make_float2(__half2float(__ushort_as_half(sv[j])), 64.0f + (float)zv[j]);
        }
    } else if (active) {
        for (int g0 = lane >> 4; g0 < nsub; g0 += 32) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int gg = g0 + 2 * j;
                if (gg < nsub) {
                    sv[j] = __half_as_ushort(Ms[sz_base + gg]);
                    zv[j] = Mz[sz_base + gg];
                }
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int gg = g0 + 2 * j;
                if (gg < nsub)
                    my_sz[rr * sz_stride + gg] = make_float2(__half2float(__ushort_as_half(sv[j])), 64.0f + (float)zv[j]);
            }
        }
    }
    // Everything above reads only static weight data; activations (and R) may
    // be produced by the preceding kernels.  After an R kernel, X is final once
    // every R CTA has passed its own wait (flags[0]), which the control warp
    // awaits meanwhile; R itself is awaited only during the main loop.  Without
    // flags, wait for the preceding grid (a no-op when launched without
    // programmatic serialization).
    if (control && lane == 0) {
        mbar_init(rbar, 1);
        if (args.flags) flag_wait_geq(args.flags + 0, (unsigned)args.nflag, args.status);
    }
    if (!args.flags) pdl_wait();
    __syncthreads();   // X is final; rbar is initialised
    // 6) the CTA's activation slice, paired and swizzled (all loads of a batch
    //    first); every thread of the CTA, the control warp included, takes part
    const int stride = (int)blockDim.x;
    {
        const int items = T * wpt;
        // warp-uniform trip count: every lane reaches the shuffles below
        for (int b0 = (int)threadIdx.x - lane; b0 < items; b0 += 4 * stride) {
            const int base = b0 + lane;
            uint4 v[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int i = base + j * stride;
                if (i < items) {
                    const int tok = i / wpt, wd = i - tok * wpt;
                    v[j] = ldcg_128(args.X + (int64_t)tok * d + (int64_t)C0 * 128 + wd * 8);
                }
            }
            // with each word, its even / odd activation sums; the 16 words of a
            // (token, group) are held by 16 consecutive lanes (stride and wpt
            // are multiples of 16), which add them in a fixed butterfly order
            // into S_E and S_O: xsum[(2 * group + e)][token]
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int i = base + j * stride;
                float se = 0.f, so = 0.f;
                if (i < items) {
                    const int tok = i / wpt, wd = i - tok * wpt;
                    uint4 p;
                    p.x = pair_lo(v[j].x, v[j].z);   // (x0,x4)
                    p.y = pair_lo(v[j].y, v[j].w);   // (x2,x6)
                    p.z = pair_hi(v[j].x, v[j].z);   // (x1,x5)
                    p.w = pair_hi(v[j].y, v[j].w);   // (x3,x7)
                    // swizzle: XOR the two low bits of the word with (bit 3, token parity)
                    xs[tok * wpt + (wd ^ (((wd >> 3) & 1) | ((tok & 1) << 1)))] = p;
                    const float2 f0 = __half22float2(u32_as_h2(p.x)), f2 = __half22float2(u32_as_h2(p.y));
                    const float2 f1 = __half22float2(u32_as_h2(p.z)), f3 = __half22float2(u32_as_h2(p.w));
                    se = (f0.x + f0.y) + (f2.x + f2.y);
                    so = (f1.x + f1.y) + (f3.x + f3.y);
                }
#pragma unroll
                for (int o = 8; o >= 1; o >>= 1) {
                    se += __shfl_xor_sync(0xffffffffu, se, o);
                    so += __shfl_xor_sync(0xffffffffu, so, o);
                }
                if (i < items && (lane & 15) == 0) {
                    const int tok = i / wpt, gc = (i - tok * wpt) >> 4;
                    xsum[(2 * gc) * 8 * NT + tok] = se;
                    xsum[(2 * gc + 1) * 8 * NT + tok] = so;
                }
            }
        }
        for (int i = threadIdx.x; i < wpt; i += stride) xs[T * wpt + i] = make_uint4(0, 0, 0, 0);
        // padding tokens: zero sums
        for (int i = threadIdx.x; i < ncta * (8 * NT - T); i += stride) {
            const int gc = i / (8 * NT - T), tok = T + (i - gc * (8 * NT - T));
            xsum[(2 * gc) * 8 * NT + tok] = 0.f;
            xsum[(2 * gc + 1) * 8 * NT + tok] = 0.f;
        }
    }
    __syncthreads();

    // 7) the control warp: once R is stored, copy it into rs (padding tokens
    //     zero) and complete rbar; the last CTA here zeroes the flags, which the
    //     next call's R kernel writes only after this grid has completed
    if (control && r > 0) {
        if (args.flags && lane == 0) flag_wait_geq(args.flags + 1, (unsigned)args.nflag, args.status);
        __syncwarp();
        const int cpr = r / 8;   // 16-byte chunks per row
        for (int c = lane; c < 8 * NT * cpr; c += 32) {
            const int tok = c / cpr, cc = c - tok * cpr;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (tok < T) v = ldcg_128(args.R + (int64_t)tok * r + cc * 8);
            *reinterpret_cast<uint4*>(rs + tok * (r + 8) + cc * 8) = v;
        }
        __syncwarp();
        if (lane == 0) {
            if (args.flags) {
                unsigned int prev;
                asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(prev) : "l"(args.flags + 2) : "memory");
                if (prev == gridDim.x - 1) {
                    args.flags[0] = 0u;
                    args.flags[1] = 0u;
                    args.flags[2] = 0u;
                }
            }
            mbar_arrive(rbar);
        }
    }

    // 8) main loop: two independent MMA chains per 128-group on (64 + q) x,
    //    then s * (D - (64 + z) S) in fp32
    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[n][i] = 0.f;
    if (active) {
        const float2* sz_lo = my_sz + g * sz_stride;
        const float2* sz_hi = sz_lo + 8 * sz_stride;
        // lanes of padding tokens read the zero row, so every read is unconditional
        const uint4* xrow[NT];
        const int xsw = ((t >> 1) & 1) | ((g & 1) << 1);   // swizzle term of this lane
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            const int tok = (n * 8 + g < T) ? n * 8 + g : T;
            xrow[n] = xs + tok * wpt + (G0 - C0) * 16;
        }
        const float* xsum_w = xsum + (G0 - C0) * 2 * 8 * NT + 2 * t;
        // Running pointers, advanced once per round of kStages stages, so that
        // every shared-memory read inside the unrolled round is base + constant:
        // activation fragment w of token block n, scale/zero pair, group sums.
        const uint4* xw[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int w = 0; w < 4; ++w) xw[n][w] = xrow[n] + ((4 * t + w) ^ xsw);
        const float2* szl = sz_lo;
        const float2* szh = sz_hi;
        const float* xsp = xsum_w;
        // lane (g, t) reads 16 B of rows g and g+8 per group
        const unsigned char* rd_lo = my_ring + g * 128 + t * 16;
        const unsigned char* rd_hi = rd_lo + 8 * 128;
        bool ok = true;
        for (int p0 = 0; p0 < npairs; p0 += kStages,
                 szl += 2 * kStages, szh += 2 * kStages, xsp += 2 * kStages * 2 * 8 * NT) {
#pragma unroll
            for (int i = 0; i < kStages; ++i) {
                const int p = p0 + i;
                if (p < npairs) {
                    if (ok) ok = mbar_wait(my_bars + i, (uint32_t)((p / kStages) & 1), args.status);
                    const unsigned char* sl = rd_lo + i * 2048;
                    const unsigned char* sh = rd_hi + i * 2048;
                    uint4 w4[2][2];
                    w4[0][0] = *reinterpret_cast<const uint4*>(sl);
                    w4[0][1] = *reinterpret_cast<const uint4*>(sh);
                    w4[1][0] = *reinterpret_cast<const uint4*>(sl + 64);
                    w4[1][1] = *reinterpret_cast<const uint4*>(sh + 64);
                    if (p + kStages < npairs) {
                        fence_proxy_async_smem();   // this lane's reads of the slot precede the refill
                        __syncwarp();
                        if (lane == 0) {
                            mbar_arrive_expect_tx(my_bars + i, 2048u);
                            tma_load_2d_hint(ring_smem + i * 2048, tmq, my_bars + i, (G0 + 2 * (p + kStages)) * 16,
                                             tile_row, wpol);
                        }
                    }
                    const bool two = 2 * p + 1 < nsub;    // warp-uniform
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (h == 1 && !two) break;
                        const int gi = 2 * i + h;          // group within this round (a constant)
                        const uint32_t wl[4] = {w4[h][0].x, w4[h][0].y, w4[h][0].z, w4[h][0].w};
                        const uint32_t wh[4] = {w4[h][1].x, w4[h][1].y, w4[h][1].z, w4[h][1].w};
                        // two MMA chains: even k (A = 16 + q/64) and odd k (A = 64 + q)
                        float te[NT][4], to[NT][4];
#pragma unroll
                        for (int w = 0; w < 4; ++w) {
                            uint32_t el[2], ol[2], eh[2], oh[2];
                            unpack_even_odd(wl[w], el, ol);   // row g
                            unpack_even_odd(wh[w], eh, oh);   // row g + 8
                            const uint32_t ae[4] = {el[0], eh[0], el[1], eh[1]};
                            const uint32_t ao[4] = {ol[0], oh[0], ol[1], oh[1]};
#pragma unroll
                            for (int n = 0; n < NT; ++n) {
                                const uint4 x = xw[n][w][gi * 16];
                                const uint32_t be[2] = {x.x, x.y};   // (x0,x4) (x2,x6)
                                const uint32_t bo[2] = {x.z, x.w};   // (x1,x5) (x3,x7)
                                if (w == 0) {
                                    mma_16816_zc(te[n], ae, be);
                                    mma_16816_zc(to[n], ao, bo);
                                } else {
                                    mma_16816(te[n], ae, be);
                                    mma_16816(to[n], ao, bo);
                                }
                            }
                        }
                        // sum_k (q - z) x = 64 D_E + D_O - (1024 + z) S_E - (64 + z) S_O, times s
                        const float2 zl = szl[gi], zh = szh[gi];   // (s, 64 + z)
                        const float cel = zl.y + 960.0f, ceh = zh.y + 960.0f;
#pragma unroll
                        for (int n = 0; n < NT; ++n) {
                            const float2 se = *reinterpret_cast<const float2*>(xsp + (2 * gi) * 8 * NT + n * 8);
                            const float2 so = *reinterpret_cast<const float2*>(xsp + (2 * gi + 1) * 8 * NT + n * 8);
                            if (ONE) {
                                float v0 = fmaf(64.0f, te[n][0], to[n][0]);
                                float v2 = fmaf(64.0f, te[n][2], to[n][2]);
                                v0 = fmaf(-zl.y, so.x, fmaf(-cel, se.x, v0));
                                v2 = fmaf(-zh.y, so.x, fmaf(-ceh, se.x, v2));
                                acc[n][0] = fmaf(zl.x, v0, acc[n][0]);
                                acc[n][2] = fmaf(zh.x, v2, acc[n][2]);
                                continue;
                            }
                            float v0 = fmaf(64.0f, te[n][0], to[n][0]);
                            float v1 = fmaf(64.0f, te[n][1], to[n][1]);
                            float v2 = fmaf(64.0f, te[n][2], to[n][2]);
                            float v3 = fmaf(64.0f, te[n][3], to[n][3]);
                            v0 = fmaf(-zl.y, so.x, fmaf(-cel, se.x, v0));
                            v1 = fmaf(-zl.y, so.y, fmaf(-cel, se.y, v1));
                            v2 = fmaf(-zh.y, so.x, fmaf(-ceh, se.x, v2));
                            v3 = fmaf(-zh.y, so.y, fmaf(-ceh, se.y, v3));
                            acc[n][0] = fmaf(zl.x, v0, acc[n][0]);
                            acc[n][1] = fmaf(zl.x, v1, acc[n][1]);
                            acc[n][2] = fmaf(zh.x, v2, acc[n][2]);
                            acc[n][3] = fmaf(zh.x, v3, acc[n][3]);
                        }
                    }
                }
            }
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int w = 0; w < 4; ++w) xw[n][w] += 2 * kStages * 16;
        }
    }
    cp_async_wait<0>();
    __syncwarp();   // A rows copied by other lanes of this warp are visible


    // 9) split-d reduction in a fixed order, into the finalising warp
    if (kc > 1) {
        // cluster: partials of tile tl go to rank tl % kc, slot [crank][tl / kc]
        const int idx0 = (crank * L.fin_slots + fslot) * NT * 4 * 32 + lane;
        if (control) {
            // no partial sums; only the cluster barrier below
        } else if (owner != crank) {
            const uint32_t local = (uint32_t)__cvta_generic_to_shared(red);
            uint32_t remote;
            asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(owner));
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(remote + (uint32_t)(idx0 + (n * 4 + i) * 32) * 4u),
                                 "f"(acc[n][i])
                                 : "memory");
        } else {
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int i = 0; i < 4; ++i) red[idx0 + (n * 4 + i) * 32] = acc[n][i];
        }
        asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
        if (!finaliser) return;
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float v = 0.f;
                for (int c = 0; c < kc; ++c) v += red[((c * L.fin_slots + fslot) * NT * 4 + n * 4 + i) * 32 + lane];
                acc[n][i] = v;
            }
    } else if (kw > 1) {
        // in-CTA: partials of tile tl from split ks at slot [ks][tl]
        if (!control) {
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int i = 0; i < 4; ++i) red[((ks * rt + tl) * NT * 4 + n * 4 + i) * 32 + lane] = acc[n][i];
        }
        __syncthreads();
        if (!finaliser) return;
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float v = 0.f;
                for (int k2 = 0; k2 < kw; ++k2) v += red[((k2 * rt + tl) * NT * 4 + n * 4 + i) * 32 + lane];
                acc[n][i] = v;
            }
    }
    if (!active) return;

    // 10) rank-r correction A_i R^T, accumulated into the same fp32 registers
    //     (R from shared memory, staged by the control warp)
    if (has_corr) {
        mbar_wait(rbar, 0u, args.status);
        const __half* a_lo = as + (fslot * 16 + g) * (r + 8);
        const __half* a_hi = a_lo + 8 * (r + 8);
        for (int kb = 0; kb < r; kb += 16) {
            const int k = kb + 4 * t;
            const bool kval = k < r;   // r % 8 == 0: 4-element chunks are all-or-nothing
            uint2 al = make_uint2(0, 0), ah = make_uint2(0, 0);
            if (kval) {
                al = *reinterpret_cast<const uint2*>(a_lo + k);
                ah = *reinterpret_cast<const uint2*>(a_hi + k);
            }
            const uint32_t a[4] = {al.x, ah.x, al.y, ah.y};
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const int tok = n * 8 + g;   // rows of padding tokens are zero in rs
                uint2 rv = make_uint2(0, 0);
                if (kval) rv = *reinterpret_cast<const uint2*>(rs + tok * (r + 8) + k);
                const uint32_t b[2] = {rv.x, rv.y};
                mma_16816(acc[n], a, b);
            }
        }
    }

    // 11) fp16 outputs (round to nearest even)
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        const int tk = n * 8 + 2 * t;
        if (tk < T) {
            M.Y[(int64_t)tk * M.ldY + row_lo] = __float2half_rn(acc[n][0]);
            M.Y[(int64_t)tk * M.ldY + row_hi] = __float2half_rn(acc[n][2]);
        }
        if (tk + 1 < T) {
            M.Y[(int64_t)(tk + 1) * M.ldY + row_lo] = __float2half_rn(acc[n][1]);
            M.Y[(int64_t)(tk + 1) * M.ldY + row_hi] = __float2half_rn(acc[n][3]);
        }
    }
}

// ---------------------------------------------------------------------------
// Host-side launchers (called from api.cu after validation).
// ---------------------------------------------------------------------------
static cudaError_t launch_ex(const void* fn, dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                             void** args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelExC(&cfg, fn, args);
}

// R = X B^T into R (fp16) with one cluster of kRcCtas CTAs.
cudaError_t launch_rproj_decode(const uint16_t* X, const uint16_t* B, int T, int d, int r, uint16_t* R,
                                unsigned int* flags, cudaStream_t st) {
    const int nt = (T <= 8) ? 1 : 2;
    const __half* Xh = reinterpret_cast<const __half*>(X);
    const __half* Bh = reinterpret_cast<const __half*>(B);
    __half* Rh = reinterpret_cast<__half*>(R);
    unsigned int* status = device_status_ptr();
    void* a1[] = {(void*)&Xh, (void*)&Bh, (void*)&T, (void*)&d, (void*)&r, (void*)&Rh, (void*)&flags, (void*)&status};
    const void* fn = (nt == 1) ? (const void*)rproj_cluster_kernel<1> : (const void*)rproj_cluster_kernel<2>;
    const size_t smem = (size_t)rc_smem_bytes(r, d, nt);
    // opt in to the largest dynamic shared memory requested so far (at most
    // the staged B slice, the partials of r <= 256 and a 16-token X slice)
    static size_t opted[2] = {48 * 1024, 48 * 1024};
    if (smem > opted[nt - 1]) {
        cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        opted[nt - 1] = smem;
    }
    return launch_ex(fn, dim3(kRcCtas), dim3(kRcWarps * 32), smem, st, true, a1);
}


// Resident CTAs of one variant and shape (cached: the occupancy query is not free).
static int resident_ctas(const void* fn, int warps, int kc, size_t smem, int num_sms) {
    struct Entry { const void* fn; int warps, kc; size_t smem; int n; };
    static Entry cache[256];
    static int used = 0;
    for (int i = 0; i < used; ++i)
        if (cache[i].fn == fn && cache[i].warps == warps && cache[i].kc == kc && cache[i].smem == smem)
            return cache[i].n;
    int n = 0;
    if (kc == 1) {
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, warps * 32, smem) == cudaSuccess)
            n = per_sm * num_sms;
    } else {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(kc);
        cfg.blockDim = dim3(warps * 32);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = kc;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, fn, &cfg) == cudaSuccess) n = clusters * kc;
    }
    (void)cudaGetLastError();
    if (used < 256) cache[used++] = {fn, warps, kc, smem, n};
    return n;
}

struct GemvShape { int rt, kw, kc, stages; size_t smem; };

// one: T == 1 (a single token: only one output column is finished)
static const void* gemv_fn(int nt, int stages, bool one = false) {
    if (nt == 1) {
        if (one)
            return stages == 8 ? (const void*)corrected_gemv_kernel<1, 8, true>
                               : (const void*)corrected_gemv_kernel<1, 4, true>;
        return stages == 8 ? (const void*)corrected_gemv_kernel<1, 8, false> : (const void*)corrected_gemv_kernel<1, 4, false>;
    }
    return stages == 8 ? (const void*)corrected_gemv_kernel<2, 8, false> : (const void*)corrected_gemv_kernel<2, 4, false>;
}

// Pick (rt, kw, kc, stages): all CTAs resident in one wave; then as many SMs
// busy as possible; then as many resident warps per SM as possible (up to 16);
// then as many weight bytes in flight per SM as possible (up to 128 KB); then
// the fewest splits of d.  If nothing fits in one wave, the fewest waves.
static GemvShape choose_shape(int tiles, int d, int T, int r, int nt, int num_sms) {
    struct Key { int tiles, d, T, r, nt; GemvShape s; };
    static Key memo[128];
    static int used = 0;
    for (int i = 0; i < used; ++i)
        if (memo[i].tiles == tiles && memo[i].d == d && memo[i].T == T && memo[i].r == r && memo[i].nt == nt)
            return memo[i].s;
    const int ngroups = d / 128;
    GemvShape best = {0, 0, 0, 0, 0};
    double best_key[5] = {1e30, 1e30, 1e30, 1e30, 1e30};
    // Cost model: the busiest SM sets the time.  CTAs of a cluster launch are
    // packed onto SMs up to their residency (observed: two 8-warp CTAs per SM
    // while other SMs idle), other launches are spread; the busiest SM's load
    // is its CTAs x row tiles x 128-groups per CTA.  Ties prefer more warps on
    // that SM (latency hiding), more bytes in flight, then fewer splits.
    // A shape may also request more shared memory than it uses (kSpreadSmem),
    // which leaves room for one CTA per SM: the launch is then spread.
    constexpr size_t kSpreadSmem = 116 * 1024;
    for (int pad = 0; pad <= 1; ++pad)
    for (int stages = 4; stages <= 8; stages *= 2)
        for (int rt = 1; rt <= kMaxWarps; ++rt)
            for (int kw = 1; rt * kw <= kMaxWarps; ++kw)
                for (int kc = 1; kc <= 8; ++kc) {
                    if (kc > 1 && kw > 1) break;
                    if (kc > ngroups || ngroups / kc < kw) continue;
                    const int warps = rt * kw;   // compute warps (+1 control warp per CTA)
                    const GemvLayout L = gemv_layout(T, d, r, rt, kw, kc, nt, stages);
                    if (L.total > 220 * 1024) continue;
                    if (pad && (size_t)L.total >= kSpreadSmem) continue;
                    const size_t smem = pad ? kSpreadSmem : (size_t)L.total;
                    const void* fn = gemv_fn(nt, stages);
                    const int res = resident_ctas(fn, warps + 1, kc, smem, num_sms);
                    if (res <= 0) continue;
                    const long ctas = (long)ceil_div(tiles, rt) * kc;
                    const double waves = (double)ctas / res;
                    const int res_sm = res / num_sms > 0 ? res / num_sms : 1;
                    long per_sm = (kc > 1) ? (ctas < res_sm ? ctas : res_sm) : (long)ceil_div((int)ctas, num_sms);
                    if (per_sm > res_sm) per_sm = res_sm;
                    const double load = (double)per_sm * rt * ceil_div(ngroups, kc);
                    const double warps_sm = (double)per_sm * warps;
                    const int groups_warp = ceil_div(ceil_div(ngroups, kc), kw);
                    const double inflight_sm = 1024.0 * (groups_warp < 2 * stages ? groups_warp : 2 * stages) * warps_sm;
                    double key[5];
                    key[0] = waves <= 1.0 ? 0.0 : waves;
                    key[1] = load;
                    key[2] = -(warps_sm < 16.0 ? warps_sm : 16.0);
                    key[3] = -(inflight_sm < 131072.0 ? inflight_sm : 131072.0);
                    key[4] = kw * kc + 0.1 * stages - 0.01 * rt + 0.001 * pad;
                    bool better = false;
                    for (int j = 0; j < 5; ++j) {
                        if (key[j] < best_key[j] - 1e-9) { better = true; break; }
                        if (key[j] > best_key[j] + 1e-9) break;
                    }
                    if (better) {
                        for (int j = 0; j < 5; ++j) best_key[j] = key[j];
                        best = {rt, kw, kc, stages, smem};
                    }
                }
    if (used < 128 && best.rt > 0) memo[used++] = {tiles, d, T, r, nt, best};
    if (std::getenv("GLOWQ_VERBOSE"))
        std::fprintf(stderr,
                     "glowq decode shape: tiles=%d d=%d T=%d r=%d -> rt=%d kw=%d kc=%d stages=%d smem=%zu ctas=%d\n",
                     tiles, d, T, r, best.rt, best.kw, best.kc, best.stages, best.smem,
                     best.rt ? ceil_div(tiles, best.rt) * best.kc : 0);
    return best;
}

cudaError_t launch_gemv_decode(const ModuleView* mods, int m, int d, int T, int r, const uint16_t* X,
                               const uint16_t* R, unsigned int* flags, int num_sms, cudaStream_t st) {
    GemvArgs a = {};
    int tiles = 0;
    for (int i = 0; i < m; ++i) {
        a.mod[i].q = mods[i].q;
        a.mod[i].s = reinterpret_cast<const __half*>(mods[i].s);
        a.mod[i].z = mods[i].z;
        a.mod[i].A = (r > 0) ? reinterpret_cast<const __half*>(mods[i].A) : nullptr;
        a.mod[i].Y = reinterpret_cast<__half*>(mods[i].Y);
        a.mod[i].ldY = mods[i].ldY;
        a.mod[i].O = (int)mods[i].O;
        a.mod[i].tile_begin = tiles;
        tiles += (int)(mods[i].O / 16);
        if (!make_map(&a.tmq[i], CU_TENSOR_MAP_DATA_TYPE_UINT32, mods[i].q, (uint64_t)(d / 8), (uint64_t)mods[i].O,
                      (uint64_t)d / 2, 32, 16, CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
    }
    if (tiles == 0) return cudaSuccess;
    const int nt = (T <= 8) ? 1 : 2;
    static bool opted = false;
    if (!opted) {
        for (int n = 1; n <= 2; ++n)
            for (int sg = 4; sg <= 8; sg *= 2)
                for (int one = 0; one <= (n == 1 ? 1 : 0); ++one) {
                    cudaError_t e = cudaFuncSetAttribute(gemv_fn(n, sg, one != 0),
                                                         cudaFuncAttributeMaxDynamicSharedMemorySize, 220 * 1024);
                    if (e != cudaSuccess) return e;
                }
        opted = true;
    }
    GemvShape sh = choose_shape(tiles, d, T, r, nt, num_sms);
    // Tuning override: GLOWQ_DECODE_SHAPE="rt,kw,kc,stages" (validated here).
    if (const char* env = std::getenv("GLOWQ_DECODE_SHAPE")) {
        int v[4] = {0, 0, 0, 0};
        if (std::sscanf(env, "%d,%d,%d,%d", &v[0], &v[1], &v[2], &v[3]) == 4 && v[0] >= 1 && v[1] >= 1 &&
            v[2] >= 1 && v[2] <= 8 && v[0] * v[1] <= kMaxWarps && (v[2] == 1 || v[1] == 1) &&
            (v[3] == 4 || v[3] == 8) && v[2] <= d / 128 && (d / 128) / v[2] >= v[1]) {
            const GemvLayout L = gemv_layout(T, d, r, v[0], v[1], v[2], nt, v[3]);
            if (L.total <= 220 * 1024) sh = {v[0], v[1], v[2], v[3], (size_t)L.total};
        }
    }
    if (sh.rt == 0) return cudaErrorInvalidValue;
    GemvPlan plan = {};
    plan.L = gemv_layout(T, d, r, sh.rt, sh.kw, sh.kc, nt, sh.stages);
    const int ngroups = d / 128;
    for (int c = 0; c < sh.kc; ++c) {
        const int c0 = c * ngroups / sh.kc, c1 = (c + 1) * ngroups / sh.kc;
        for (int k = 0; k <= sh.kw; ++k) plan.gsplit[c * sh.kw + k] = c0 + k * (c1 - c0) / sh.kw;
    }
    a.m = m;
    a.d = d;
    a.T = T;
    a.r = r;
    a.num_tiles = tiles;
    a.rt = sh.rt;
    a.kw = sh.kw;
    a.kc = sh.kc;
    a.flags = (r > 0) ? flags : nullptr;
    a.nflag = kRcCtas;
    a.X = reinterpret_cast<const __half*>(X);
    a.R = reinterpret_cast<const __half*>(R);
    a.status = device_status_ptr();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ceil_div(tiles, sh.rt) * sh.kc);
    cfg.blockDim = dim3((sh.rt * sh.kw + 1) * 32);   // compute warps + the control warp
    cfg.dynamicSmemBytes = sh.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int na = 0;
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = sh.kc;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
    // always programmatic: the weight stream starts while the preceding kernel finishes
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    cfg.attrs = attr;
    cfg.numAttrs = na;
    void* args[] = {(void*)&a, (void*)&plan};
    return cudaLaunchKernelExC(&cfg, gemv_fn(nt, sh.stages, T == 1), args);
}

}  // namespace glowq
