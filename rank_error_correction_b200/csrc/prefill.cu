// prefill.cu -- large-T path of the GlowQ corrected linear layer on the
// 5th-generation tensor cores (tcgen05, accumulators in TMEM, operands staged
// by TMA).
//
// GlowQ pages, papernotes.org summary, key design 4: R = X B_shared^T once per
// input-sharing group, then y_i = W_i^(q) X + A_i R for every module; solo
// modules compute their own R inline.
//
// Two kernels, chained with programmatic dependent launch:
//   rproj_tc_kernel        R = X B^T (T x r), M = 128 tokens per CTA, N = r,
//                          both operands fp16 by TMA, fp32 TMEM accumulator,
//                          rounded to fp16.
//   corrected_gemm_kernel  one 128-row x 256-token tile of y per CTA:
//                          D[o][t] = sum_k w_hat[o][k] X[t][k] + sum_j A[o][j] R[t][j]
//                          - a producer warp streams X tiles (SW128) and packed
//                            INT4 tiles with TMA into a 4-stage ring;
//                          - four transform warps dequantise each INT4 tile to
//                            the exact fp16 w_hat = fp16((q - z) s) straight into
//                            the canonical K-major 128B-swizzled layout the MMA
//                            reads;
//                          - one thread issues tcgen05.mma (M=128, N=256, K=16)
//                            into a 256-column fp32 TMEM accumulator;
//                          - the rank-r correction is one more K=64 slab of the
//                            same accumulator, A_i and R tiles fetched by TMA
//                            (zero-filled beyond r), so no separate kernel or
//                            extra pass over y runs;
//                          - the transform warps then drain TMEM (tcgen05.ld)
//                            and store y in fp16.
// Every wait on an mbarrier is bounded; a wait that runs out records
// GLOWQ_ERR_TIMEOUT in the device status word.
#include <cuda.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "internal.cuh"

namespace glowq {

// ---------------------------------------------------------------------------
// tcgen05 / TMA device helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Shared-memory matrix descriptor: K-major operand in the canonical 128-byte
// swizzled layout (rows of 128 B, 8-row atoms of 1024 B, atoms 1024 B apart).
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t smem_addr) {
    uint64_t desc = 0;
    desc |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);          // start address (16-byte units)
    desc |= (uint64_t)1u << 16;                              // leading byte offset (unused for SW128 K-major)
    desc |= (uint64_t)(1024u >> 4) << 32;                    // stride byte offset: 8-row atoms 1024 B apart
    desc |= (uint64_t)1u << 46;                              // descriptor version for sm_100
    desc |= (uint64_t)2u << 61;                              // layout: 128-byte swizzle
    return desc;
}

// Instruction descriptor, kind::f16: fp16 A and B, fp32 accumulator, both
// operands K-major, shape M x N.
__host__ __device__ constexpr uint32_t f16_idesc(int M, int N) {
    return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` once all previously issued tcgen05.mma of this thread complete.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 2-D tiled TMA store (shared -> global), bulk-group completion.
__device__ __forceinline__ void tma_store_2d(const void* map, uint32_t src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(src), "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void named_barrier_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------
// Corrected GEMM: persistent, one CTA per SM, 128 x 256 output tiles taken
// round-robin; the fp32 accumulator is double-buffered in TMEM (2 x 256
// columns) so the epilogue of one tile overlaps the main loop of the next.
// Warp roles (448 threads):
//   warp 0       TMA producer (X tiles, INT4 tiles; A_i / R tiles of the slab)
//   warp 1       TMEM allocation; one thread issues tcgen05.mma
//   warps 2-9    transform: INT4 tile -> exact fp16 w_hat (SW128 K-major);
//                two threads per row, each half of the k-block
//   warps 10-13  epilogue: TMEM -> fp16 y
// ---------------------------------------------------------------------------
constexpr int kBM = 128;          // output rows per tile (TMEM lanes)
constexpr int kBN = 256;          // tokens per tile (TMEM columns)
constexpr int kBK = 64;           // k per stage: one 128-byte swizzle atom of fp16
constexpr int kGemmStages = 4;
constexpr int kXBytes = kBN * kBK * 2;       // 32 KB
constexpr int kWBytes = kBM * kBK * 2;       // 16 KB
constexpr int kQBytes = kBM * (kBK / 8) * 4; // 4 KB packed codes (32B-swizzled rows)
constexpr int kStageBytesG = kXBytes + kWBytes + kQBytes;   // multiple of 1024
constexpr int kGemmThreads = 448;            // 14 warps
constexpr int kTransformThreads = 256;
constexpr int kAccCols = 2 * kBN;            // double-buffered accumulator
constexpr int kEpiChunk = 32;                // tokens per epilogue chunk (TMEM columns)
constexpr int kEpiBytes = kEpiChunk * kBM * 2;   // 8 KB: [32 tokens][128 rows] fp16

struct PrefillModule {
    const __half* s;
    const uint8_t* z;
    __half* Y;
    int64_t ldY;
    int O;
    int mtile_begin;
    int has_A;
};

struct PrefillArgs {
    CUtensorMap tmX;                       // X [T][d] fp16, box {64, 256}, SW128
    CUtensorMap tmR;                       // R [T][r] fp16, box {64, 256}, SW128
    CUtensorMap tmQ[GLOWQ_MAX_MODULES];    // qweight [O][d/8] u32, box {8, 128}, SW32
    CUtensorMap tmA[GLOWQ_MAX_MODULES];    // A [O][r] fp16, box {64, 128}, SW128
    CUtensorMap tmY[GLOWQ_MAX_MODULES];    // Y [T][ldY] fp16 (O columns), box {128, 32} (TMA store)
    PrefillModule mod[GLOWQ_MAX_MODULES];
    int m;
    int d;
    int T;
    int r;
    int ntiles_n;                          // token tiles
    int ntiles;                            // all tiles
    int wait_dep;                          // R comes from the preceding (PDL) kernel
    unsigned int* status;
};

struct __align__(8) GemmBarriers {
    uint64_t full[kGemmStages];    // TMA bytes landed (expect_tx by the producer)
    uint64_t dq[kGemmStages];      // transform warps wrote w_hat (256 arrivals)
    uint64_t empty[kGemmStages];   // MMAs reading the stage completed (tcgen05.commit)
    uint64_t acc_full[2];          // accumulator buffer complete (tcgen05.commit)
    uint64_t acc_empty[2];         // accumulator buffer drained (128 epilogue arrivals)
    uint32_t tmem_base;
};

struct TileCoord {
    int mi, m0, n0, nslab;
};

__device__ __forceinline__ TileCoord tile_coord(const PrefillArgs& args, int tile) {
    TileCoord c;
    const int mt = tile / args.ntiles_n;
    const int nt = tile - mt * args.ntiles_n;
    int mi = 0;
    for (int i = 1; i < args.m; ++i)
        if (mt >= args.mod[i].mtile_begin) mi = i;
    c.mi = mi;
    c.m0 = (mt - args.mod[mi].mtile_begin) * kBM;
    c.n0 = nt * kBN;
    c.nslab = (args.r > 0 && args.mod[mi].has_A) ? (args.r + kBK - 1) / kBK : 0;
    return c;
}

__global__ void __launch_bounds__(kGemmThreads, 1) corrected_gemm_kernel(const __grid_constant__ PrefillArgs args) {
    extern __shared__ __align__(1024) unsigned char gsm_raw[];
    // 1024-byte alignment of the stage buffers (swizzle atoms)
    unsigned char* gsm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(gsm_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* epi = gsm + kGemmStages * kStageBytesG;            // 2 x kEpiBytes
    GemmBarriers* bars = reinterpret_cast<GemmBarriers*>(epi + 2 * kEpiBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nkb = args.d / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGemmStages; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->dq[s], kTransformThreads);
            mbar_init(&bars->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->acc_full[b], 1);
            mbar_init(&bars->acc_empty[b], 128);
        }
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&bars->tmem_base, kAccCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    pdl_launch_dependents();

    if (warp == 0) {
        // ---------------- producer ----------------
        if (lane == 0) {
            bool ok = true, waited = false;
            int g = 0;   // global k-block counter of this CTA (ring position)
            for (int tile = blockIdx.x; tile < args.ntiles; tile += gridDim.x) {
                const TileCoord c = tile_coord(args, tile);
                const int nblocks = nkb + c.nslab;
                for (int i = 0; i < nblocks; ++i, ++g) {
                    const int s = g % kGemmStages;
                    if (g >= kGemmStages && ok) ok = mbar_wait(&bars->empty[s], ((g / kGemmStages) - 1) & 1, args.status);
                    unsigned char* st = gsm + s * kStageBytesG;
                    const uint32_t xs = smem_u32(st), ws = smem_u32(st + kXBytes), qs = smem_u32(st + kXBytes + kWBytes);
                    if (i < nkb) {
                        mbar_arrive_expect_tx(&bars->full[s], kXBytes + kQBytes);
                        tma_load_2d(xs, &args.tmX, &bars->full[s], i * kBK, c.n0);
                        tma_load_2d(qs, &args.tmQ[c.mi], &bars->full[s], i * (kBK / 8), c.m0);
                    } else {
                        if (!waited && args.wait_dep) {   // R is complete
                            pdl_wait();
                            waited = true;
                        }
                        const int j = i - nkb;
                        mbar_arrive_expect_tx(&bars->full[s], kXBytes + kWBytes);
                        tma_load_2d(xs, &args.tmR, &bars->full[s], j * kBK, c.n0);
                        tma_load_2d(ws, &args.tmA[c.mi], &bars->full[s], j * kBK, c.m0);
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t idesc = f16_idesc(kBM, kBN);
            bool ok = true;
            int g = 0, tl = 0;
            for (int tile = blockIdx.x; tile < args.ntiles; tile += gridDim.x, ++tl) {
                const TileCoord c = tile_coord(args, tile);
                const int nblocks = nkb + c.nslab;
                const int buf = tl & 1;
                if (tl >= 2 && ok) ok = mbar_wait(&bars->acc_empty[buf], ((tl >> 1) - 1) & 1, args.status);
                tc_fence_after();
                const uint32_t dacc = tmem + (uint32_t)(buf * kBN);
                for (int i = 0; i < nblocks; ++i, ++g) {
                    const int s = g % kGemmStages;
                    const uint32_t par = (g / kGemmStages) & 1;
                    // dq completes once per block (slab blocks too, after their TMA landed)
                    if (ok) ok = mbar_wait(&bars->dq[s], par, args.status);
                    tc_fence_after();
                    unsigned char* st = gsm + s * kStageBytesG;
                    const uint32_t xs = smem_u32(st), ws = smem_u32(st + kXBytes);
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k) {
                        const uint64_t ad = sw128_kmajor_desc(ws + k * 32);
                        const uint64_t bd = sw128_kmajor_desc(xs + k * 32);
                        umma_f16(dacc, ad, bd, idesc, (i > 0 || k > 0) ? 1u : 0u);
                    }
                    umma_commit(&bars->empty[s]);   // frees the stage once these MMAs complete
                }
                umma_commit(&bars->acc_full[buf]);  // this tile's accumulator is complete
            }
        }
    } else if (warp < 10) {
        // ---------------- transform (warps 2..9) ----------------
        const int tt = threadIdx.x - 64;
        const int row = tt & 127;                      // tile row owned by this thread
        const int half = tt >> 7;                      // which 32 k of the 64-k block
        const int ngroups = args.d / 128;
        const uint32_t swz = (uint32_t)(row & 7);
        bool ok = true;
        int g = 0;
        // scale/zero of the current and the next 3 groups (a shift register
        // refilled 4 groups ahead, across tile boundaries)
        int cur_tile = blockIdx.x;
        TileCoord cc = tile_coord(args, cur_tile < args.ntiles ? cur_tile : 0);
        int f_tile = cur_tile, f_grp = 0;              // next group to fetch
        TileCoord fc = cc;
        auto fetch = [&]() -> uint32_t {
            uint32_t v = 0;
            if (f_tile < args.ntiles) {
                const int orow = fc.m0 + row;
                const PrefillModule& FM = args.mod[fc.mi];
                if (orow < FM.O) {
                    const int64_t o = (int64_t)orow * ngroups + f_grp;
                    v = (uint32_t)__half_as_ushort(FM.s[o]) | ((uint32_t)FM.z[o] << 16);
                }
                if (++f_grp == ngroups) {
                    f_grp = 0;
                    f_tile += gridDim.x;
                    if (f_tile < args.ntiles) fc = tile_coord(args, f_tile);
                }
            }
            return v;
        };
        uint32_t sz0 = fetch(), sz1 = fetch(), sz2 = fetch(), sz3 = fetch();
        for (; cur_tile < args.ntiles; cur_tile += gridDim.x) {
            cc = tile_coord(args, cur_tile);
            const int nblocks = nkb + cc.nslab;
            for (int i = 0; i < nkb; ++i, ++g) {
                const int s = g % kGemmStages;
                if (ok) ok = mbar_wait(&bars->full[s], (g / kGemmStages) & 1, args.status);
                unsigned char* st = gsm + s * kStageBytesG;
                // 32-byte-swizzled INT4 rows: 16-byte half h of row r sits at r*32 + ((h ^ (r>>2)&1) << 4)
                const unsigned char* qrow = st + kXBytes + kWBytes + row * 32;
                const uint32_t hsw = (uint32_t)((row >> 2) & 1);
                const uint4 q0 = *reinterpret_cast<const uint4*>(qrow + (((uint32_t)half ^ hsw) << 4));
                const uint32_t sz = sz0;                             // group i/2
                if ((i & 1) == 1) {                                  // group done: shift, fetch 4 ahead
                    sz0 = sz1;
                    sz1 = sz2;
                    sz2 = sz3;
                    sz3 = fetch();
                }
                const __half2 sc = __half2half2(__ushort_as_half((unsigned short)(sz & 0xffffu)));
                const __half2 bz = __half2half2(__ushort_as_half((unsigned short)(0x6400u | ((sz >> 16) & 0xffu))));
                const uint32_t words[4] = {q0.x, q0.y, q0.z, q0.w};
                // row `row` of the W tile: 8 chunks of 16 B (8 fp16 in k order), chunk c at c ^ (row % 8)
                unsigned char* wrow = st + kXBytes + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int c = half * 4 + j;
                    __half2 p[4];
                    dequant_word(words[j], bz, sc, p);   // pairs (0,4) (1,5) (2,6) (3,7), exact w_hat
                    const uint32_t u0 = h2_as_u32(p[0]), u1 = h2_as_u32(p[1]), u2 = h2_as_u32(p[2]), u3 = h2_as_u32(p[3]);
                    uint4 o;
                    o.x = pair_lo(u0, u1);   // (0,1)
                    o.y = pair_lo(u2, u3);   // (2,3)
                    o.z = pair_hi(u0, u1);   // (4,5)
                    o.w = pair_hi(u2, u3);   // (6,7)
                    *reinterpret_cast<uint4*>(wrow + (((uint32_t)c ^ swz) << 4)) = o;
                }
                fence_proxy_async_smem();   // generic-proxy writes visible to the tensor cores
                mbar_arrive(&bars->dq[s]);
            }
            // slab blocks are filled by TMA alone; still advance dq once per block
            // (after the TMA landed) so its phases follow the ring position
            for (int i = nkb; i < nblocks; ++i, ++g) {
                const int s = g % kGemmStages;
                if (ok) ok = mbar_wait(&bars->full[s], (g / kGemmStages) & 1, args.status);
                mbar_arrive(&bars->dq[s]);
            }
        }
    } else {
        // ---------------- epilogue (warps 10..13) ----------------
        // Each 32-token chunk of the accumulator is transposed through shared
        // memory ([32 tokens][128 rows] fp16) and written by one TMA store,
        // which clips rows >= O and tokens >= T.  Two staging buffers: a buffer
        // is rewritten only after the store issued from it two chunks earlier
        // has finished reading it.
        const int quarter = warp & 3;                  // TMEM lanes 32*quarter .. +31
        const int row = quarter * 32 + lane;
        const bool leader = (warp == 10 && lane == 0);
        bool ok = true;
        int tl = 0, chunk = 0;
        for (int tile = blockIdx.x; tile < args.ntiles; tile += gridDim.x, ++tl) {
            const TileCoord c = tile_coord(args, tile);
            const int buf = tl & 1;
            if (ok) ok = mbar_wait(&bars->acc_full[buf], (tl >> 1) & 1, args.status);
            tc_fence_after();
            const uint32_t tacc = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * kBN);
#pragma unroll 1
            for (int ch = 0; ch < kBN / kEpiChunk; ++ch, ++chunk) {
                uint32_t v[32];
                tmem_ld32(tacc + ch * kEpiChunk, v);
                unsigned char* sb = epi + (chunk & 1) * kEpiBytes;
                if (leader) bulk_wait_read<1>();          // the store from this buffer is done reading
                named_barrier_sync(1, 128);
                __half* col = reinterpret_cast<__half*>(sb) + row;
#pragma unroll
                for (int j = 0; j < 32; ++j) col[j * kBM] = __float2half_rn(__uint_as_float(v[j]));
                fence_proxy_async_smem();
                named_barrier_sync(1, 128);
                if (leader) {
                    tma_store_2d(&args.tmY[c.mi], smem_u32(sb), c.m0, c.n0 + ch * kEpiChunk);
                    bulk_commit();
                }
            }
            tc_fence_before();
            mbar_arrive(&bars->acc_empty[buf]);        // buffer may be overwritten
        }
        if (leader) bulk_wait_all();
    }
    // the R kernel is complete before this grid is (even if no tile read R)
    if (args.wait_dep) pdl_wait();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, kAccCols);
}

// ---------------------------------------------------------------------------
// R = X B^T on the tensor cores: one 128-token tile per CTA, N = r (padded to 16)
// ---------------------------------------------------------------------------
constexpr int kRStages = 4;
constexpr int kRThreads = 192;

struct RprojArgs {
    CUtensorMap tmX;   // X [T][d], box {64, 128}, SW128
    CUtensorMap tmB;   // B [r][d], box {64, rn}, SW128
    __half* R;         // T x r
    int d, T, r, rn;
    unsigned int* status;
};

struct __align__(8) RprojBarriers {
    uint64_t full[kRStages];
    uint64_t empty[kRStages];
    uint64_t acc;
    uint32_t tmem_base;
};

__host__ __device__ inline int rproj_stage_bytes(int rn) { return 128 * kBK * 2 + ((rn * kBK * 2 + 1023) / 1024) * 1024; }
__host__ __device__ inline uint32_t tmem_cols_for(int n) {
    uint32_t c = 32;
    while (c < (uint32_t)n) c <<= 1;
    return c;
}

__global__ void __launch_bounds__(kRThreads, 1) rproj_tc_kernel(const __grid_constant__ RprojArgs args) {
    extern __shared__ __align__(1024) unsigned char rsm_raw[];
    unsigned char* rsm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(rsm_raw) + 1023) & ~uintptr_t(1023));
    const int sbytes = rproj_stage_bytes(args.rn);
    RprojBarriers* bars = reinterpret_cast<RprojBarriers*>(rsm + kRStages * sbytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = blockIdx.x * 128;
    const int nkb = args.d / kBK;
    const uint32_t ncols = tmem_cols_for(args.rn);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRStages; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        mbar_init(&bars->acc, 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&bars->tmem_base, ncols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    pdl_wait();                 // X may be produced by the preceding kernel
    pdl_launch_dependents();

    if (warp == 0) {
        if (lane == 0) {
            bool ok = true;
            const uint32_t bytes = 128 * kBK * 2 + args.rn * kBK * 2;
            for (int i = 0; i < nkb; ++i) {
                const int s = i % kRStages;
                if (i >= kRStages && ok) ok = mbar_wait(&bars->empty[s], ((i / kRStages) - 1) & 1, args.status);
                unsigned char* st = rsm + s * sbytes;
                mbar_arrive_expect_tx(&bars->full[s], bytes);
                tma_load_2d(smem_u32(st), &args.tmX, &bars->full[s], i * kBK, t0);
                tma_load_2d(smem_u32(st + 128 * kBK * 2), &args.tmB, &bars->full[s], i * kBK, 0);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = f16_idesc(128, args.rn);
            bool ok = true;
            for (int i = 0; i < nkb; ++i) {
                const int s = i % kRStages;
                if (ok) ok = mbar_wait(&bars->full[s], (i / kRStages) & 1, args.status);
                tc_fence_after();
                unsigned char* st = rsm + s * sbytes;
                const uint32_t as = smem_u32(st), bs = smem_u32(st + 128 * kBK * 2);
#pragma unroll
                for (int k = 0; k < kBK / 16; ++k)
                    umma_f16(tmem, sw128_kmajor_desc(as + k * 32), sw128_kmajor_desc(bs + k * 32), idesc,
                             (i > 0 || k > 0) ? 1u : 0u);
                umma_commit(&bars->empty[s]);
            }
            umma_commit(&bars->acc);
        }
    } else {
        const int quarter = warp & 3;
        const int tok = t0 + quarter * 32 + lane;
        mbar_wait(&bars->acc, 0, args.status);
        tc_fence_after();
        const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
        const int r = args.r;
#pragma unroll 1
        for (int c = 0; c < args.rn; c += 32) {
            uint32_t v[32];
            tmem_ld32(tl + c, v);
            if (tok < args.T) {
                __half* dst = args.R + (int64_t)tok * r + c;
#pragma unroll
                for (int j = 0; j < 32; j += 8) {
                    if (c + j < r) {   // r % 8 == 0: 8-column chunks are all-or-nothing
                        uint4 o;
                        o.x = h2_as_u32(__floats2half2_rn(__uint_as_float(v[j]), __uint_as_float(v[j + 1])));
                        o.y = h2_as_u32(__floats2half2_rn(__uint_as_float(v[j + 2]), __uint_as_float(v[j + 3])));
                        o.z = h2_as_u32(__floats2half2_rn(__uint_as_float(v[j + 4]), __uint_as_float(v[j + 5])));
                        o.w = h2_as_u32(__floats2half2_rn(__uint_as_float(v[j + 6]), __uint_as_float(v[j + 7])));
                        *reinterpret_cast<uint4*>(dst + j) = o;
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, ncols);
}

// ---------------------------------------------------------------------------
// Host side: tensor maps and launches
// ---------------------------------------------------------------------------

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2-D row-major tensor [outer][inner] of `esize`-byte elements, row pitch `pitch` bytes.
bool make_map(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
              uint64_t pitch, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {pitch};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static size_t gemm_smem_bytes() {
    return (size_t)kGemmStages * kStageBytesG + 2 * kEpiBytes + sizeof(GemmBarriers) + 1024;
}
static size_t rproj_smem_bytes(int rn) { return (size_t)kRStages * rproj_stage_bytes(rn) + sizeof(RprojBarriers) + 1024; }

static cudaError_t launch_with(const void* fn, dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
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

cudaError_t launch_rproj_prefill(const uint16_t* X, const uint16_t* B, int64_t T, int d, int r, uint16_t* R,
                                 cudaStream_t st) {
    static bool opted = false;
    if (!opted) {
        cudaError_t e = cudaFuncSetAttribute((const void*)rproj_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)rproj_smem_bytes(256));
        if (e != cudaSuccess) return e;
        opted = true;
    }
    RprojArgs a;
    std::memset(&a, 0, sizeof(a));
    const int rn = (r + 15) / 16 * 16;
    if (!make_map(&a.tmX, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, X, (uint64_t)d, (uint64_t)T, (uint64_t)d * 2, kBK, 128,
                  CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (!make_map(&a.tmB, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, B, (uint64_t)d, (uint64_t)r, (uint64_t)d * 2, kBK,
                  (uint32_t)rn, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    a.R = reinterpret_cast<__half*>(R);
    a.d = d;
    a.T = (int)T;
    a.r = r;
    a.rn = rn;
    a.status = device_status_ptr();
    void* args[] = {(void*)&a};
    return launch_with((const void*)rproj_tc_kernel, dim3((unsigned)((T + 127) / 128)), dim3(kRThreads),
                       rproj_smem_bytes(rn), st, true, args);
}

glowq_status prefill_group_forward(const ModuleView* mods, int m, int d, const uint16_t* B, int r, const uint16_t* X,
                                   int64_t T, uint16_t* R, int num_sms, cudaStream_t st) {
    if (T > ((int64_t)1 << 30)) return GLOWQ_ERR_SHAPE;
    if (!encode_fn()) return GLOWQ_ERR_CUDA;
    const bool use_r = r > 0 && B != nullptr;
    if (use_r) {
        if (launch_rproj_prefill(X, B, T, d, r, R, st) != cudaSuccess) return GLOWQ_ERR_CUDA;
    }
    static bool opted = false;
    if (!opted) {
        if (cudaFuncSetAttribute((const void*)corrected_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)gemm_smem_bytes()) != cudaSuccess)
            return GLOWQ_ERR_CUDA;
        opted = true;
    }
    PrefillArgs* a = new PrefillArgs;
    std::memset(a, 0, sizeof(*a));
    bool ok = make_map(&a->tmX, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, X, (uint64_t)d, (uint64_t)T, (uint64_t)d * 2, kBK,
                       kBN, CU_TENSOR_MAP_SWIZZLE_128B);
    if (use_r)
        ok = ok && make_map(&a->tmR, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, R, (uint64_t)r, (uint64_t)T, (uint64_t)r * 2, kBK,
                            kBN, CU_TENSOR_MAP_SWIZZLE_128B);
    int mtiles = 0;
    for (int i = 0; i < m && ok; ++i) {
        const ModuleView& mv = mods[i];
        ok = ok && make_map(&a->tmQ[i], CU_TENSOR_MAP_DATA_TYPE_UINT32, mv.q, (uint64_t)(d / 8), (uint64_t)mv.O,
                            (uint64_t)d / 2, kBK / 8, kBM, CU_TENSOR_MAP_SWIZZLE_32B);
        const bool has_A = use_r && mv.A != nullptr;
        if (has_A)
            ok = ok && make_map(&a->tmA[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, mv.A, (uint64_t)r, (uint64_t)mv.O,
                                (uint64_t)r * 2, kBK, kBM, CU_TENSOR_MAP_SWIZZLE_128B);
        ok = ok && make_map(&a->tmY[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, mv.Y, (uint64_t)mv.O, (uint64_t)T,
                            (uint64_t)mv.ldY * 2, kBM, kEpiChunk, CU_TENSOR_MAP_SWIZZLE_NONE);
        a->mod[i].s = reinterpret_cast<const __half*>(mv.s);
        a->mod[i].z = mv.z;
        a->mod[i].Y = reinterpret_cast<__half*>(mv.Y);
        a->mod[i].ldY = mv.ldY;
        a->mod[i].O = (int)mv.O;
        a->mod[i].mtile_begin = mtiles;
        a->mod[i].has_A = has_A ? 1 : 0;
        mtiles += (int)((mv.O + kBM - 1) / kBM);
    }
    if (!ok) {
        delete a;
        return GLOWQ_ERR_CUDA;
    }
    a->m = m;
    a->d = d;
    a->T = (int)T;
    a->r = use_r ? r : 0;
    a->ntiles_n = (int)((T + kBN - 1) / kBN);
    a->wait_dep = use_r ? 1 : 0;
    a->status = device_status_ptr();
    const int64_t ntiles = (int64_t)mtiles * a->ntiles_n;
    a->ntiles = (int)ntiles;
    void* args[] = {(void*)a};
    // persistent grid: one CTA per SM (fewer if there are fewer tiles)
    const int64_t grid = ntiles < num_sms ? ntiles : num_sms;
    cudaError_t e = cudaSuccess;
    if (grid > 0)
        e = launch_with((const void*)corrected_gemm_kernel, dim3((unsigned)grid), dim3(kGemmThreads), gemm_smem_bytes(),
                        st, use_r, args);
    delete a;
    return e == cudaSuccess ? GLOWQ_OK : GLOWQ_ERR_CUDA;
}

}  // namespace glowq
