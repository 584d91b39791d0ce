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
//   corrected_gemm_kernel  one 256-row x 256-token tile of y per CTA pair
//                          (thread-block cluster of 2, tcgen05 cta_group::2):
//                          D[o][t] = sum_k w_hat[o][k] X[t][k] + sum_j A[o][j] R[t][j]
//                          - in each CTA a producer warp streams its half of the
//                            X tile (SW128) and its 128 rows of packed INT4 with
//                            TMA into a 5-stage ring;
//                          - eight transform warps per CTA dequantise each INT4
//                            tile to the exact fp16 w_hat = fp16((q - z) s)
//                            straight into the canonical K-major 128B-swizzled
//                            layout the MMA reads;
//                          - one thread of the leader CTA issues tcgen05.mma
//                            (M=256, N=256, K=16) into fp32 TMEM accumulators
//                            split across the pair (128 rows each);
//                          - the rank-r correction is one more K=64 slab of the
//                            same accumulator, A_i and R tiles fetched by TMA
//                            (zero-filled beyond r), so no separate kernel or
//                            extra pass over y runs;
//                          - four epilogue warps per CTA drain TMEM (tcgen05.ld)
//                            and store y in fp16 with TMA.
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
// Fetch a TMA descriptor (a kernel parameter) ahead of its first use.
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void named_barrier_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------
// Corrected GEMM on CTA pairs.  A cluster of two CTAs computes one 256-row x
// 256-token tile of y with tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16):
// CTA p of the pair stages W rows [128p, 128p+128) of the tile (dequantised by
// its own transform warps) and tokens [128p, 128p+128) of X; the pair's tensor
// cores read both halves of X, and CTA p's TMEM receives the fp32 accumulator
// of its 128 W rows for all 256 tokens.  Per SM this halves the X tile staged
// in shared memory and read by the MMA, relative to a 128 x 256 tile on one SM.
// Persistent: clusters take pair tiles round-robin; the accumulator is double-
// buffered in TMEM (2 x 256 columns) so the drain of one tile overlaps the main
// loop of the next.
// Synchronisation inside a pair:
//   full[s]      per CTA: TMA bytes of its own halves landed
//   dq[s]        leader only: w_hat written and the stage's TMA landed, in both
//                CTAs (each warp of the owning transform group arrives, 2 x 4)
//   empty[s]     per CTA: the pair's MMAs reading stage s completed (the
//                leader's tcgen05.commit arrives on both CTAs' barriers)
//   acc_full[b]  per CTA: accumulator buffer b complete (leader's commit, both)
//   acc_empty[b] leader only: both CTAs drained buffer b (one arrival per
//                epilogue warp, 2 x 4)
// Warp roles (448 threads per CTA):
//   warp 0       TMA producer of this CTA's halves (X, INT4; R, A_i for the slab)
//   warp 1       TMEM allocation (both CTAs); the leader's lane 0 issues the MMAs
//   warps 2-9    transform: INT4 tile -> exact fp16 w_hat (SW128 K-major);
//                two groups of four warps on alternate k-blocks, one thread per row
//   warps 10-13  epilogue: TMEM -> fp16 y of this CTA's 128 rows
// ---------------------------------------------------------------------------
constexpr int kBM = 128;          // W rows per CTA (TMEM lanes)
constexpr int kPairM = 2 * kBM;   // W rows per pair tile (MMA M)
constexpr int kBK = 64;           // k per stage: one 128-byte swizzle atom of fp16
constexpr int kGemmStages = 6;                // even: each stage belongs to one transform group
constexpr int kEpiBufs = 1;                   // epilogue staging buffers
constexpr int kWBytes = kBM * kBK * 2;       // 16 KB
constexpr int kQBytes = kBM * (kBK / 8) * 4; // 4 KB packed codes (32B-swizzled rows)
constexpr int kGemmThreads = 448;            // 14 warps
constexpr int kTransformThreads = 256;
constexpr int kEpiThreads = 128;
constexpr int kEpiChunk = 32;                // tokens per epilogue chunk (TMEM columns)
constexpr int kEpiBytes = kEpiChunk * kBM * 2;   // 8 KB: [32 tokens][128 rows] fp16
static_assert(kGemmStages % 2 == 0, "transform groups own alternate stages");

// The pair tile's token width BN (MMA N, TMEM columns per accumulator): 256
// for prefill, 64 for small batches (17 <= T <= 64), where N = 256 would
// spend four times the MMA time of the tokens present on every k-block.
template <int BN>
struct PairTile {
    static constexpr int kN = BN;                          // tokens per pair tile
    static constexpr int kHalf = BN / 2;                   // tokens staged by each CTA
    static constexpr int kXBytes = kHalf * kBK * 2;        // X half-tile of a stage
    static constexpr int kStageBytes = kXBytes + kWBytes + kQBytes;   // multiple of 1024
    static constexpr int kAccCols = 2 * BN;                // double-buffered accumulator
    static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "MMA N (cta_group::2, M = 256)");
    static_assert(kStageBytes % 1024 == 0, "stage buffers hold whole swizzle atoms");
    static_assert(kGemmStages * kStageBytes + kEpiBufs * kEpiBytes + 1024 + 256 <= 232448, "shared memory per CTA");
};

struct PrefillModule {
    const void* s;     // INT4 fp16 scales [O][d/128]; MXFP4 / NVFP4 scale bytes [O][d/32] / [O][d/16]
    const uint8_t* z;  // INT4 zeros
    const float* ts;   // NVFP4 tensor scale (device)
    __half* Y;
    int64_t ldY;
    int O;
    int mtile_begin;
    int has_A;
};

struct PrefillArgs {
    CUtensorMap tmX;                       // X [T][d] fp16, box {64, 128}, SW128
    CUtensorMap tmR;                       // R [T][r] fp16, box {64, 128}, SW128
    // INT4 qweight in 16-row x 64-k blocks as 4-D {8 words, 16 rows, d/64
    // blocks, O/16 tiles}, box {8, 16, 1, 8} (eight contiguous 512-byte blocks);
    // FP4 codes [O][d/8] u32, box {8, 128}; both land as 128 rows x 32 B, SW32
    CUtensorMap tmQ[GLOWQ_MAX_MODULES];
    CUtensorMap tmA[GLOWQ_MAX_MODULES];    // A [O][r] fp16, box {64, 128}, SW128
    CUtensorMap tmY[GLOWQ_MAX_MODULES];    // Y [T][ldY] fp16 (O columns), box {128, 32} (TMA store)
    PrefillModule mod[GLOWQ_MAX_MODULES];
    int m;
    int d;
    int T;
    int r;
    int ntiles_n;                          // token tiles
    int ntiles;                            // all pair tiles
    // k-split work units: tiles [0, split_from) are one unit each; every later
    // tile is S units, part j covering k-blocks [j kbs, min((j+1) kbs, d/64)).
    // Each part stores fp32 partial sums to its slot; the last part to count
    // itself on the tile's ticket adds the S slots in ascending j and stores y.
    int split_from;
    int S;
    int kbs;                               // k-blocks per part (even: whole 128-groups)
    int nunits;
    float* slots;                          // [(tile - split_from) S + j][2 CTAs][128 rows][BN tokens] fp32
    unsigned int* tickets;                 // [(tile - split_from)][2 CTAs], zero between calls
    int wait_dep;                          // R comes from the preceding (PDL) kernel
    const float* tok_scale;                // W4A8: per-token scale s_t of the outputs (nullptr: none)
    unsigned int* status;
};

struct __align__(8) GemmBarriers {
    uint64_t full[kGemmStages];
    uint64_t dq[kGemmStages];
    uint64_t empty[kGemmStages];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint32_t tmem_base;
    uint32_t last_part;                    // epilogue: this CTA counted last on its tile's ticket
};

struct TileCoord {
    int mi, m0, n0;
    int kb0, nkb;     // k-blocks [kb0, kb0 + nkb) of the base product
    int nslab;        // correction slab blocks (the tile's last part only)
    int split;        // stored as a partial (0: y stored directly)
    int slot0;        // slot of part 0 of the tile
    int part;
    int ticket;       // ticket index of the tile (times 2 CTAs)
};

// Work unit u: m0 = first W row of the pair tile within module mi, n0 = first
// token, and its range of k.
template <int BN>
__device__ __forceinline__ TileCoord tile_coord(const PrefillArgs& args, int u) {
    TileCoord c;
    int tile = u, part = 0, nparts = 1;
    c.split = 0;
    c.slot0 = 0;
    c.ticket = 0;
    if (u >= args.split_from) {
        const int v = u - args.split_from;
        const int rel = v / args.S;
        part = v - rel * args.S;
        tile = args.split_from + rel;
        nparts = args.S;
        c.split = nparts > 1;
        c.slot0 = rel * args.S;
        c.ticket = rel;
    }
    const int mt = tile / args.ntiles_n;
    const int nt = tile - mt * args.ntiles_n;
    int mi = 0;
    for (int i = 1; i < args.m; ++i)
        if (mt >= args.mod[i].mtile_begin) mi = i;
    c.mi = mi;
    c.m0 = (mt - args.mod[mi].mtile_begin) * kPairM;
    c.n0 = nt * BN;
    const int nkb_all = args.d / kBK;
    c.part = part;
    c.kb0 = nparts > 1 ? part * args.kbs : 0;
    c.nkb = (part == nparts - 1) ? nkb_all - c.kb0 : args.kbs;
    c.nslab = (part == nparts - 1 && args.r > 0 && args.mod[mi].has_A) ? (args.r + kBK - 1) / kBK : 0;
    return c;
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_count_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrive on a barrier of either CTA of the pair (default .release.cta semantics,
// as for a local arrive: the consumer of these arrivals is the tensor core of
// the pair's leader, which reads this CTA's shared memory through the async
// proxy after the fence.proxy.async of the writers).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t caddr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(caddr) : "memory");
}
// Bounded wait whose completing arrivals may come from the other CTA of the pair.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, unsigned int* status,
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
// One k-block of pair MMAs (4 x K=16) plus the commits that free its stage in
// both CTAs, preceded by a non-blocking probe of another barrier's phase.  The
// probe's result is consumed only after the MMAs and commits are issued, so its
// shared-memory round trip overlaps the issue.  `adesc` / `bdesc` describe the
// first K=16 slice of the stage; slice k starts 32 bytes further (+2 in the
// descriptor's 16-byte address field).  Returns the probe result.
__device__ __forceinline__ uint32_t umma_kblock_pair_probe(uint32_t dacc, uint64_t adesc, uint64_t bdesc,
                                                           uint32_t idesc, uint32_t accumulate, uint32_t empty_local,
                                                           uint32_t empty_peer, uint32_t probe_bar,
                                                           uint32_t probe_parity) {
    uint32_t ready;
    asm volatile(
        "{\n\t.reg .pred pr, pa, pt;\n\t.reg .b64 a1, a2, a3, b1, b2, b3;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 pr, [%6], %7;\n\t"
        "setp.ne.b32 pa, %3, 0;\n\t"
        "setp.eq.b32 pt, %3, %3;\n\t"
        "add.s64 a1, %8, 2;\n\tadd.s64 a2, %8, 4;\n\tadd.s64 a3, %8, 6;\n\t"
        "add.s64 b1, %9, 2;\n\tadd.s64 b2, %9, 4;\n\tadd.s64 b3, %9, 6;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%1], %8, %9, %2, pa;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%1], a1, b1, %2, pt;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%1], a2, b2, %2, pt;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%1], a3, b3, %2, pt;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%4];\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%5];\n\t"
        "selp.u32 %0, 1, 0, pr;\n\t}"
        : "=r"(ready)
        : "r"(dacc), "r"(idesc), "r"(accumulate), "r"(empty_local), "r"(empty_peer), "r"(probe_bar),
          "r"(probe_parity), "l"(adesc), "l"(bdesc)
        : "memory");
    return ready;
}
__device__ __forceinline__ void umma_f16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive on the barrier at cluster address `caddr` once the pair MMAs issued so far complete.
__device__ __forceinline__ void umma_commit_pair(uint32_t caddr) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(caddr)
                 : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// E8M0 scale code -> fp16 bits of 2^(e - 127), clamped to [2^-24, 2^15] (0 below).
__device__ __forceinline__ uint32_t pf_e8m0_f16(uint32_t e) {
    if (e >= 113u && e <= 142u) return (e - 112u) << 10;
    if (e > 142u) return 0x7800u;
    if (e >= 103u) return 1u << (e - 103u);
    return 0u;
}
// fp16 bits of fp16_RN(e4m3 * s_t) (the E4M3 value is exact in fp32; one
// rounding to fp32, one to fp16).
__device__ __forceinline__ uint32_t pf_e4m3_st_f16(uint32_t c, float st) {
    uint32_t h;
    asm("{\n\t.reg .b16 b;\n\t.reg .b32 p;\n\tcvt.u16.u32 b, %1;\n\tcvt.rn.f16x2.e4m3x2 p, b;\n\t"
        "mov.b32 %0, p;\n\t}" : "=r"(h) : "r"(c & 0xffu));
    const float v = __half2float(__ushort_as_half((unsigned short)(h & 0xffffu))) * st;
    return (uint32_t)__half_as_ushort(__float2half_rn(v));
}

// FMT: GLOWQ_FMT_INT4 (w_hat = fp16((q - z) s)), GLOWQ_FMT_MXFP4 or
// GLOWQ_FMT_NVFP4 (w_hat = fp16 of the E2M1 value times the block scale,
// see the transform warps).
template <int FMT, int BN>
__global__ void __launch_bounds__(kGemmThreads, 1) corrected_gemm_kernel(const __grid_constant__ PrefillArgs args) {
    using TC = PairTile<BN>;
    extern __shared__ __align__(1024) unsigned char gsm_raw[];
    // 1024-byte alignment of the stage buffers (swizzle atoms); the same offset in both CTAs
    unsigned char* gsm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(gsm_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* epi = gsm + kGemmStages * TC::kStageBytes;            // kEpiBufs x kEpiBytes
    GemmBarriers* bars = reinterpret_cast<GemmBarriers*>(epi + kEpiBufs * kEpiBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t crank = cluster_ctarank();            // 0 = leader (issues the MMAs)
    const int first_tile = (int)cluster_id_x();
    const int tile_step = (int)cluster_count_x();
    const int row_off = (int)crank * kBM;                // this CTA's W rows within the pair tile
    const int tok_off = (int)crank * TC::kHalf;             // this CTA's tokens within the pair tile

    if (threadIdx.x == 32) {   // descriptors, fetched while thread 0 initialises the barriers
        prefetch_tmap(&args.tmX);
        if (args.r > 0) prefetch_tmap(&args.tmR);
        for (int i = 0; i < args.m; ++i) {
            prefetch_tmap(&args.tmQ[i]);
            if (args.mod[i].has_A) prefetch_tmap(&args.tmA[i]);
            prefetch_tmap(&args.tmY[i]);
        }
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < kGemmStages; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->dq[s], 2 * kTransformThreads / 64);    // one arrival per warp of the owning group
            mbar_init(&bars->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->acc_full[b], 1);
            mbar_init(&bars->acc_empty[b], 2 * kEpiThreads / 32);
        }
        fence_mbar_init();
    }
    cluster_sync_all();                                  // barriers of both CTAs initialised
    if (warp == 1) tmem_alloc_pair(&bars->tmem_base, TC::kAccCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    pdl_launch_dependents();

    if (warp == 0) {
        // ---------------- producer (both CTAs) ----------------
        if (lane == 0) {
            bool ok = true, waited = false;
            int g = 0;   // ring position of this CTA
            for (int unit = first_tile; unit < args.nunits; unit += tile_step) {
                const TileCoord c = tile_coord<BN>(args, unit);
                const int nblocks = c.nkb + c.nslab;
                for (int i = 0; i < nblocks; ++i, ++g) {
                    const int s = g % kGemmStages;
                    if (g >= kGemmStages && ok) ok = mbar_wait(&bars->empty[s], ((g / kGemmStages) - 1) & 1, args.status);
                    unsigned char* st = gsm + s * TC::kStageBytes;
                    const uint32_t xs = smem_u32(st), ws = smem_u32(st + TC::kXBytes), qs = smem_u32(st + TC::kXBytes + kWBytes);
                    if (i < c.nkb) {
                        const int kb = c.kb0 + i;
                        mbar_arrive_expect_tx(&bars->full[s], TC::kXBytes + kQBytes);
                        tma_load_2d(xs, &args.tmX, &bars->full[s], kb * kBK, c.n0 + tok_off);
                        if constexpr (FMT == GLOWQ_FMT_INT4)
                            tma_load_4d(qs, &args.tmQ[c.mi], &bars->full[s], 0, 0, kb, (c.m0 + row_off) / 16);
                        else
                            tma_load_2d(qs, &args.tmQ[c.mi], &bars->full[s], kb * (kBK / 8), c.m0 + row_off);
                    } else {
                        if (!waited && args.wait_dep) {   // R is complete
                            pdl_wait();
                            waited = true;
                        }
                        const int j = i - c.nkb;
                        mbar_arrive_expect_tx(&bars->full[s], TC::kXBytes + kWBytes);
                        tma_load_2d(xs, &args.tmR, &bars->full[s], j * kBK, c.n0 + tok_off);
                        tma_load_2d(ws, &args.tmA[c.mi], &bars->full[s], j * kBK, c.m0 + row_off);
                    }
                }
            }
            // the leader's commits for the last stages land here before this CTA may exit
            for (int p = (g > kGemmStages ? g - kGemmStages : 0); p < g && ok; ++p)
                ok = mbar_wait(&bars->empty[p % kGemmStages], (p / kGemmStages) & 1, args.status);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (leader CTA) ----------------
        if (crank == 0 && lane == 0) {
            constexpr uint32_t idesc = f16_idesc(kPairM, TC::kN);
            constexpr uint64_t kStageDesc = (uint64_t)(TC::kStageBytes >> 4);   // descriptor step per stage
            // loop-invariant addresses: everything per stage is base + stage * step
            const uint64_t adesc0 = sw128_kmajor_desc(smem_u32(gsm + TC::kXBytes));   // W of stage 0
            const uint64_t bdesc0 = sw128_kmajor_desc(smem_u32(gsm));             // X of stage 0
            const uint32_t empty_l0 = smem_u32(&bars->empty[0]);
            const uint32_t empty_p0 = cluster_addr(&bars->empty[0], 1);
            const uint32_t dq0 = smem_u32(&bars->dq[0]);
            bool ok = true;
            int tl = 0;
            int s = 0;              // stage of the current ring position
            uint32_t ph = 0;        // its phase parity
            // The barrier of the next ring position is probed (non-blocking) while
            // this position's MMAs are issued, so the shared-memory round trip of
            // the probe does not idle the tensor pipe.
            bool next_ready = false;
            for (int unit = first_tile; unit < args.nunits; unit += tile_step, ++tl) {
                const TileCoord c = tile_coord<BN>(args, unit);
                const int nblocks = c.nkb + c.nslab;
                const int buf = tl & 1;
                if (tl >= 2 && ok) ok = mbar_wait_cluster(&bars->acc_empty[buf], ((tl >> 1) - 1) & 1, args.status);
                tc_fence_after();
                const uint32_t dacc = tmem + (uint32_t)(buf * TC::kN);
                for (int i = 0; i < nblocks; ++i) {
                    // both CTAs' w_hat written and TMA landed (slab blocks: TMA only)
                    if (!next_ready && ok) ok = mbar_wait_cluster(&bars->dq[s], ph, args.status);
                    tc_fence_after();
                    const int sn = (s + 1 == kGemmStages) ? 0 : s + 1;
                    const uint32_t phn = (s + 1 == kGemmStages) ? (ph ^ 1u) : ph;
                    // frees stage s in both CTAs once these MMAs complete; probes the next
                    // position (all earlier phases of its barrier completed and were
                    // waited on, so the parity probe cannot see a stale phase)
                    next_ready = umma_kblock_pair_probe(dacc, adesc0 + (uint64_t)s * kStageDesc,
                                                        bdesc0 + (uint64_t)s * kStageDesc, idesc, i > 0 ? 1u : 0u,
                                                        empty_l0 + 8u * (uint32_t)s, empty_p0 + 8u * (uint32_t)s,
                                                        dq0 + 8u * (uint32_t)sn, phn) != 0;
                    s = sn;
                    ph = phn;
                }
                umma_commit_pair(smem_u32(&bars->acc_full[buf]));
                umma_commit_pair(cluster_addr(&bars->acc_full[buf], 1));
            }
            // both epilogues' releases of the last buffers land before the pair may exit
            for (int t = (tl > 2 ? tl - 2 : 0); t < tl && ok; ++t)
                ok = mbar_wait_cluster(&bars->acc_empty[t & 1], (t >> 1) & 1, args.status);
        }
    } else if (warp < 10) {
        // ---------------- transform (warps 2..9, both CTAs) ----------------
        // Warps 2-5 take the even ring positions, warps 6-9 the odd ones, so two
        // k-blocks are converted at once; one thread per W row converts all
        // 64 k of its row (8 packed words).  With an even number of stages each
        // stage always belongs to the same warp group, which therefore waits on
        // every phase of its barriers in order.
        const int tt = threadIdx.x - 64;
        const int row = tt & 127;                      // tile row owned by this thread
        const int par = tt >> 7;                       // ring-position parity of this warp group
        const int ngroups = args.d / 128;
        const uint32_t swz = (uint32_t)(row & 7);
        const uint32_t hsw = (uint32_t)((row >> 2) & 1);
        bool ok = true;
        int gbase = 0;                                 // ring position of the tile's first block
        // scale/zero of the current and the next 3 groups (a shift register
        // refilled 4 groups ahead, across tile boundaries)
        int cur_tile = first_tile;
        int f_tile = cur_tile, f_grp = 0;              // next group to fetch (unit, group within it)
        TileCoord fc = tile_coord<BN>(args, cur_tile < args.nunits ? cur_tile : 0);
        // per group: INT4 (s | z << 16) in .x; MXFP4 the four block scales as
        // fp16 in .x .y; NVFP4 the eight fp16_RN(e4m3 * s_t) in .x .. .w
        auto fetch = [&]() -> uint4 {
            uint4 v = make_uint4(0, 0, 0, 0);
            if (f_tile < args.nunits) {
                const int orow = fc.m0 + row_off + row;
                const PrefillModule& FM = args.mod[fc.mi];
                if (orow < FM.O) {
                    const int64_t o = (int64_t)orow * ngroups + (fc.kb0 >> 1) + f_grp;
                    if constexpr (FMT == GLOWQ_FMT_INT4) {
                        v.x = (uint32_t)__half_as_ushort(static_cast<const __half*>(FM.s)[o]) |
                              ((uint32_t)FM.z[o] << 16);
                    } else if constexpr (FMT == GLOWQ_FMT_MXFP4) {
                        const uint32_t e4 = static_cast<const uint32_t*>(FM.s)[o];
                        v.x = pf_e8m0_f16(e4 & 0xffu) | (pf_e8m0_f16((e4 >> 8) & 0xffu) << 16);
                        v.y = pf_e8m0_f16((e4 >> 16) & 0xffu) | (pf_e8m0_f16(e4 >> 24) << 16);
                    } else {
                        const uint2 e8 = static_cast<const uint2*>(FM.s)[o];
                        const float st = __ldg(FM.ts);
                        v.x = pf_e4m3_st_f16(e8.x, st) | (pf_e4m3_st_f16(e8.x >> 8, st) << 16);
                        v.y = pf_e4m3_st_f16(e8.x >> 16, st) | (pf_e4m3_st_f16(e8.x >> 24, st) << 16);
                        v.z = pf_e4m3_st_f16(e8.y, st) | (pf_e4m3_st_f16(e8.y >> 8, st) << 16);
                        v.w = pf_e4m3_st_f16(e8.y >> 16, st) | (pf_e4m3_st_f16(e8.y >> 24, st) << 16);
                    }
                }
                if (++f_grp == (fc.nkb >> 1)) {
                    f_grp = 0;
                    f_tile += tile_step;
                    if (f_tile < args.nunits) fc = tile_coord<BN>(args, f_tile);
                }
            }
            return v;
        };
        uint4 sz0 = fetch(), sz1 = fetch(), sz2 = fetch(), sz3 = fetch();
        for (; cur_tile < args.nunits; cur_tile += tile_step) {
            const TileCoord cc = tile_coord<BN>(args, cur_tile);
            const int nblocks = cc.nkb + cc.nslab;
            // a unit's nkb is even, so block i of it (group i/2) is ours when (gbase + i) % 2 == par
            for (int i = (par ^ gbase) & 1; i < nblocks; i += 2) {
                const int g = gbase + i;
                const int s = g % kGemmStages;
                if (ok) ok = mbar_wait(&bars->full[s], (g / kGemmStages) & 1, args.status);
                if (i < cc.nkb) {
                    unsigned char* st = gsm + s * TC::kStageBytes;
                    // 32-byte-swizzled INT4 rows: 16-byte half h of row r sits at r*32 + ((h ^ (r>>2)&1) << 4)
                    const unsigned char* qrow = st + TC::kXBytes + kWBytes + row * 32;
                    const uint4 qa = *reinterpret_cast<const uint4*>(qrow + (hsw << 4));
                    const uint4 qb = *reinterpret_cast<const uint4*>(qrow + ((hsw ^ 1u) << 4));
                    const uint4 sz = sz0;                            // group i/2 (one block of it is ours)
                    sz0 = sz1;
                    sz1 = sz2;
                    sz2 = sz3;
                    sz3 = fetch();
                    const uint32_t words[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
                    // row `row` of the W tile: 8 chunks of 16 B (8 fp16 in k order), chunk c at c ^ (row % 8)
                    unsigned char* wrow = st + TC::kXBytes + (row >> 3) * 1024 + (row & 7) * 128;
                    if constexpr (FMT != GLOWQ_FMT_INT4) {
                        // this k-block is half (i & 1) of its group: 2 MXFP4 / 4 NVFP4 blocks;
                        // word c holds k 8c .. 8c+7 (bytes = pairs in k order)
                        const bool second = (i & 1) != 0;
                        const uint32_t s01 = second ? (FMT == GLOWQ_FMT_MXFP4 ? sz.y : sz.z) : sz.x;
                        const uint32_t s23 = second ? sz.w : sz.y;   // NVFP4 blocks 2, 3 of the half
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            uint32_t sb;
                            if constexpr (FMT == GLOWQ_FMT_MXFP4) sb = (c < 4) ? (s01 & 0xffffu) : (s01 >> 16);
                            else sb = (c < 2) ? (s01 & 0xffffu) : (c < 4) ? (s01 >> 16) : (c < 6) ? (s23 & 0xffffu) : (s23 >> 16);
                            const __half2 sc = __half2half2(__ushort_as_half((unsigned short)sb));
                            uint32_t pr[4];
                            asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
                                "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
                                "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
                                "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
                                "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
                                "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
                                : "=r"(pr[0]), "=r"(pr[1]), "=r"(pr[2]), "=r"(pr[3])
                                : "r"(words[c]));
                            uint4 o;
                            o.x = h2_as_u32(__hmul2(u32_as_h2(pr[0]), sc));
                            o.y = h2_as_u32(__hmul2(u32_as_h2(pr[1]), sc));
                            o.z = h2_as_u32(__hmul2(u32_as_h2(pr[2]), sc));
                            o.w = h2_as_u32(__hmul2(u32_as_h2(pr[3]), sc));
                            *reinterpret_cast<uint4*>(wrow + (((uint32_t)c ^ swz) << 4)) = o;
                        }
                    } else {
                    const __half2 sc = __half2half2(__ushort_as_half((unsigned short)(sz.x & 0xffffu)));
                    const __half2 bz = __half2half2(__ushort_as_half((unsigned short)(0x6400u | ((sz.x >> 16) & 0xffu))));
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        __half2 p[4];
                        dequant_word(words[c], bz, sc, p);   // pairs (0,4) (1,5) (2,6) (3,7), exact w_hat
                        const uint32_t u0 = h2_as_u32(p[0]), u1 = h2_as_u32(p[1]), u2 = h2_as_u32(p[2]), u3 = h2_as_u32(p[3]);
                        uint4 o;
                        o.x = pair_lo(u0, u1);   // (0,1)
                        o.y = pair_lo(u2, u3);   // (2,3)
                        o.z = pair_hi(u0, u1);   // (4,5)
                        o.w = pair_hi(u2, u3);   // (6,7)
                        *reinterpret_cast<uint4*>(wrow + (((uint32_t)c ^ swz) << 4)) = o;
                    }
                    }   // INT4
                    fence_proxy_async_smem();   // generic-proxy writes visible to the tensor cores
                }
                // slab blocks are filled by TMA alone; they are still reported (after
                // the TMA landed) so the leader's dq phases follow the ring position
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(cluster_addr(&bars->dq[s], 0));   // one arrival per warp
            }
            gbase += nblocks;
        }
    } else {
        // ---------------- epilogue (warps 10..13, both CTAs) ----------------
        // Each 32-token chunk of this CTA's accumulator is transposed through
        // shared memory ([32 tokens][128 rows] fp16) and written by one TMA
        // store, which clips rows >= O and tokens >= T.  A staging buffer is
        // rewritten only after the store issued from it has finished reading it.
        // A part of a k-split tile instead stores its fp32 sums to its slot,
        // frees the accumulator, and counts itself on the tile's ticket; the
        // part that counts last adds the tile's slots in ascending part order
        // (the same order whichever part is last, so y does not depend on
        // timing) and stores y.  No CTA waits for another.
        const int quarter = warp & 3;                  // TMEM lanes 32*quarter .. +31
        const int row = quarter * 32 + lane;
        const bool leader = (warp == 10 && lane == 0);
        bool ok = true;
        int tl = 0, chunk = 0;
        // fp16 of 32 tokens of this thread's row -> staging buffer -> TMA store
        auto store_chunk = [&](const float (&f)[32], const TileCoord& c, int ch) {
            unsigned char* sb = epi + (chunk % kEpiBufs) * kEpiBytes;
            ++chunk;
            if (leader) bulk_wait_read<kEpiBufs - 1>();   // the store from this buffer is done reading
            named_barrier_sync(1, kEpiThreads);
            __half* col = reinterpret_cast<__half*>(sb) + row;
            const int tok0 = c.n0 + ch * kEpiChunk;
            if (args.tok_scale) {   // W4A8: y = s_t (X' w_hat^T + R' A^T), one rounding
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float ts = (tok0 + j < args.T) ? __ldg(args.tok_scale + tok0 + j) : 0.f;
                    col[j * kBM] = __float2half_rn(f[j] * ts);
                }
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) col[j * kBM] = __float2half_rn(f[j]);
            }
            fence_proxy_async_smem();
            named_barrier_sync(1, kEpiThreads);
            const int orow0 = c.m0 + row_off;
            if (leader && orow0 < args.mod[c.mi].O && tok0 < args.T) {
                tma_store_2d(&args.tmY[c.mi], smem_u32(sb), orow0, tok0);
                bulk_commit();
            }
        };
        for (int unit = first_tile; unit < args.nunits; unit += tile_step, ++tl) {
            const TileCoord c = tile_coord<BN>(args, unit);
            const int buf = tl & 1;
            if (ok) ok = mbar_wait(&bars->acc_full[buf], (tl >> 1) & 1, args.status);
            tc_fence_after();
            const uint32_t tacc = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * TC::kN);
            if (!c.split) {
#pragma unroll 1
                for (int ch = 0; ch < TC::kN / kEpiChunk; ++ch) {
                    uint32_t v[32];
                    tmem_ld32(tacc + ch * kEpiChunk, v);
                    float f[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(v[j]);
                    store_chunk(f, c, ch);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(cluster_addr(&bars->acc_empty[buf], 0));   // buffer may be overwritten
                continue;
            }
            // this part's sums: slot [128 rows][BN tokens] of this CTA
            const size_t slot_floats = (size_t)kBM * BN;
            float* mine = args.slots + ((size_t)(c.slot0 + c.part) * 2 + crank) * slot_floats + (size_t)row * BN;
#pragma unroll 1
            for (int ch = 0; ch < TC::kN / kEpiChunk; ++ch) {
                uint32_t v[32];
                tmem_ld32(tacc + ch * kEpiChunk, v);
                float4* dst = reinterpret_cast<float4*>(mine + ch * kEpiChunk);
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    __stcg(dst + q, make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                                __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3])));
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(cluster_addr(&bars->acc_empty[buf], 0));   // sums are in the slot
            __threadfence();                               // this thread's slot stores before the count
            named_barrier_sync(1, kEpiThreads);
            if (leader) {
                unsigned int* tk = args.tickets + c.ticket * 2 + crank;
                unsigned int prev;
                asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(prev) : "l"(tk) : "memory");
                const uint32_t last = (prev == (unsigned)(args.S - 1)) ? 1u : 0u;
                if (last) atomicExch(tk, 0u);             // every part has counted: ready for the next call
                *reinterpret_cast<volatile uint32_t*>(&bars->last_part) = last;
            }
            named_barrier_sync(1, kEpiThreads);
            if (*reinterpret_cast<volatile uint32_t*>(&bars->last_part) == 0u) continue;
            __threadfence();                               // the other parts' slots are visible
            const float* part0 = args.slots + ((size_t)c.slot0 * 2 + crank) * slot_floats + (size_t)row * BN;
#pragma unroll 1
            for (int ch = 0; ch < TC::kN / kEpiChunk; ++ch) {
                // two parts' loads in flight per L2 round trip, added in ascending part order
                float f[32];
                const float4* src0 = reinterpret_cast<const float4*>(part0 + ch * kEpiChunk);
#pragma unroll 1
                for (int p = 0; p < args.S; p += 2) {
                    const float4* src = src0 + (size_t)p * (2 * slot_floats / 4);
                    const bool pair = p + 1 < args.S;
                    float4 x[8], y[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) x[q] = __ldcg(src + q);
                    if (pair) {
#pragma unroll
                        for (int q = 0; q < 8; ++q) y[q] = __ldcg(src + 2 * slot_floats / 4 + q);
                    }
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        if (p == 0) {
                            f[4 * q] = x[q].x; f[4 * q + 1] = x[q].y; f[4 * q + 2] = x[q].z; f[4 * q + 3] = x[q].w;
                        } else {
                            f[4 * q] += x[q].x; f[4 * q + 1] += x[q].y; f[4 * q + 2] += x[q].z; f[4 * q + 3] += x[q].w;
                        }
                        if (pair) {
                            f[4 * q] += y[q].x; f[4 * q + 1] += y[q].y; f[4 * q + 2] += y[q].z; f[4 * q + 3] += y[q].w;
                        }
                    }
                }
                store_chunk(f, c, ch);
            }
        }
        if (leader) bulk_wait_all();
    }
    // the R kernel is complete before this grid is (even if no tile read R)
    if (args.wait_dep) pdl_wait();
    tc_fence_before();
    __syncwarp();
    cluster_sync_all();                                  // no arrivals or MMA reads into either CTA remain
    if (warp == 1) tmem_dealloc_pair(tmem, TC::kAccCols);
}

// ---------------------------------------------------------------------------
// R = X B^T on the tensor cores: CTA (x, y) computes tokens [128x, 128x+128)
// over the y-th of `chunks` slices of d (N = r padded to 16).  With one chunk
// it writes R in fp16; otherwise fp32 partial sums partial[y][t][j], which
// rproj_sum_kernel adds in ascending y (a fixed order: R is deterministic).
// Splitting d keeps ~all SMs busy when T / 128 is far below the SM count.
// ---------------------------------------------------------------------------
constexpr int kRStages = 4;
constexpr int kRThreads = 192;
constexpr int kRMaxChunks = 8;

struct RprojArgs {
    CUtensorMap tmX;   // X [T][d], box {64, 128}, SW128
    CUtensorMap tmB;   // B [r][d], box {64, rn}, SW128
    __half* R;         // T x r (chunks == 1)
    const float* tok_scale;   // W4A8: also write R_scaled = fp16(s_t R) (nullptr: none)
    __half* R_scaled;
    float* partial;    // chunks x T x r (chunks > 1)
    int d, T, r, rn, chunks;
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
    const int nkb_all = args.d / kBK;
    const int kb0 = (int)((int64_t)blockIdx.y * nkb_all / args.chunks);
    const int kb1 = (int)((int64_t)(blockIdx.y + 1) * nkb_all / args.chunks);
    const int nkb = kb1 - kb0;
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
                tma_load_2d(smem_u32(st), &args.tmX, &bars->full[s], (kb0 + i) * kBK, t0);
                tma_load_2d(smem_u32(st + 128 * kBK * 2), &args.tmB, &bars->full[s], (kb0 + i) * kBK, 0);
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
            if (tok < args.T && args.chunks > 1) {
                float* dst = args.partial + ((int64_t)blockIdx.y * args.T + tok) * r + c;
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    if (c + j < r) {   // r % 8 == 0: 4-column chunks are all-or-nothing
                        float4 o;
                        o.x = __uint_as_float(v[j]);
                        o.y = __uint_as_float(v[j + 1]);
                        o.z = __uint_as_float(v[j + 2]);
                        o.w = __uint_as_float(v[j + 3]);
                        *reinterpret_cast<float4*>(dst + j) = o;
                    }
                }
            } else if (tok < args.T) {
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
                        if (args.R_scaled) {
                            const float ts = args.tok_scale[tok];
                            o.x = h2_as_u32(__floats2half2_rn(__uint_as_float(v[j]) * ts, __uint_as_float(v[j + 1]) * ts));
                            o.y = h2_as_u32(__floats2half2_rn(__uint_as_float(v[j + 2]) * ts, __uint_as_float(v[j + 3]) * ts));
                            o.z = h2_as_u32(__floats2half2_rn(__uint_as_float(v[j + 4]) * ts, __uint_as_float(v[j + 5]) * ts));
                            o.w = h2_as_u32(__floats2half2_rn(__uint_as_float(v[j + 6]) * ts, __uint_as_float(v[j + 7]) * ts));
                            *reinterpret_cast<uint4*>(args.R_scaled + (int64_t)tok * r + c + j) = o;
                        }
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, ncols);
}

// R[i] = fp16_RN(sum_y partial[y][i]) in ascending y, four elements per thread.
__global__ void __launch_bounds__(256) rproj_sum_kernel(const float4* __restrict__ partial, int chunks, int n4,
                                                         uint2* __restrict__ R, const float* __restrict__ tok_scale,
                                                         uint2* __restrict__ R_scaled, int r) {
    pdl_launch_dependents();
    pdl_wait();                 // partial sums complete
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n4) return;
    // L2 loads (the partial sums were written while this grid was already
    // resident), every slice's load in flight at once, added in ascending y
    uint4 u[kRMaxChunks];
#pragma unroll
    for (int y = 0; y < kRMaxChunks; ++y)
        if (y < chunks) u[y] = ldcg_128(partial + (int64_t)y * n4 + i);
    float4 acc = make_float4(__uint_as_float(u[0].x), __uint_as_float(u[0].y), __uint_as_float(u[0].z),
                             __uint_as_float(u[0].w));
#pragma unroll
    for (int y = 1; y < kRMaxChunks; ++y) {
        if (y < chunks) {
            acc.x += __uint_as_float(u[y].x);
            acc.y += __uint_as_float(u[y].y);
            acc.z += __uint_as_float(u[y].z);
            acc.w += __uint_as_float(u[y].w);
        }
    }
    uint2 o;
    o.x = h2_as_u32(__floats2half2_rn(acc.x, acc.y));
    o.y = h2_as_u32(__floats2half2_rn(acc.z, acc.w));
    R[i] = o;
    if (R_scaled) {   // W4A8: fp16(s_t R) for the caller
        const float ts = tok_scale[(4 * i) / r];
        o.x = h2_as_u32(__floats2half2_rn(acc.x * ts, acc.y * ts));
        o.y = h2_as_u32(__floats2half2_rn(acc.z * ts, acc.w * ts));
        R_scaled[i] = o;
    }
}

// Number of d slices of the prefill R projection: enough CTAs to cover the
// SMs, at most kRMaxChunks, at least 4 k-blocks per slice.
int prefill_r_chunks(int64_t T, int d, int num_sms) {
    const int ntok = (int)((T + 127) / 128);
    int c = num_sms / (ntok > 0 ? ntok : 1);
    if (c > kRMaxChunks) c = kRMaxChunks;
    if (c > d / kBK / 4) c = d / kBK / 4;
    return c < 1 ? 1 : c;
}
size_t prefill_partial_bytes(int64_t T, int r) { return (size_t)kRMaxChunks * (size_t)T * (size_t)r * sizeof(float); }

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

// INT4 codes in 16-row x 64-k blocks (512 B, blocks along k within a 16-row
// tile): a 128-row x 64-k box is 8 tiles' blocks of one k-block, written to
// shared memory in row order like the row-major layout's 2-D box.
static bool make_map_q4(CUtensorMap* map, const void* q, int d, int64_t O) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {8, 16, (cuuint64_t)(d / 64), (cuuint64_t)(O / 16)};
    const cuuint64_t strides[3] = {32, 512, (cuuint64_t)(d / 64) * 512};
    const cuuint32_t box[4] = {8, 16, 1, kBM / 16};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, const_cast<void*>(q), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static size_t gemm_smem_bytes(int bn) {
    return (size_t)kGemmStages * (bn == 64 ? PairTile<64>::kStageBytes : PairTile<256>::kStageBytes) +
           kEpiBufs * kEpiBytes + sizeof(GemmBarriers) + 1024;
}
// CTA pairs of the GEMM that can be resident at once (one CTA per SM).
int gemm_max_pairs(int num_sms) {
    static int cached_dev = -1, cached = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return num_sms / 2;
    }
    if (dev == cached_dev) return cached;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(num_sms / 2 * 2));
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = gemm_smem_bytes(256);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (cudaFuncSetAttribute((const void*)corrected_gemm_kernel<GLOWQ_FMT_INT4, 256>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gemm_smem_bytes(256)) != cudaSuccess ||
        cudaOccupancyMaxActiveClusters(&clusters, (const void*)corrected_gemm_kernel<GLOWQ_FMT_INT4, 256>, &cfg) !=
            cudaSuccess ||
        clusters <= 0) {
        cudaGetLastError();
        clusters = num_sms / 2;
    }
    if (std::getenv("GLOWQ_VERBOSE")) std::fprintf(stderr, "glowq prefill: %d resident CTA pairs\n", clusters);
    cached_dev = dev;
    cached = clusters;
    return cached;
}

int prefill_tile_n(int64_t T) { return T <= kSmallBatchMaxTokens ? 64 : 256; }
size_t prefill_slot_bytes(int bn) { return (size_t)2 * kBM * bn * sizeof(float); }

// Work decomposition of the tcgen05 GEMM.  Small batches (tile width 64) are
// weight-streaming: with few 256-row tiles (an o_proj or down_proj has 16-20)
// most CTA pairs would idle, so each tile's k range is split into S parts
// (whole 128-groups, at least kMinSplitBlocks k-blocks each) when that
// shortens the busiest pair's work: per round of units the k-blocks of one
// unit plus its fixed cost (kUnitCost), and for a split the partial sums and
// their reduction (kSplitBaseCost + S kSplitPartCost).  Larger T keeps whole
// tiles.
SplitPlan plan_prefill_split(int64_t T, int d, int64_t mtiles, int pairs, int64_t max_slots) {
    SplitPlan p;
    p.bn = prefill_tile_n(T);
    p.ntiles_n = (T + p.bn - 1) / p.bn;
    p.ntiles = mtiles * p.ntiles_n;
    const int nkb = d / kBK;
    p.split_from = p.ntiles;
    p.S = 1;
    p.kbs = nkb;
    p.slots = 0;
    if (p.bn != 64 || pairs <= 0 || p.ntiles <= 0) return p;
    // Tuning override: GLOWQ_SPLIT_S=S forces S parts per tile (1 <= S <= 8;
    // ignored when the parts would be empty or the slots or tickets do not fit).
    if (const char* env = std::getenv("GLOWQ_SPLIT_S")) {
        const int S = std::atoi(env);
        if (S == 1) return p;
        if (S >= 2 && S <= kMaxSplit) {
            const int kbs = ((nkb + S - 1) / S + 1) & ~1;
            const int64_t units = p.ntiles * S;
            if ((int64_t)(S - 1) * kbs < nkb && units <= max_slots && p.ntiles * 2 <= kMaxTickets) {
                p.S = S;
                p.kbs = kbs;
                p.split_from = 0;
                p.slots = units;
                return p;
            }
        }
    }
    int64_t best = (p.ntiles + pairs - 1) / pairs * (int64_t)(nkb + kUnitCost);
    for (int S = 2; S <= kMaxSplit; ++S) {
        const int kbs = ((nkb + S - 1) / S + 1) & ~1;
        if (kbs < kMinSplitBlocks) break;
        if ((int64_t)(S - 1) * kbs >= nkb) continue;      // the last part would be empty
        const int64_t units = p.ntiles * S;
        if (units > max_slots || p.ntiles * 2 > kMaxTickets) break;
        const int64_t cost = (units + pairs - 1) / pairs * (int64_t)(kbs + kUnitCost) + kSplitBaseCost +
                             (int64_t)S * kSplitPartCost;
        if (cost < best) {
            best = cost;
            p.S = S;
            p.kbs = kbs;
            p.split_from = 0;
            p.slots = units;
        }
    }
    return p;
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
                                 float* partial, int num_sms, cudaStream_t st, const float* tok_scale,
                                 uint16_t* R_scaled) {
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
    const int chunks = partial ? prefill_r_chunks(T, d, num_sms) : 1;
    a.R = reinterpret_cast<__half*>(R);
    a.tok_scale = tok_scale;
    a.R_scaled = reinterpret_cast<__half*>(R_scaled);
    a.partial = partial;
    a.d = d;
    a.T = (int)T;
    a.r = r;
    a.rn = rn;
    a.chunks = chunks;
    a.status = device_status_ptr();
    void* args[] = {(void*)&a};
    cudaError_t e = launch_with((const void*)rproj_tc_kernel, dim3((unsigned)((T + 127) / 128), (unsigned)chunks),
                                dim3(kRThreads), rproj_smem_bytes(rn), st, true, args);
    if (e != cudaSuccess || chunks == 1) return e;
    const float4* p4 = reinterpret_cast<const float4*>(partial);
    const int n4 = (int)(T * r / 4);
    uint2* R4 = reinterpret_cast<uint2*>(R);
    uint2* RS4 = reinterpret_cast<uint2*>(R_scaled);
    void* a2[] = {(void*)&p4, (void*)&chunks, (void*)&n4, (void*)&R4, (void*)&tok_scale, (void*)&RS4, (void*)&r};
    return launch_with((const void*)rproj_sum_kernel, dim3((unsigned)((n4 + 255) / 256)), dim3(256), 0, st, true, a2);
}

template <int BN>
static const void* gemm_kernel_for(int fmt) {
    return fmt == GLOWQ_FMT_MXFP4   ? (const void*)corrected_gemm_kernel<GLOWQ_FMT_MXFP4, BN>
           : fmt == GLOWQ_FMT_NVFP4 ? (const void*)corrected_gemm_kernel<GLOWQ_FMT_NVFP4, BN>
                                    : (const void*)corrected_gemm_kernel<GLOWQ_FMT_INT4, BN>;
}

glowq_status prefill_group_forward(const ModuleView* mods, int m, int d, const uint16_t* B, int r, const uint16_t* X,
                                   int64_t T, uint16_t* R, float* partial, int num_sms, cudaStream_t st, int fmt,
                                   const float* tok_scale, uint16_t* R_scaled, unsigned int* tickets, float* slots,
                                   int64_t max_slots) {
    if (T > ((int64_t)1 << 30)) return GLOWQ_ERR_SHAPE;
    if (!encode_fn()) return GLOWQ_ERR_CUDA;
    const bool use_r = r > 0 && B != nullptr;
    if (use_r) {
        if (launch_rproj_prefill(X, B, T, d, r, R, partial, num_sms, st, tok_scale, R_scaled) != cudaSuccess)
            return GLOWQ_ERR_CUDA;
    }
    static bool opted = false;
    if (!opted) {
        const int f[3] = {GLOWQ_FMT_INT4, GLOWQ_FMT_MXFP4, GLOWQ_FMT_NVFP4};
        for (int i = 0; i < 3; ++i)
            if (cudaFuncSetAttribute(gemm_kernel_for<256>(f[i]), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)gemm_smem_bytes(256)) != cudaSuccess ||
                cudaFuncSetAttribute(gemm_kernel_for<64>(f[i]), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)gemm_smem_bytes(64)) != cudaSuccess)
                return GLOWQ_ERR_CUDA;
        opted = true;
    }
    int64_t mtiles = 0;
    for (int i = 0; i < m; ++i) mtiles += (mods[i].O + kPairM - 1) / kPairM;
    const int max_pairs = gemm_max_pairs(num_sms);
    const SplitPlan plan = plan_prefill_split(T, d, mtiles, max_pairs, (tickets && slots) ? max_slots : 0);
    const int bn = plan.bn;
    PrefillArgs* a = new PrefillArgs;
    std::memset(a, 0, sizeof(*a));
    bool ok = make_map(&a->tmX, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, X, (uint64_t)d, (uint64_t)T, (uint64_t)d * 2, kBK,
                       (uint32_t)(bn / 2), CU_TENSOR_MAP_SWIZZLE_128B);
    if (use_r)
        ok = ok && make_map(&a->tmR, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, R, (uint64_t)r, (uint64_t)T, (uint64_t)r * 2, kBK,
                            (uint32_t)(bn / 2), CU_TENSOR_MAP_SWIZZLE_128B);
    int mt = 0;
    for (int i = 0; i < m && ok; ++i) {
        const ModuleView& mv = mods[i];
        ok = ok && ((fmt == GLOWQ_FMT_INT4)
                        ? make_map_q4(&a->tmQ[i], mv.q, d, mv.O)
                        : make_map(&a->tmQ[i], CU_TENSOR_MAP_DATA_TYPE_UINT32, mv.q, (uint64_t)(d / 8), (uint64_t)mv.O,
                                   (uint64_t)d / 2, kBK / 8, kBM, CU_TENSOR_MAP_SWIZZLE_32B));
        const bool has_A = use_r && mv.A != nullptr;
        if (has_A)
            ok = ok && make_map(&a->tmA[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, mv.A, (uint64_t)r, (uint64_t)mv.O,
                                (uint64_t)r * 2, kBK, kBM, CU_TENSOR_MAP_SWIZZLE_128B);
        ok = ok && make_map(&a->tmY[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, mv.Y, (uint64_t)mv.O, (uint64_t)T,
                            (uint64_t)mv.ldY * 2, kBM, kEpiChunk, CU_TENSOR_MAP_SWIZZLE_NONE);
        a->mod[i].s = mv.s;
        a->mod[i].z = mv.z;
        a->mod[i].ts = mv.ts;
        a->mod[i].Y = reinterpret_cast<__half*>(mv.Y);
        a->mod[i].ldY = mv.ldY;
        a->mod[i].O = (int)mv.O;
        a->mod[i].mtile_begin = mt;
        a->mod[i].has_A = has_A ? 1 : 0;
        mt += (int)((mv.O + kPairM - 1) / kPairM);
    }
    if (!ok) {
        delete a;
        return GLOWQ_ERR_CUDA;
    }
    a->m = m;
    a->d = d;
    a->T = (int)T;
    a->r = use_r ? r : 0;
    a->ntiles_n = (int)plan.ntiles_n;
    a->ntiles = (int)plan.ntiles;
    a->split_from = (int)plan.split_from;
    a->S = plan.S;
    a->kbs = plan.kbs;
    a->nunits = (int)(plan.split_from + (plan.ntiles - plan.split_from) * plan.S);
    a->slots = plan.S > 1 ? slots : nullptr;
    a->tickets = plan.S > 1 ? tickets : nullptr;
    a->wait_dep = use_r ? 1 : 0;
    a->tok_scale = tok_scale;
    a->status = device_status_ptr();
    void* args[] = {(void*)a};
    // persistent grid: as many CTA pairs as fit at once (fewer if there are fewer units)
    const int64_t pairs = a->nunits < max_pairs ? a->nunits : max_pairs;
    cudaError_t e = cudaSuccess;
    if (pairs > 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(2 * pairs));
        cfg.blockDim = dim3(kGemmThreads);
        cfg.dynamicSmemBytes = gemm_smem_bytes(bn);
        cfg.stream = st;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = use_r ? 2 : 1;
        e = cudaLaunchKernelExC(&cfg, bn == 64 ? gemm_kernel_for<64>(fmt) : gemm_kernel_for<256>(fmt), args);
    }
    delete a;
    return e == cudaSuccess ? GLOWQ_OK : GLOWQ_ERR_CUDA;
}

}  // namespace glowq
