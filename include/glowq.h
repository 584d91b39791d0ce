/*
 * glowq.h -- C ABI of libglowq, the B200 (sm_100a) GlowQ corrected quantised
 * linear layer.
 *
 * What it computes (GlowQ: Group-Shared Low-Rank Approximation for Quantized
 * LLMs; papernotes.org summary, key design 4, and the experimental set-up
 * paragraph): for an input-sharing group of m modules (Q/K/V, or gate/up) with
 * INT4 g128 weights W_i^(q), per-module left factors A_i and one shared right
 * factor B,
 *
 *     R   = X B^T                      (once per group, in the anchor step)
 *     y_i = X deq(W_i^(q))^T + R A_i^T (every module of the group)
 *
 * and solo modules (o_proj, down_proj) compute y = X deq(W)^T + (X B^T) A^T
 * with their own B, nothing shared.  GlowQ-S (same key design) enables the
 * correction only on the top-k units ranked by g_ner(u) = ||E_u||_F^2 /
 * ||W_u||_F^2, falling back to layer order when the signal is weak.
 *
 * Conventions (all calls):
 *   - Matrices are row-major.  X is token-major: T x d.  Outputs are T x O.
 *   - fp16 values travel as their IEEE binary16 bit patterns (uint16_t).
 *   - Device pointers are caller-owned device memory; the library never
 *     allocates or frees them.  Host pointers are marked "host".
 *   - Every call that takes `stream` (a cudaStream_t, NULL = legacy default
 *     stream) is asynchronous on that stream: it validates its arguments on
 *     the host, enqueues kernels and returns.  Errors found on the host are
 *     returned before anything is enqueued.  A launch failure returns
 *     GLOWQ_ERR_CUDA.  Faults detected inside kernels (a bounded wait that ran
 *     out) are recorded in a per-device status word read by
 *     glowq_get_device_status().
 *   - Alignment: every device pointer 16-byte aligned; d % 128 == 0;
 *     out_features % 16 == 0; ldY % 8 == 0 and ldY >= out_features;
 *     r % 8 == 0 with 0 <= r <= 256 (r == 0 disables the correction).
 *   - No exception crosses this boundary.
 */
#ifndef GLOWQ_H
#define GLOWQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GLOWQ_API __attribute__((visibility("default")))
#else
#define GLOWQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum glowq_status {
    GLOWQ_OK = 0,
    GLOWQ_ERR_ARG = 1,          /* null pointer, negative size, bad enum    */
    GLOWQ_ERR_SHAPE = 2,        /* size constraint violated (d % 128, ...)  */
    GLOWQ_ERR_ALIGN = 3,        /* pointer or leading dimension misaligned  */
    GLOWQ_ERR_CUDA = 4,         /* CUDA runtime error while enqueueing      */
    GLOWQ_ERR_TIMEOUT = 5,      /* a device-side bounded wait ran out       */
    GLOWQ_ERR_UNSUPPORTED = 6,  /* valid request outside this build's scope */
    GLOWQ_ERR_NUMERIC = 7       /* a factorisation met a non-positive pivot  */
} glowq_status;

#define GLOWQ_GROUP_SIZE 128    /* INT4 quantisation group along d          */
#define GLOWQ_MAX_RANK 256      /* largest correction rank r                */
#define GLOWQ_MAX_MODULES 8     /* largest input-sharing group (m)          */

/*
 * One quantised module of a group.  Device pointers:
 *   qweight  O * d/8 uint32 words: code k of row o is nibble (k % 8) of word
 *                      kw = k/8 of that row, lowest nibble first (codes
 *                      0..15).  The words are stored in blocks of 16 rows x
 *                      64 k (16 x 8 words, 512 B): word kw of row o is at
 *                      index ((o/16) * (d/64) + kw/8) * 128 + (o%16) * 8
 *                      + kw%8, i.e. blocks along k within a 16-row tile,
 *                      tiles in row order.  Every call that takes a qweight
 *                      uses this layout (glowq_pack_int4 writes it); a decode
 *                      ring stage (16 rows x 256 k) is then 2 KB of
 *                      contiguous memory.
 *   scales   [O][d/128] fp16 bits (s)
 *   zeros    [O][d/128] uint8   (z, 0..15)
 *            dequantised weight w_hat[o][k] = fp16_RN((q - z) * s)
 *   A        [O][r]    fp16 bits, left factor; NULL disables this module's
 *                      correction (a GlowQ-S unit that is not restored)
 *   Y        output, T rows of ldY fp16 elements; columns [0, O) written
 */
typedef struct glowq_module {
    const uint32_t* qweight;
    const uint16_t* scales;
    const uint8_t* zeros;
    const uint16_t* A;
    int64_t out_features;
    uint16_t* Y;
    int64_t ldY;
} glowq_module;

/*
 * INT4 g128 asymmetric round-to-nearest quantisation and packing (set-up
 * paragraph: INT4 weights, group size 128).  Per row o and group j, in IEEE
 * fp32 round-to-nearest-even without fused multiply-add:
 *   mn = min(min w, 0), mx = max(max w, 0)
 *   s  = fp16_RN((mx - mn) / 15)   (s == 0 -> 1.0, s == inf -> 65504)
 *   z  = clamp(rint(-mn / s), 0, 15)
 *   q  = clamp(rint(w / s) + z, 0, 15)      (NaN weights -> code 0)
 * W: device, O x d fp32.  Outputs: qweight (O * d/8 words in the block
 * layout described at glowq_module), scales [O][d/128], zeros [O][d/128]
 * (device, caller-allocated).  group_size must be 128; O % 16 == 0.
 */
GLOWQ_API glowq_status glowq_pack_int4(const float* W, int64_t O, int64_t d, int32_t group_size,
                             uint32_t* qweight, uint16_t* scales, uint8_t* zeros,
                             void* stream);

/*
 * Dequantise to fp16: W_deq[o][k] = fp16_RN((q - z) * s), one rounding of the
 * exact product.  qweight in the block layout (glowq_module); W_deq: device,
 * O x d fp16 bits, row-major.  O % 16 == 0.  Used to check the packed format;
 * the forward kernels dequantise in registers / shared memory and never
 * materialise W_deq.
 */
GLOWQ_API glowq_status glowq_dequant_int4(const uint32_t* qweight, const uint16_t* scales,
                                const uint8_t* zeros, int64_t O, int64_t d,
                                int32_t group_size, uint16_t* W_deq, void* stream);

/*
 * Base-weight formats (thelatestinai.com GlowQ page, Table 13: GlowQ's
 * correction applied on top of INT4, MXFP4 and NVFP4 base weights).  The
 * pages name MXFP4 and NVFP4 without defining them; their public definitions
 * are used, each a reading:
 *   E2M1 element (4 bits): sign bit 3, exponent bits 2..1 (bias 1), mantissa
 *     bit 0; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6.  Encoding: nearest
 *     magnitude, ties to the even mantissa, saturating at 6; zero and NaN
 *     encode as 0 (so a tiny negative value gives +0).
 *   MXFP4: blocks of 32 consecutive k of a row share an E8M0 scale
 *     X = 2^(floor(log2 amax) - 2) (code clamped to 0..254; 2^-127 for an
 *     all-zero block); elements E2M1(w / X) in IEEE fp32.
 *   NVFP4: one fp32 tensor scale s_t = amax_tensor / (6 * 448) (1 for an
 *     all-zero tensor); blocks of 16 k share an E4M3 scale
 *     S = E4M3(amax_block / (6 s_t)) (nearest, ties to even, saturating at
 *     448); elements E2M1(w / (S s_t)), 0 when S s_t == 0.  All scale
 *     arithmetic in IEEE fp32 without fused multiply-add.
 *   Packing: codes [O][d/8] uint32, code k of a row in nibble (k % 8) of word
 *   k / 8 (as for INT4); scales [O][d/32] (MXFP4, E8M0) or [O][d/16]
 *   (NVFP4, E4M3) bytes, row-major.
 *   Dequantised weight: w_hat = fp16_RN(exact e2m1 * scale (* s_t)).
 */
typedef enum glowq_format {
    GLOWQ_FMT_INT4 = 0,
    GLOWQ_FMT_MXFP4 = 1,
    GLOWQ_FMT_NVFP4 = 2
} glowq_format;

/*
 * MXFP4 or NVFP4 quantisation and packing of W (device, O x d fp32, d % 128
 * == 0).  Outputs (device, caller-allocated): codes [O][d/8] uint32, scales
 * [O][d/32] (MXFP4) or [O][d/16] (NVFP4) bytes, and for NVFP4 the tensor
 * scale s_t in tensor_scale[0] (one float; ignored for MXFP4, may be NULL).
 * Errors: GLOWQ_ERR_ARG (null pointer, negative size, fmt not MXFP4/NVFP4),
 * GLOWQ_ERR_SHAPE (d % 128), GLOWQ_ERR_ALIGN (W not 16-byte aligned, codes
 * not 4-byte aligned, tensor_scale not 4-byte aligned).
 */
GLOWQ_API glowq_status glowq_pack_fp4(glowq_format fmt, const float* W, int64_t O, int64_t d, uint32_t* codes,
                                      uint8_t* scales, float* tensor_scale, void* stream);

/*
 * Dequantise MXFP4 / NVFP4 codes to fp16 (device, O x d): w_hat =
 * fp16_RN(e2m1 * 2^(e - 127)) or fp16_RN(e2m1 * e4m3 * s_t), the product
 * formed exactly.  Arguments as for glowq_pack_fp4; tensor_scale is read on
 * the device (NVFP4 only).  Used to check the packed formats; the forward
 * kernels never materialise w_hat in HBM.
 */
GLOWQ_API glowq_status glowq_dequant_fp4(glowq_format fmt, const uint32_t* codes, const uint8_t* scales,
                                         const float* tensor_scale, int64_t O, int64_t d, uint16_t* W_deq,
                                         void* stream);

/*
 * Bytes of device scratch the forward calls need for T tokens at rank r:
 *   - a 4096-byte zero region at offset 0: the hand-off flags (bytes 0..255),
 *     through which the decode GEMV (T <= 16) learns, while it already streams
 *     weights, that the kernel computing R = X B^T has seen X final and has
 *     stored R, and the k-split tickets (bytes 256..4095, see
 *     glowq_workspace_bytes_for);
 *   - for T > 16, the fp32 partial sums of R split along d into up to 8 slices
 *     (added in a fixed order, so R does not depend on timing);
 *   - the solo call's R.
 * 0 when r == 0 or T == 0 (no workspace is required then).  The caller
 * allocates it once and may reuse it across calls issued in order on one
 * stream (any T); calls that may overlap need separate workspaces.
 * Ownership: caller's device memory, 16-byte aligned.  The first 4096 bytes
 * must be zero before the first call that uses the workspace; every call that
 * completes leaves them zero.  After a call returned GLOWQ_ERR_CUDA, or
 * glowq_get_device_status reported GLOWQ_ERR_TIMEOUT, zero them again.
 */
GLOWQ_API size_t glowq_workspace_bytes(int64_t T, int32_t r);

/*
 * Workspace size that also lets one forward call of this shape split the
 * reduction over d across CTA pairs (any r >= 0, also r == 0):
 *   T, r, d        as for the forward call
 *   out_features   host array of the m modules' output widths
 * Small batches (16 < T <= 64) run the tensor-core GEMM on 64-token tiles,
 * whose 256-row tiles are too few to occupy every SM (an o_proj or down_proj
 * has 16-20); each tile's d range is then split into S parts of whole
 * 128-groups, each part stores its fp32 sums to a slot behind the other
 * workspace regions (2 x 128 x 64 x 4 bytes per part), and the part that
 * counts last on the tile's ticket (zero region, bytes 256..4095) adds the S
 * slots in ascending part order and stores Y.  The order of the sum is fixed,
 * so Y does not depend on timing; no CTA waits for another.  A forward call
 * splits only when its workspace (workspace_bytes) reaches at least one slot
 * past the zero region, the partial sums of R and the solo R (past the 4096
 * zero bytes alone when r == 0), and uses as many parts as the rest holds;
 * with less it runs whole tiles.  Any workspace passed, also with r == 0,
 * follows the zero-region rule of glowq_workspace_bytes.  Returns
 * glowq_workspace_bytes(T, r) when the call would not split (T <= 16, T > 64,
 * enough tiles, invalid arguments).
 */
GLOWQ_API size_t glowq_workspace_bytes_for(int64_t T, int32_t r, int64_t d, const int64_t* out_features,
                                           int32_t m);

/*
 * Input-sharing group forward (key design 4): R = X B^T is computed once and
 * written to R_out; then every module i computes
 *   Y_i = X w_hat_i^T + R A_i^T   (A_i == NULL: Y_i = X w_hat_i^T)
 * in one launch over the stacked rows of all modules.
 *   mods       host array of m module descriptors (mods[0] is the anchor)
 *   m          1..GLOWQ_MAX_MODULES
 *   d          shared input dimension
 *   B          device, r x d fp16 bits, shared right factor (NULL iff r == 0)
 *   r          correction rank, 0..256, multiple of 8
 *   X          device, T x d fp16 bits
 *   T          tokens (>= 0; T == 0 is a no-op)
 *   R_out      device, T x r fp16 bits (the cached projection; NULL iff r == 0)
 *   workspace  device scratch of at least glowq_workspace_bytes(T, r) bytes
 *              (glowq_workspace_bytes_for: the size that enables the k-split;
 *              may be NULL when r == 0; 16-byte aligned when not NULL)
 * Small T (<= 16) runs the weight-streaming decode kernels; larger T runs the
 * tcgen05 tensor-core kernels (64-token tiles up to T = 64, 256 above).
 * Tuning overrides, read from the environment at every call (for measuring,
 * e.g. with rank_error_correction_b200/tune.py; invalid values are ignored):
 * GLOWQ_DECODE_SHAPE="rt,kw,kc,stages" sets the decode kernel's work shape,
 * GLOWQ_SPLIT_S=S the number of parts per tile of the small-batch k-split.  Accumulation is fp32; R and Y are rounded to
 * fp16 (round-to-nearest-even).
 */
GLOWQ_API glowq_status glowq_group_forward(const glowq_module* mods, int32_t m, int64_t d,
                                 const uint16_t* B, int32_t r, const uint16_t* X,
                                 int64_t T, uint16_t* R_out, void* workspace,
                                 size_t workspace_bytes, void* stream);

/*
 * Solo module forward (key design 4, o_proj / down_proj): its own
 * R = X B^T is computed inline into the workspace and consumed at once;
 * Y = X w_hat^T + R A^T.  A NULL mod->A or r == 0 gives plain W4A16.
 * Arguments as for glowq_group_forward.
 */
GLOWQ_API glowq_status glowq_solo_forward(const glowq_module* mod, int64_t d, const uint16_t* B,
                                int32_t r, const uint16_t* X, int64_t T, void* workspace,
                                size_t workspace_bytes, void* stream);

/*
 * One MXFP4 / NVFP4 module of a group (formats and packing as for
 * glowq_pack_fp4).  Device pointers:
 *   codes         [O][d/8] uint32 E2M1 codes
 *   scales        [O][d/32] E8M0 (MXFP4, 4-byte aligned) or [O][d/16] E4M3
 *                 (NVFP4, 8-byte aligned) bytes
 *   tensor_scale  NVFP4: one float s_t; ignored (may be NULL) for MXFP4
 *   A, out_features, Y, ldY  as in glowq_module
 */
typedef struct glowq_fp4_module {
    const uint32_t* codes;
    const uint8_t* scales;
    const float* tensor_scale;
    const uint16_t* A;
    int64_t out_features;
    uint16_t* Y;
    int64_t ldY;
} glowq_fp4_module;

/*
 * Group and solo forward with MXFP4 / NVFP4 base weights (thelatestinai.com
 * GlowQ page, Table 13: the group-shared correction on top of these base
 * datatypes), W4A16: Y_i = X w_hat_i^T + R A_i^T with R = X B^T computed once
 * per group, as glowq_group_forward / glowq_solo_forward do for INT4 (same
 * arguments, workspace and errors; all modules of a call share one format).
 * The kernels form each weight in fp16 from its exact E2M1 value and block
 * scale (one conversion per pair of codes, one multiply): MXFP4 as
 * fp16_RN(e2m1 * 2^(e - 127)), block scales outside [2^-24, 2^15] clamped to
 * that range (below 2^-24: 0); NVFP4 at T <= 16 as the exact e2m1 * e4m3 with
 * the tensor scale s_t applied to the fp32 sums, at T > 16 (tensor-core path,
 * where the correction shares the accumulator) as
 * fp16_RN(e2m1 * fp16_RN(e4m3 * s_t)).
 */
GLOWQ_API glowq_status glowq_group_forward_fp4(glowq_format fmt, const glowq_fp4_module* mods, int32_t m, int64_t d,
                                               const uint16_t* B, int32_t r, const uint16_t* X, int64_t T,
                                               uint16_t* R_out, void* workspace, size_t workspace_bytes,
                                               void* stream);
GLOWQ_API glowq_status glowq_solo_forward_fp4(glowq_format fmt, const glowq_fp4_module* mod, int64_t d,
                                              const uint16_t* B, int32_t r, const uint16_t* X, int64_t T,
                                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * W4A8: FP8 E4M3 activations (thelatestinai.com GlowQ page, Tables 14-15:
 * GlowQ with 8-bit activations; the format is not defined there, a reading):
 * each token t gets one fp32 scale s_t = amax_t / 448 (1 for an all-zero
 * row) and codes E4M3(x / s_t), nearest with ties to even, saturating at 448,
 * NaN -> 0x7f; the layer consumes x_hat = dec(code) s_t.
 * glowq_quantize_act_e4m3: X (device, T x d fp16) -> codes (device, T x d
 * bytes; may be NULL), scales (device, T floats), X_q (device, T x d fp16 of
 * the exact code values dec(code), so x_hat = s_t X_q).
 */
GLOWQ_API glowq_status glowq_quantize_act_e4m3(const uint16_t* X, int64_t T, int64_t d, uint8_t* codes,
                                               float* scales, uint16_t* X_q, void* stream);

/* Device scratch of the W4A8 forward calls (it includes the forward workspace). */
GLOWQ_API size_t glowq_w4a8_workspace_bytes(int64_t T, int64_t d, int32_t r);

/*
 * W4A8 group and solo forward with INT4 base weights: R = x_hat B^T and
 * Y_i = x_hat w_hat_i^T + R A_i^T with x_hat the FP8 activations above.
 * Computed exactly as s_t (X_q w_hat_i^T + X_q B^T A_i^T) on the fp16 tensor
 * cores (X_q holds exact fp16 values), the per-token scale applied to the
 * fp32 sums before the one rounding to fp16.  Arguments as for
 * glowq_group_forward / glowq_solo_forward; X is the fp16 input (quantised
 * inside the call); workspace of glowq_w4a8_workspace_bytes(T, d, r).
 */
GLOWQ_API glowq_status glowq_group_forward_w4a8(const glowq_module* mods, int32_t m, int64_t d, const uint16_t* B,
                                                int32_t r, const uint16_t* X, int64_t T, uint16_t* R_out,
                                                void* workspace, size_t workspace_bytes, void* stream);
GLOWQ_API glowq_status glowq_solo_forward_w4a8(const glowq_module* mod, int64_t d, const uint16_t* B, int32_t r,
                                               const uint16_t* X, int64_t T, void* workspace,
                                               size_t workspace_bytes, void* stream);

/*
 * Solo module forward that allocates nothing (the GlowQ pages have no
 * counterpart: this is a deployment convenience of this library).
 *
 * Same computation and arguments as glowq_solo_forward, minus the workspace:
 * the scratch it needs (the hand-off flags, R and, for T > 16, the split-d
 * partial sums of R) lives in a fixed array compiled into the library,
 * glowq_noalloc_scratch_bytes() (1 MiB) on every device that loads the
 * library, held until process exit.  It is meant for callers that cannot
 * allocate device memory when they call -- e.g. a custom op or plugin running
 * inside another runtime's enqueue step, where that runtime owns every device
 * allocation.  The call itself performs no cudaMalloc/cudaFree and no other
 * allocation of device memory.
 *   - Sizes whose scratch need, glowq_workspace_bytes(T, r), exceeds
 *     glowq_noalloc_scratch_bytes() are rejected with GLOWQ_ERR_SHAPE before
 *     anything is enqueued.  At r = 64 the largest accepted T is 480 (for
 *     T > 16 the split-d partial sums need 8 x T x r x 4 bytes).  The rest of
 *     the array serves the k-split of small batches (glowq_workspace_bytes_for)
 *     as far as it reaches.
 *   - The first call on a device looks up the array's device address (once per
 *     device, with that device current) and keeps it for the life of the CUDA
 *     context (not across a cudaDeviceReset); make that first call before any
 *     stream capture.
 *   - All calls on a device share the one array, which keeps the last call's
 *     contents: calls that may overlap on the GPU (different streams without
 *     ordering between them) race on it.  Each call first clears the
 *     array's 4096-byte zero region (hand-off flags, k-split tickets) on
 *     `stream` (cudaMemsetAsync, which allocates nothing), so flags or tickets
 *     left non-zero by a failed or timed-out call never reach the next one;
 *     every other value a call reads there is written earlier by the same
 *     call.
 */
GLOWQ_API glowq_status glowq_solo_forward_noalloc(const glowq_module* mod, int64_t d, const uint16_t* B,
                                                  int32_t r, const uint16_t* X, int64_t T, void* stream);

/* Size of the fixed scratch array used by glowq_solo_forward_noalloc. */
GLOWQ_API size_t glowq_noalloc_scratch_bytes(void);

/*
 * One module of a group for the offline solve: its fp32 weight and INT4 pack
 * (device pointers, as produced by glowq_pack_int4).
 */
typedef struct glowq_solve_module {
    const float* W;             /* O x d fp32 */
    const uint32_t* qweight;    /* O * d/8 words, block layout (glowq_module) */
    const uint16_t* scales;     /* [O][d/128] fp16 bits */
    const uint8_t* zeros;       /* [O][d/128] */
    int64_t out_features;       /* O */
} glowq_solve_module;

/* Device scratch bytes glowq_group_solve needs for `rows` stacked rows (sum of
   out_features), input dimension d, rank r and oversampling p. */
GLOWQ_API size_t glowq_solve_workspace_bytes(int64_t rows, int64_t d, int32_t r, int32_t p);

/*
 * Offline whitened group solve on the GPU (papernotes.org summary, key
 * designs 1-3; thelatestinai.com GlowQ page, Tables 11-12: randomised SVD of
 * the covariance-aligned core with oversampling p and q power iterations).
 * For the stacked error E_cat = [W_1 - w_hat_1; ...] (M = sum O_i rows):
 *   E_w = E_cat Sx^{1/2};  Halko randomised SVD of E_w with the test matrix
 *   Omega (d x (r+p)), orthonormalising after every product (Y = E_w Omega,
 *   then q times E_w^T Q and E_w Z);  A = Q U_r S_r^{1/2} (M x r, the row
 *   blocks are the A_i), B = S_r^{1/2} V_r^T Sx^{+1/2} (r x d);  the top r
 *   singular values sigma_j of E_w; g_ec = sum_j sigma_j^2 / ||E_w||_F^2.
 * E_w has the singular values and right vectors of the pages' thin-QR core
 * M = R_e Sx^{1/2} (E_w = Q_e M), so the factors are the core's.  All
 * arithmetic is float64 on the device.
 *   mods, m        host array of 1..GLOWQ_MAX_MODULES modules (out_features
 *                  % 16 == 0, qweight in the block layout of glowq_module)
 *   Sx_half        device, d x d float64 Sx^{1/2} (symmetric)
 *   Sx_half_pinv   device, d x d float64 pseudo-inverse of Sx^{1/2}
 *   r, p, q        rank (>= 1, r % 8 == 0), oversampling (even, r + p <= 112
 *                  and <= min(M, d)), power iterations (0..16)
 *   Omega          device, d x (r+p) float64 Gaussian test matrix (caller's draw)
 *   A, B           device outputs, float64, M x r and r x d
 *   sing, g_ec     device outputs, r doubles and one double (either may be NULL)
 *   A16, B16       optional device outputs, the same factors rounded to fp16
 *   workspace      device scratch of glowq_solve_workspace_bytes(M, d, r, p)
 * Errors: GLOWQ_ERR_ARG / GLOWQ_ERR_SHAPE / GLOWQ_ERR_ALIGN before anything is
 * enqueued; a non-positive Cholesky pivot while orthonormalising (a
 * rank-deficient iterate) records GLOWQ_ERR_NUMERIC in the device status word.
 */
GLOWQ_API glowq_status glowq_group_solve(const glowq_solve_module* mods, int32_t m, int64_t d,
                                         const double* Sx_half, const double* Sx_half_pinv, int32_t r, int32_t p,
                                         int32_t q, const double* Omega, double* A, double* B, double* sing,
                                         double* g_ec, uint16_t* A16, uint16_t* B16, void* workspace,
                                         size_t workspace_bytes, void* stream);

/*
 * GlowQ-S selective restore (key design 4; about half of the units restored
 * in the pages' efficiency results).  Host-only.
 *   err_fro2[u] = ||E_u||_F^2, w_fro2[u] = ||W_u||_F^2  (host, n_units)
 *   layer_idx[u], kind[u]   tie-break / fallback keys  (host, n_units)
 *   k                       units to restore, 0..n_units
 * Ranking: descending g_ner = err/w; exact ties by ascending (layer, kind,
 * unit index).  Weak-signal fallback: if any score is NaN, or all scores lie
 * within a relative spread of 1e-6 of the largest, the ranking is the plain
 * layer order.  Outputs (host): restore_mask[u] = 1 for the first k units of
 * the ranking, order[0..n_units) = the ranking (may be NULL).
 * *used_fallback (may be NULL) is set to 1 when the layer order was used.
 */
GLOWQ_API glowq_status glowq_select_restore(const double* err_fro2, const double* w_fro2,
                                  const int32_t* layer_idx, const int32_t* kind,
                                  int32_t n_units, int32_t k, uint8_t* restore_mask,
                                  int32_t* order, int32_t* used_fallback);

/*
 * GlowQ-S selective restore by a caller-computed importance score (key
 * design 4 names two scores; the other one, the covariance-aligned GSVD
 * energy capture g_ec(u) = sum_{j<=r} sigma_j(M_u)^2 / ||M_u||_F^2, comes out
 * of the offline solve's core M_u).  Host-only.
 *   score[u]                 importance of unit u, larger = restore first (host, n_units)
 *   layer_idx, kind, k, restore_mask, order, used_fallback: as for
 *   glowq_select_restore, with the same tie-break and weak-signal fallback.
 * Errors: GLOWQ_ERR_ARG for n_units < 0, k outside 0..n_units, or a NULL
 * array with n_units > 0.
 */
GLOWQ_API glowq_status glowq_select_restore_scores(const double* score, const int32_t* layer_idx,
                                         const int32_t* kind, int32_t n_units, int32_t k,
                                         uint8_t* restore_mask, int32_t* order,
                                         int32_t* used_fallback);

/*
 * Per-row squared norms for g_ner: row_norms[2*o] = ||W[o] - w_hat[o]||^2 and
 * row_norms[2*o+1] = ||W[o]||^2 (fp64, deterministic), from a module's fp32
 * weight and its packed form.  Summing the rows of every module of a unit
 * gives err_fro2 and w_fro2 for glowq_select_restore.
 *   W          device, O x d fp32; qweight in the block layout (glowq_module)
 *   row_norms  device, 2*O doubles (caller-allocated); O % 16 == 0
 */
GLOWQ_API glowq_status glowq_error_norms(const float* W, const uint32_t* qweight,
                               const uint16_t* scales, const uint8_t* zeros,
                               int64_t O, int64_t d, double* row_norms, void* stream);

/* Reads and clears this device's status word (GLOWQ_OK, GLOWQ_ERR_TIMEOUT,
   GLOWQ_ERR_NUMERIC, or GLOWQ_ERR_ALIGN if a decode kernel found its shared
   memory base not 1 KB-aligned and skipped its work); synchronises `stream`
   first. */
GLOWQ_API glowq_status glowq_get_device_status(void* stream);

/*
 * Self-test of the failure path (no counterpart on the pages): enqueues one
 * single-thread kernel that waits on a shared-memory barrier nobody arrives
 * on, with the same bounded wait the forward kernels use, limited to `polls`
 * polls (1..65536).  The wait runs out, the kernel records GLOWQ_ERR_TIMEOUT
 * in the device status word and returns; the context stays usable.  Returns
 * GLOWQ_ERR_ARG for polls outside the range, GLOWQ_ERR_CUDA if the launch
 * fails, else GLOWQ_OK (read the outcome with glowq_get_device_status).
 */
GLOWQ_API glowq_status glowq_selftest_wait_timeout(uint32_t polls, void* stream);

/* Static description of a status code. */
GLOWQ_API const char* glowq_status_string(glowq_status s);

/* Library version, "major.minor.patch". */
GLOWQ_API const char* glowq_version(void);

#ifdef __cplusplus
}
#endif
#endif /* GLOWQ_H */
