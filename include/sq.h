/*
 * sq.h -- C ABI of libsq, the SquareQ W4 quantized linear layer on NVIDIA B200
 * (sm_100a).
 *
 * The layer (SquareQ README, section "SquareQ v3 -- W4 (Hadamard-256 +
 * low-rank + int4 / NVFP4)"):
 *
 *     W = lora_up . lora_down^T + inverse_H256( dequant( residual ) )
 *
 * H256 is the block-diagonal normalised Sylvester Hadamard matrix of order 256
 * over the input dimension K ("Rotation" paragraph); it is symmetric and
 * orthogonal, so inverse_H256 = H256.  The residual is stored either as int4
 * with fp16 group-32 scales chosen by an MSE sweep over scale fractions, or as
 * NVFP4 (e2m1 codes, ue4m3 scales per 16 values in the tiled scale layout, one
 * fp32 global scale) ("Residual codecs" paragraph).  lora_up / lora_down are
 * the rank-32 bf16 low-rank branch ("Low-rank branch" paragraph).
 *
 * Conventions for every entry point:
 *   - Pointers marked "device" must point to device memory of the current
 *     device; the library never allocates, frees, copies to the host or
 *     synchronises.  Work is enqueued on `stream` (a cudaStream_t passed as
 *     void*, NULL = legacy default stream) and runs asynchronously.
 *   - Matrices are row-major and densely packed.  bf16 and fp16 values are
 *     passed as their 16-bit patterns (uint16_t).
 *   - Arguments are validated on the host before anything is enqueued; a
 *     failed check returns a status and enqueues nothing.  A CUDA launch error
 *     returns SQ_ERR_CUDA.  There is no fallback path: a device other than
 *     compute capability 10.0 returns SQ_ERR_DEVICE.
 *   - Shapes: K % 256 == 0 (the rotation's block size), N % 128 == 0, M >= 1.
 *     All device pointers must be 16-byte aligned, workspaces 256-byte aligned.
 *   - Rounding: every narrowing conversion is round-to-nearest-even; fp32
 *     arithmetic follows the order stated for each operation, so integer and
 *     packed outputs are reproducible bit for bit.
 *   - Caller-owned workspace: its size comes from sq_workspace_bytes().  It
 *     must not be shared by calls that may run concurrently.
 */
#ifndef SQ_H
#define SQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SQ_API __attribute__((visibility("default")))
#else
#define SQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SQ_OK = 0,
    SQ_ERR_NULL = 1,       /* a required pointer is NULL                          */
    SQ_ERR_SHAPE = 2,      /* K % 256, N % 128, M < 1, group not 32/64, too large */
    SQ_ERR_ALIGN = 3,      /* pointer not 16-byte (workspace: 256-byte) aligned   */
    SQ_ERR_WORKSPACE = 4,  /* workspace smaller than sq_workspace_bytes()         */
    SQ_ERR_DEVICE = 5,     /* current device is not sm_100 (B200 class)          */
    SQ_ERR_CUDA = 6,       /* a CUDA call or launch failed                        */
    SQ_ERR_ARG = 7,        /* bad enum / flag value                               */
    SQ_ERR_TIMEOUT = 8,    /* a kernel gave up a bounded wait (device status word) */
    SQ_ERR_NONFINITE = 9,  /* SQ_CHECK_FINITE met a NaN or an infinity (status word) */
    SQ_ERR_INDEX = 10      /* a device-side index check failed and its access was
                              skipped (library built with SQ_DEBUG_CHECKS; status word) */
} sq_status;

typedef enum {
    SQ_FMT_INT4_G32 = 1,   /* int4 codes [N, K/2], fp16 scales [N, K/32]          */
    SQ_FMT_NVFP4 = 2,      /* e2m1 codes [N, K/2], ue4m3 tiled scales, fp32 g_w   */
    SQ_FMT_INT4_G64 = 3,   /* int4 codes [N, K/2], fp16 scales [N, K/64]          */
    SQ_FMT_INT8_ROW = 4    /* int8 codes [N, K], fp32 scales [N], rank-16 low rank */
} sq_format;

/* operations for sq_workspace_bytes() */
typedef enum {
    SQ_OP_BUILD_INT4 = 1,
    SQ_OP_BUILD_NVFP4 = 2,
    SQ_OP_ACT_QUANT_NVFP4 = 3,
    SQ_OP_LINEAR_FWD_NVFP4 = 4,
    SQ_OP_LINEAR_FWD_INT4 = 5,
    SQ_OP_RECONSTRUCT = 6,
    SQ_OP_LINEAR_FWD_INT8 = 7,
    SQ_OP_BUILD_INT8 = 8,
    SQ_OP_LINEAR_BWD_DX = 9,
    SQ_OP_SVD_INIT = 10
} sq_op;

/* flags */
#define SQ_ACT_STATIC_SCALE    0x1u  /* sq_act_quant_nvfp4 / sq_linear_fwd: *g_x is an input */
#define SQ_RECON_RESIDUAL_ONLY 0x2u  /* sq_reconstruct_bf16: drop the low-rank term        */
#define SQ_RECON_TRANSPOSED    0x4u  /* sq_reconstruct_bf16: write W^T [K, N] instead of W  */
#define SQ_OUT_BF16            0x8u  /* sq_linear_fwd(_noalloc): y is bf16 = bf16(y_fp32)   */
#define SQ_CHECK_FINITE        0x10u /* sq_act_quant_nvfp4 / sq_linear_fwd(_noalloc): scan x
                                        for NaN and infinities first; a hit sets the status
                                        word that sq_check_device_status reports as
                                        SQ_ERR_NONFINITE (the call itself still runs)      */

/*
 * A built weight.  All pointers are device pointers owned by the caller.
 *   fmt        SQ_FMT_INT4_G32, SQ_FMT_INT4_G64, SQ_FMT_NVFP4 or SQ_FMT_INT8_ROW
 *   N, K       output / input features (SQ_FMT_INT8_ROW: K <= 16384)
 *   codes      4-bit formats: [N, K/2] uint8, value 2k in the low nibble of
 *              byte k (int4: 4-bit two's complement in [-7, 7]; NVFP4: e2m1);
 *              SQ_FMT_INT8_ROW: [N, K] int8 in [-127, 127]
 *   scales     int4: fp16 bits [N, K/32] (group 32) or [N, K/64] (group 64);
 *              NVFP4: ue4m3 bytes in the tiled layout, sq_sf_bytes(N, K) bytes;
 *              SQ_FMT_INT8_ROW: fp32 [N], one per row
 *   g_w        NVFP4 only: 1 float, the per-tensor global scale
 *   lora_up    bf16 [N, 32] ([N, 16] for SQ_FMT_INT8_ROW), or NULL for no
 *              low-rank branch
 *   lora_down  bf16 [K, 32] ([K, 16] for SQ_FMT_INT8_ROW), or NULL for no
 *              low-rank branch
 */
typedef struct {
    int32_t fmt;
    int64_t N;
    int64_t K;
    const uint8_t *codes;
    const void *scales;
    const float *g_w;
    const uint16_t *lora_up;
    const uint16_t *lora_down;
} sq_weight;

/* Human-readable name of a status code (static string). */
SQ_API const char *sq_status_str(int status);

/* ABI version, currently 1. */
SQ_API int sq_abi_version(void);

/*
 * 1 if this library was built with SQ_DEBUG_CHECKS, else 0.  In such a build
 * the kernels that write the layer's outputs (the activation passes, the
 * NVFP4, int4 and int8 builders, the reconstructs) check every store's index
 * against the size of the buffer it writes before the store; a store that
 * would fall outside is skipped and sets bit 2 of the call's device status
 * word (the workspace's, or the library's own for calls without one), which
 * sq_check_device_status reports as SQ_ERR_INDEX.  Nothing traps.  The
 * results of a debug build are the same bits as those of a release build.
 */
SQ_API int sq_debug_checks(void);

/*
 * Text of the last failing CUDA call or device check made by this thread
 * inside libsq (static thread-local buffer; "" if none).
 */
SQ_API const char *sq_last_error_detail(void);

/*
 * Bytes of a tiled NVFP4 scale buffer for `rows` rows of K values:
 * ceil(rows/128)*128 * K/16.  The layout is the public cuBLAS / tcgen05
 * 1D block-scaling layout: 512-byte tiles of 128 rows x 4 scales; scale
 * (r, c), C = K/16, sits at byte
 *   ((r/128)*(C/4) + c/4)*512 + (r%32)*16 + ((r%128)/32)*4 + c%4.
 * Rows past `rows` up to the next multiple of 128 hold 0.
 */
SQ_API size_t sq_sf_bytes(int64_t rows, int64_t K);

/* Workspace bytes an operation needs for the given shape (M unused for builds). */
SQ_API size_t sq_workspace_bytes(int op, int64_t M, int64_t N, int64_t K);

/*
 * int4 builder (SquareQ README, "Residual codecs": int4 codes with one scale
 * per group of 32 or 64 values, its fraction of the absmax chosen by MSE).  For each row of R [N, K] fp32 (device): rotate
 * every 256-block with H256, then for each group of `group` (32 or 64)
 * rotated values r_i with a = max|r_i| try the fractions f_j = (50 + 2j)/100,
 * j = 0..25:
 *   s_j = fp16(RN(RN(f_j a) / 7)),  q_i = clamp(rint(RN(r_i RN(1/s_j))), -7, 7),
 *   error_j = sum over an xor butterfly (strides 16,8,4,2,1) of RN((r_i - q_i s_j)^2)
 * for each 32 consecutive values (group 64: the two 32-value sums added,
 * RN(first + second)); a scale of 0 gives q = 0 and error r_i^2.  Keep the
 * smallest error, the smaller j on ties.  Outputs (device): codes [N, K/2],
 * scales fp16 bits [N, K/group], frac_idx [N, K/group] winning j (may be
 * NULL).  The weight is then SQ_FMT_INT4_G32 or SQ_FMT_INT4_G64.  Rotated
 * values must stay below 458000 in magnitude (fp16 scale range).
 */
SQ_API sq_status sq_build_int4(const float *R, int64_t N, int64_t K, int32_t group,
                        uint8_t *codes, uint16_t *scales, uint8_t *frac_idx,
                        void *stream);

/*
 * SVD init of the low-rank branch (SquareQ README, "Low-rank branch": a
 * rank-32 bf16 branch from the weight's SVD; "v3.1 -- int8-residual mode": rank 16):
 * the step before the builders.  From W [N, K] fp32 (device) it writes, for
 * the `rank` (32, or 16 for SQ_FMT_INT8_ROW) largest singular values sigma,
 * lora_up = bf16(U sqrt(sigma)) [N, rank] and lora_down = bf16(V sqrt(sigma))
 * [K, rank] (an even split between the factors), and the residual
 *   R[n, k] = RN(W[n, k] - L[n, k]),  L = fmaf chain of the bf16 factors over
 *   the rank as in sq_reconstruct_bf16,
 * fp32 [N, K] (device; R may equal W).  The singular subspace is found by
 * `iters` (1..100) rounds of subspace iteration on 32 columns from the
 * caller's start block omega [K, 32] fp32 (device; e.g. seeded N(0, 1)
 * draws): each round one product with W and one with W^T (fp32, fixed
 * summation order), each followed by CholeskyQR with fp64 Grams (twice for the
 * final U).  With B = W^T U from the last round, the Cholesky factor of B^T B
 * and a one-sided Jacobi iteration on its columns give sigma and the rotation
 * of the factors.  Deterministic for a given shape and omega.  The accuracy of
 * the rank-r product against the exact truncated SVD improves as
 * (sigma_33 / sigma_r)^(2 iters); R is RN(W - L) of whatever factors result
 * (it absorbs what they miss).
 * ws: sq_workspace_bytes(SQ_OP_SVD_INIT, 0, N, K) bytes, 256-byte aligned,
 * caller-owned.  Errors: SQ_ERR_NULL, SQ_ERR_SHAPE (N, K as for the builders),
 * SQ_ERR_ARG (iters, rank), SQ_ERR_ALIGN (16 bytes; ws 256), SQ_ERR_WORKSPACE,
 * and SQ_ERR_CUDA with sq_last_error_detail() naming the launch that failed.
 */
SQ_API sq_status sq_svd_init(const float *W, int64_t N, int64_t K, const float *omega, int32_t iters,
                             int32_t rank, uint16_t *lora_up, uint16_t *lora_down, float *R, void *ws,
                             size_t ws_bytes, void *stream);

/*
 * int8 per-row builder (SquareQ README, "v3.1 -- int8-residual mode": the
 * rotated residual of a rank-16 branch in int8, one MSE-chosen scale per row).  For each row of
 * R [N, K] fp32 (device, K <= 16384): rotate every 256-block with H256; with
 * a = max|r_k| over the row try the fractions f_j = (50 + 2j)/100,
 * j = 0..25, of the int4 sweep:
 *   s_j = RN(RN(f_j a) / 127) (fp32),  q_k = clamp(rint(RN(r_k RN(1/s_j))), -127, 127),
 *   error_j = sum of RN(fmaf(-q_k, s_j, r_k)^2): per 256-block, each 32-value
 *             group by the xor butterfly (strides 16, 8, 4, 2, 1), the 8 group
 *             sums by a butterfly over the group index (strides 4, 2, 1), then
 *             the blocks added in order from block 0
 * (a scale of 0 gives q = 0 and error r_k^2); keep the smallest error, the
 * smaller j on ties.  Outputs (device): codes [N, K] int8, scales [N] fp32,
 * frac_idx [N] winning j (may be NULL).  The weight is SQ_FMT_INT8_ROW, whose
 * low-rank branch has rank 16.
 */
SQ_API sq_status sq_build_int8(const float *R, int64_t N, int64_t K, int8_t *codes, float *scales,
                               uint8_t *frac_idx, void *stream);

/*
 * NVFP4 builder (SquareQ README, "Residual codecs": e2m1 codes, one ue4m3
 * scale per 16 values in the tiled order, one fp32 scale for the tensor).  Pass 1 rotates R
 * [N, K] fp32 (device) and takes A = max|H R|; g_w = RN(A / 2688), i.e.
 * A / (6 * 448).  Pass 2 rotates again and, per 16 values with b = max|r|:
 *   sf = ue4m3(RN(b / RN(6 g_w))),  code_i = e2m1(RN(r_i RN(1 / RN(value(sf) g_w))))
 * (sf == 0 or g_w == 0 gives zero codes; negative values rounding to 0 keep
 * the sign bit, code 0x8).  Outputs (device): codes [N, K/2], sf_tiled
 * (sq_sf_bytes(N, K) bytes), g_w (1 float).  ws: sq_workspace_bytes(
 * SQ_OP_BUILD_NVFP4, 0, N, K) bytes of device scratch (holds the absmax).
 */
SQ_API sq_status sq_build_nvfp4(const float *R, int64_t N, int64_t K,
                         uint8_t *codes, uint8_t *sf_tiled, float *g_w,
                         void *ws, size_t ws_bytes, void *stream);

/*
 * Activation quantisation, the prologue of the NVFP4 forward (SquareQ README,
 * the op-level parity paragraph of the FP4 forward: the Hadamard rotation, block
 * quantisation and tiled scales of x, fused in front of the GEMM).  x [M, K] bf16 (device) is rotated; g_x = RN(max|H x| / 2688)
 * unless SQ_ACT_STATIC_SCALE is set, in which case *g_x (device) is read as
 * given.  Then the same block-16 step as sq_build_nvfp4 with g_x.  Outputs
 * (device): codes [M, K/2], sf_tiled (sq_sf_bytes(M, K) bytes, padding rows
 * 0), g_x (written unless static).  If lora_down (bf16 [K, 32]) and t are
 * both non-NULL, also t[m, r] = sum_k x[m, k] lora_down[k, r] as fp32 [M, 32]
 * (the low-rank input; fp32 accumulation, order unspecified but fixed for a
 * given M and K, so t is the same on every run).  ws: sq_workspace_bytes(
 * SQ_OP_ACT_QUANT_NVFP4, M, 0, K) bytes (the status word, the absmax and,
 * when K is split over several CTAs, their partial t tiles).  flags:
 * SQ_ACT_STATIC_SCALE, SQ_CHECK_FINITE (the status word is the first 4 bytes
 * of ws).
 */
SQ_API sq_status sq_act_quant_nvfp4(const uint16_t *x, int64_t M, int64_t K,
                             uint8_t *codes, uint8_t *sf_tiled, float *g_x,
                             const uint16_t *lora_down, float *t, uint32_t flags,
                             void *ws, size_t ws_bytes, void *stream);

/*
 * Forward y = x W^T (SquareQ README, the op-level parity paragraph of the FP4
 * forward: rotation, block quantisation and tiled scales of x, the
 * GEMM and its epilogue; "Residual codecs": the int4 codec runs dequant-first;
 * "v3.1 -- int8-residual mode" for int8).
 * y [M, N] fp32 (device; with SQ_OUT_BF16 bf16, the
 * round-to-nearest-even of the same fp32 value, rounded once in the GEMM's
 * epilogue), x [M, K] bf16 (device).
 * Because H is symmetric, x W^T = H(x) deq(Q)^T + (x lora_down) lora_up^T.
 *   NVFP4: the activation prologue above, then a block-scaled e2m1 x e2m1
 *          tensor-core GEMM (tcgen05, fp32 accumulation in tensor memory),
 *          y = g_x g_w acc + t lora_up^T.
 *   int4:  "dequant-first": xb = bf16(H x), wb = bf16(q s), y = xb wb^T +
 *          t lora_up^T on bf16 tensor cores (fp32 accumulation); either
 *          group size (SQ_FMT_INT4_G32 / _G64).  The GEMM's own warps
 *          dequantise each 256-row tile of W once into a ring of R such tiles
 *          in the workspace (R x 256 x K bf16), from which the GEMM loads it;
 *          R = min(ceil(N / 256), ceil(74 / ceil(M / 256)) + 2), the tiles in
 *          flight at once: at M = 4480, 7 tiles whatever N is.
 *   int8:  the same with wb = bf16(RN(q s_row)) and the rank-16 branch
 *          (SQ_FMT_INT8_ROW; workspace op SQ_OP_LINEAR_FWD_INT8).
 * The low-rank term is accumulated on the tensor cores in the same
 * accumulator.  Accuracy: max|y - y_exact| / max|y_exact| <= 2e-3 against the
 * exact result on the same quantised operands (fp32 y; a bf16 y adds its own
 * rounding, up to 2^-9 of |y|).  flags: SQ_ACT_STATIC_SCALE
 * (NVFP4; *g_x is then an input, g_x must be non-NULL), SQ_OUT_BF16,
 * SQ_CHECK_FINITE.  g_x (device, may be NULL unless static) receives the
 * activation global scale.  ws:
 * sq_workspace_bytes(SQ_OP_LINEAR_FWD_NVFP4 or _INT4, M, N, K) bytes.
 */
SQ_API sq_status sq_linear_fwd(const sq_weight *w, const uint16_t *x, int64_t M, void *y,
                        float *g_x, uint32_t flags, void *ws, size_t ws_bytes,
                        void *stream);

/*
 * sq_linear_fwd without a caller workspace.  The SquareQ pages have no
 * counterpart of this call: it is a library convenience for callers that
 * cannot allocate device memory at the point of the forward -- plain C hosts
 * without a device allocator of their own, and latency-critical loops where
 * cudaMalloc (which may synchronise the device, and may fail under memory
 * pressure) is not allowed.  Nothing is allocated: the workspace is a fixed
 * 96 MiB scratch array in libsq's own device memory, one per device.
 *
 * Same arguments, results and accuracy as sq_linear_fwd, minus (ws,
 * ws_bytes).  scratch_out (host, may be NULL) receives the device address of
 * the scratch this call used; pass it to sq_check_device_status to read the
 * call's device status word.
 *
 * Limit: sq_workspace_bytes(SQ_OP_LINEAR_FWD_NVFP4, _INT4 or _INT8, M, N,
 * K) must be at most 100663296 (96 MiB); larger shapes return
 * SQ_ERR_WORKSPACE before any work, with the sizes in
 * sq_last_error_detail().  (At N = 16384, K = 6144: NVFP4 fits M up to
 * 26544 rows; int4, which needs bf16(H x) (M K 2 bytes) and its W ring
 * (R x 256 x K x 2 bytes, see sq_linear_fwd), fits M from 513 to 6536
 * rows; below 513 rows R grows towards all 64 tiles of W.)
 *
 * The first call on each device looks up the scratch's address
 * (cudaGetSymbolAddress, with that device current), which may load libsq's
 * device code; make that first call before any stream capture.  The address
 * is kept with the ID of the CUDA context it was looked up in and looked up
 * again in a new context (after cudaDeviceReset, or after the primary context
 * was released and created again), so a call never uses an address from a
 * context that no longer exists.  Nothing has
 * to start at zero: each call clears the status word and the absmax
 * accumulator at the start of its own stream work, like sq_linear_fwd.
 *
 * All calls on a device share the one scratch: calls that may overlap on the
 * device (different streams without an event between them, or several host
 * threads) race on it and give wrong results.  Order them on one stream.
 */
SQ_API sq_status sq_linear_fwd_noalloc(const sq_weight *w, const uint16_t *x, int64_t M, void *y,
                                       float *g_x, uint32_t flags, void **scratch_out, void *stream);

/*
 * bf16 reconstruct of W for the backward pass (SquareQ README, the op-level parity
 * paragraph: the backward rebuilds W in bf16 from the forward's payload).  For each element
 *   d = q s (int4, either group size), RN(q s_row) (int8) or
 *       RN(RN(e2m1 value(sf)) g_w) (NVFP4),
 *   h = H256 applied to each 256-block of d along K,
 *   L = fmaf(U[n,R-1], D[k,R-1], ... fmaf(U[n,0], D[k,0], 0)), R the rank
 *       (32; 16 for SQ_FMT_INT8_ROW),
 *   W[n, k] = bf16(RN(L + h))          (bf16(h) with SQ_RECON_RESIDUAL_ONLY
 *                                       or NULL low-rank pointers).
 * W_out: [N, K] bf16 (device), or with SQ_RECON_TRANSPOSED the same values as
 * W^T [K, N] (the layout the backward GEMM reads).  With the low-rank term the
 * kernel's producer and consumer warps hand tiles over through bounded waits;
 * a wait that gives up (a fault of the library, never expected) stops the
 * kernel early and sets the library's status word, which
 * sq_check_device_status(NULL, stream) reports as SQ_ERR_TIMEOUT.
 */
SQ_API sq_status sq_reconstruct_bf16(const sq_weight *w, uint16_t *W_out, uint32_t flags,
                              void *stream);

/*
 * Backward of the layer's input: dx = dy W, dy [M, N] bf16 (device), dx [M, K]
 * fp32 (device), W the bf16 reconstruct of the weight (low-rank term
 * included when the weight has one).  In the SquareQ README the backward
 * rebuilds W in bf16 from the forward's payload and then runs an ordinary bf16
 * GEMM ("End-to-end" paragraph); here the reconstruct writes W^T into
 * the workspace and the library's bf16 tensor-core GEMM (fp32 accumulation in
 * tensor memory) reduces over N.  Accuracy: max|dx - dx_exact| /
 * max|dx_exact| <= 2e-3 against dy W on the same bf16 operands.  ws:
 * sq_workspace_bytes(SQ_OP_LINEAR_BWD_DX, M, N, K) bytes (holds W^T).
 */
SQ_API sq_status sq_linear_bwd_dx(const sq_weight *w, const uint16_t *dy, int64_t M, float *dx, void *ws,
                                  size_t ws_bytes, void *stream);

/*
 * Optional instrumentation for timing the tensor-core GEMM on its own: when
 * both handles are non-NULL, every later sq_linear_fwd or sq_linear_bwd_dx call
 * made by this host thread records start_event immediately before and
 * stop_event immediately after its GEMM launch, on the call's stream.  The handles are cudaEvent_t
 * values passed as void*, created and owned by the caller; (NULL, NULL) turns
 * recording off.  No work is added or skipped.
 */
SQ_API sq_status sq_set_gemm_events(void *start_event, void *stop_event);

/*
 * The same instrumentation for any of the launches below (SQ_STAGE_GEMM is
 * what sq_set_gemm_events sets): SQ_STAGE_ACT_PASS1 brackets the activation
 * pass that takes max|H x| and t = x lora_down (sq_act_quant_nvfp4 and the
 * NVFP4 sq_linear_fwd), SQ_STAGE_ACT_QUANT the pass that quantises H x.  An
 * event between two launches keeps the second one from starting its set-up
 * early (the launches overlap otherwise), so a timed call is a little slower
 * than an untimed one.  Returns SQ_ERR_ARG for an unknown stage.
 */
#define SQ_STAGE_GEMM       0
#define SQ_STAGE_ACT_PASS1  1
#define SQ_STAGE_ACT_QUANT  2
#define SQ_STAGE_COUNT      3
SQ_API sq_status sq_set_stage_events(int32_t stage, void *start_event, void *stop_event);

/*
 * Read back and clear the device status word that a kernel sets when it gives
 * up a bounded wait (SQ_ERR_TIMEOUT), or that the SQ_CHECK_FINITE scan sets
 * on a NaN or an infinity in x (SQ_ERR_NONFINITE; a timeout is reported
 * first); ws is the workspace of the sq_linear_fwd
 * call to check (each such call clears the word when it starts).  With ws ==
 * NULL it reads the library's own word on the current device, which the calls
 * without a workspace (sq_reconstruct_bf16) set instead.  This call
 * synchronises `stream` and copies 4 bytes to the host.
 */
SQ_API sq_status sq_check_device_status(void *ws, void *stream);

/*
 * Self-test of the device-side index check (any build): one thread checks the
 * index one past a bound of 256 with the same routine the SQ_DEBUG_CHECKS
 * kernels use.  The check fails, the (never made) access is skipped and bit 2
 * of the status word at ws is set; sq_check_device_status(ws, stream) then
 * returns SQ_ERR_INDEX and the context stays usable.  ws: at least 256 bytes
 * of device memory (only the first word is used), 256-byte aligned.
 */
SQ_API sq_status sq_selftest_index_check(void *ws, void *stream);

/*
 * Self-test of the failure detection every kernel relies on: all waits in the
 * library are bounded; a kernel that gives up a wait sets the status word of
 * its workspace and returns (no trap), and sq_check_device_status reports
 * SQ_ERR_TIMEOUT.  This call launches one kernel whose wait can never be
 * satisfied, with a limit of limit_us microseconds (1 .. 1000000), on `stream`:
 * afterwards sq_check_device_status(ws, stream) must return SQ_ERR_TIMEOUT and
 * the context stays usable.  ws: at least 256 bytes of device memory (only
 * the status word is written).
 */
SQ_API sq_status sq_selftest_wait_timeout(void *ws, uint32_t limit_us, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SQ_H */
