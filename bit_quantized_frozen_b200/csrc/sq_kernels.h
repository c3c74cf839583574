// sq_kernels.h -- internal launchers of libsq (not part of the C ABI).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace sq {

// low-rank operands of the NVFP4 forward (and the final t of the activation
// quantiser), written by the activation quant kernel before its blocks
// (t_part == nullptr: nothing to write)
struct LowrankOut {
    const float *t_part = nullptr;   // [parts, M, 32] fp32 partial tiles of t = x lora_down (summed in order)
    int parts = 1;
    float *t_out = nullptr;          // [M, 32] fp32 t, or NULL
    const float *g_w = nullptr;      // weight global scale (beta = g_x g_w)
    uint16_t *tsplit = nullptr;      // [M, 64] bf16, or NULL
    const uint16_t *U = nullptr;     // lora_up [N, 32] bf16
    int64_t N = 0;
    uint16_t *udup = nullptr;        // [N, 64] bf16, or NULL
};

// K split of the activation pass that computes t = x lora_down: the pass
// writes this many partial [M, 32] tiles (1: t itself), a function of the
// shape only, so t is the same on every device for a given shape
int act_t_parts(int64_t M, int64_t K);

cudaError_t launch_absmax_rot_f32(const float *in, int64_t rows, int64_t K, uint32_t *amax, int sms,
                                  cudaStream_t s);
cudaError_t launch_absmax_rot_bf16(const uint16_t *in, int64_t rows, int64_t K, uint32_t *amax, int sms,
                                   cudaStream_t s);
cudaError_t launch_nvfp4_quant_f32(const float *in, int64_t rows, int64_t K, const uint32_t *amax,
                                   const float *g_static, float *g_out, uint8_t *codes, uint8_t *sf, int sms,
                                   cudaStream_t s);
cudaError_t launch_nvfp4_quant_bf16(const uint16_t *in, int64_t rows, int64_t K, const uint32_t *amax,
                                    const float *g_static, float *g_out, uint8_t *codes, uint8_t *sf,
                                    const LowrankOut &lr, uint32_t *status, int sms, cudaStream_t s);
cudaError_t launch_int4_build(const float *R, int64_t N, int64_t K, int group, uint8_t *codes, uint16_t *scales,
                              uint8_t *frac, int sms, cudaStream_t s);
// int8 per-row builder (K <= 16384) and the rank-16 -> rank-32 widening
cudaError_t launch_int8_build(const float *R, int64_t N, int64_t K, int8_t *codes, float *scales, uint8_t *frac,
                              int sms, cudaStream_t s);
cudaError_t launch_widen_rank16(const uint16_t *src, int64_t rows, uint16_t *dst, int sms, cudaStream_t s);
// t_part: act_t_parts(M, K) partial tiles [parts, M, 32] (NULL: no t)
cudaError_t launch_act_pass1(const uint16_t *x, int64_t M, int64_t K, const uint16_t *D, uint32_t *amax,
                             float *t_part, uint16_t *xb, uint32_t *status, int sms, cudaStream_t s);
cudaError_t launch_lowrank_finish(const float *t_part, int parts, int64_t M, const float *g_x, const float *g_w,
                                  uint16_t *tsplit, const uint16_t *U, int64_t N, uint16_t *udup, int sms,
                                  cudaStream_t s);
// the library's own device status word (set by kernels of calls without a workspace)
cudaError_t library_status_word(uint32_t **p);

// sets kStatusNonfinite in *status if any of the n bf16 values of x is a NaN or an infinity
cudaError_t launch_check_finite_bf16(const uint16_t *x, int64_t n, uint32_t *status, int sms, cudaStream_t s);

// fmt: 1 int4 group 32, 2 NVFP4, 3 int4 group 64, 4 int8 per row (rank 16)
cudaError_t launch_reconstruct(int fmt, const uint8_t *codes, const void *scales, const float *g_w,
                               const uint16_t *U, const uint16_t *D, int64_t N, int64_t K, int with_lowrank,
                               int transposed, uint16_t *W, int sms, cudaStream_t s);

// SVD init of the low-rank branch (sq_svd.cu): omega [K, 32] fp32 start block, output rank 32
// or 16 (up [N, rank], down [K, rank], R with the rank-r chain); on an error *stage names the
// launch that reported it
size_t svd_workspace_bytes(int64_t N, int64_t K);
cudaError_t launch_svd_init(const float *W, int64_t N, int64_t K, const float *omega, int iters, int rank,
                            uint16_t *up, uint16_t *down, float *R, void *ws, int sms, cudaStream_t s,
                            const char **stage);

// forward GEMM y = beta (A B^T + tsplit udup^T), see sq_gemm.cu
// B operand of the GEMM: bf16 by TMA, NVFP4 codes + tiled scales by TMA, or
// int4 / int8 payload turned into bf16(q s) in shared memory by the kernel
enum GemmMode { kGemmBf16 = 0, kGemmNvfp4 = 1, kGemmInt4G32 = 2, kGemmInt4G64 = 3, kGemmInt8 = 4 };

struct GemmLaunch {
    int mode;                // GemmMode
    const void *a;           // [M, K/2] u8 (NVFP4) or [M, K] bf16
    const void *b;           // [N, K/2] u8 (NVFP4, int4), [N, K] int8 or [N, K] bf16
    const void *b_scales;    // int4: fp16 [N, K/G]; int8: fp32 [N]
    uint16_t *wring;         // int4 / int8: W ring [ring_slots * 256, K] bf16 (workspace)
    uint32_t *ring_ctr;      // int4 / int8: 2 * ring_slots counters, zero before the launch
    int ring_slots;
    const uint8_t *sfa;      // NVFP4 scales of a (tiled)
    const uint8_t *sfb;      // NVFP4 scales of b (tiled)
    const float *g_x;        // NVFP4: device scalars, beta = g_x * g_w
    const float *g_w;
    const uint16_t *tsplit;  // [M, 64] bf16 or NULL (no low-rank step)
    const uint16_t *udup;    // [N, 64] bf16 or NULL
    void *y;                 // [M, N] fp32, or bf16 with out_bf16
    int out_bf16;            // 1: y = bf16(RNE) of the fp32 result
    uint32_t *status;        // device status word
    int64_t M, N, K;
};

cudaError_t launch_gemm(const GemmLaunch &g, int sms, cudaStream_t stream);

// ID of the current CUDA context (unique for the life of the process; a context created
// after cudaDeviceReset gets a new one), 0 if it cannot be read.  Per-device caches of
// symbol addresses and function attributes are keyed on it: a new context loads the
// library's device code again, so those have to be looked up or set again.
unsigned long long current_context_id();

// 2D row-major tensor map [rows, inner] of esize-byte elements, box [box_rows, box_inner]
bool make_tmap(CUtensorMap *m, CUtensorMapDataType dt, int esize, const void *base, uint64_t inner,
               uint64_t rows, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw);

}  // namespace sq
