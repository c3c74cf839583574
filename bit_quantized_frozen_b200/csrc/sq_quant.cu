// sq_quant.cu -- the non-GEMM kernels of the SquareQ W4 layer: the NVFP4
// builder (Hadamard-256 + tensor absmax, then block quantisation into the
// tiled scale layout), the int4 and int8 builders with their scale-fraction
// sweeps, the activation prologue of the forwards (absmax, bf16(H x) and t on
// tcgen05 in one read of x, then the NVFP4 quantisation), the low-rank
// operands, and the bf16 reconstructs.  (The int4 / int8 weight is
// dequantised inside the GEMM, sq_gemm.cu.)
//
// What bounds each: the NVFP4 builder's passes stream HBM; the int4 / int8
// builders are bound by the FP32 / ALU issue of their 26-trial sweeps; the
// reconstruct with the low-rank term by the FMA pipe (its rank-r fmaf chain)
// and the latency of its decode and transform; the activation passes and the
// residual-only reconstruct by the L1 data pipe (Hadamard shuffles) and the
// FP32 pipe, below their HBM floors.  Persistent grids are sized from the
// SM count; loads and stores are contiguous per warp or go through TMA.  They
// follow the SquareQ README, section "SquareQ v3 -- W4", as stated operation
// by operation in include/sq.h.
#include "sq_kernels.h"
#include "sq_device.cuh"
#include "sq_ptx.cuh"

namespace sq {

// the library's own device status word, for kernels whose call takes no
// workspace (timeouts of bounded waits, failed index checks of debug builds)
__device__ uint32_t g_library_status;

// ---------------------------------------------------------------------------
// Block streamer.  The input ([rows, K], K % 256 == 0) is viewed as a 2-D
// tensor of 32-value rows; a producer warp (warp 8) TMA-loads chunks of 256
// such rows (32 Hadamard blocks) into a ring of shared-memory stages, with the
// 128-byte (fp32) or 64-byte (bf16) swizzle so that eight consumer warps can
// each read their own 32-value row conflict free.  Consumer warp w, lane L
// gets row 32w + L of the chunk: block 4w + L/8, values 32(L%8)..+31 -- the
// layout of fwht256_l32.  Rows past the tensor are zero-filled by the TMA.
// ---------------------------------------------------------------------------
constexpr int kStreamConsumers = 8;
constexpr int kStreamThreads = 32 * (kStreamConsumers + 1);

template <typename T>
struct StreamCfg {
    static constexpr int kStages = sizeof(T) == 4 ? 3 : 4;
    static constexpr int kChunkBytes = 32 * kHad * (int)sizeof(T);            // 32 blocks
    static constexpr int kSmem = kStages * kChunkBytes + 2 * kStages * 8 + 16 + 1024;
};

template <typename T>
__device__ __forceinline__ void read_row(const uint8_t *buf, int row, float (&v)[32])
{
    if (sizeof(T) == 4) {          // 128-byte rows, chunk i at i ^ (row & 7)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 a = *reinterpret_cast<const float4 *>(buf + row * 128 + 16 * (i ^ (row & 7)));
            v[4 * i] = a.x; v[4 * i + 1] = a.y; v[4 * i + 2] = a.z; v[4 * i + 3] = a.w;
        }
    } else {                       // 64-byte rows, chunk i at i ^ ((row >> 1) & 3)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 a = *reinterpret_cast<const uint4 *>(buf + row * 64 + 16 * (i ^ ((row >> 1) & 3)));
            const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                v[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
                v[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
            }
        }
    }
}

// Runs f(block, v, valid) on every 256-block of the stream, one call per lane
// per chunk in consumer warps (all 32 lanes of a warp call f together, so f
// may shuffle).  total_blocks may exceed the tensor (zero blocks).  pre(c) is
// run once by every consumer thread c (0 .. 32 * consumers - 1) before its
// first chunk, while the first loads are in flight.
struct NoPrologue {
    __device__ void operator()(int) const {}
};

template <typename T, typename F, typename P = NoPrologue>
__device__ __forceinline__ void stream_blocks(const CUtensorMap *tm, int64_t total_blocks, uint32_t *status, F &&f,
                                              P &&pre = P())
{
    using Cfg = StreamCfg<T>;
    extern __shared__ uint8_t stream_smem_raw[];
    uint8_t *smem =
        reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(stream_smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kStages * Cfg::kChunkBytes);
    const uint32_t full = smem_u32(bars), empty = smem_u32(bars + Cfg::kStages);
    volatile uint32_t *abort_flag = reinterpret_cast<uint32_t *>(bars + 2 * Cfg::kStages);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int st = 0; st < Cfg::kStages; ++st) {
            mbar_init(full + 8 * st, 1);
            mbar_init(empty + 8 * st, kStreamConsumers);
        }
        *abort_flag = 0u;
        fence_mbar_init();
    }
    __syncthreads();
    const int64_t chunks = (total_blocks + 31) / 32;
    if (warp == kStreamConsumers) {
        if (lane == 0) {
            prefetch_tmap(tm);
            int it = 0;
            for (int64_t c = blockIdx.x; c < chunks; c += gridDim.x, ++it) {
                const int st = it % Cfg::kStages;
                const uint32_t ph = (uint32_t)(it / Cfg::kStages) & 1u;
                if (!mbar_wait(empty + 8 * st, ph ^ 1u, abort_flag, status))
                    break;
                mbar_arrive_expect_tx(full + 8 * st, Cfg::kChunkBytes);
                tma_load_2d(smem_u32(smem + st * Cfg::kChunkBytes), tm, 0, (int32_t)(c * 256), full + 8 * st);
            }
        }
        __syncwarp();
    } else {
        pre(threadIdx.x);
        int it = 0;
        for (int64_t c = blockIdx.x; c < chunks; c += gridDim.x, ++it) {
            const int st = it % Cfg::kStages;
            const uint32_t ph = (uint32_t)(it / Cfg::kStages) & 1u;
            int ok = 1;
            if (lane == 0)
                ok = mbar_wait(full + 8 * st, ph, abort_flag, status) ? 1 : 0;
            if (__shfl_sync(0xffffffffu, ok, 0) == 0)
                break;
            float v[32];
            read_row<T>(smem + st * Cfg::kChunkBytes, 32 * warp + lane, v);
            __syncwarp();
            if (lane == 0)
                mbar_arrive(empty + 8 * st);
            const int64_t block = 32 * c + 4 * warp + (lane >> 3);
            f(block, v, block < total_blocks);
        }
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------
// pass 1 of the NVFP4 builder: A = max |H in| over a [rows, K] matrix, folded
// into *amax (u32 bits of a non-negative float)
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kStreamThreads) absmax_rot_kernel(const __grid_constant__ CUtensorMap tm,
                                                                    int64_t blocks, uint32_t *__restrict__ amax)
{
    const int lane = threadIdx.x & 31;
    grid_dep_launch();                              // the quantisation pass may start loading
    float m = 0.0f;
    stream_blocks<T>(&tm, blocks, nullptr, [&](int64_t, float (&v)[32], bool) {
        fwht256_l32<false>(v, lane);
#pragma unroll
        for (int i = 0; i < 32; i += 2)
            m = fmax3(m, fabsf(v[i]), fabsf(v[i + 1]));
    });
    // max |v / 16| == (max |v|) / 16 bit for bit: rounding is monotonic
    m = __fmul_rn(m, 0.0625f);
#pragma unroll
    for (int x = 16; x >= 1; x >>= 1)
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, x));
    __shared__ float wmax[kStreamConsumers + 1];
    if (lane == 0)
        wmax[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float b = 0.0f;
        for (int w = 0; w < kStreamConsumers; ++w)
            b = fmaxf(b, wmax[w]);
        atomic_max_nonneg(amax, b);
    }
}

// ---------------------------------------------------------------------------
// low-rank operands of the forward's extra MMA step.  With beta = g_x g_w (1
// when either scale is absent or the product is 0): tt = t / beta,
// tsplit[m] = [bf16(tt) | bf16(tt - bf16(tt))] (bf16 [M, 64]), and
// udup[n] = [U[n] | U[n]] (bf16 [N, 64]).
// ---------------------------------------------------------------------------
__device__ __forceinline__ float lowrank_beta(float g_x, const float *g_w)
{
    if (!g_w)
        return 1.0f;
    const float b = __fmul_rn(g_x, *g_w);
    return b == 0.0f ? 1.0f : b;
}

// unit i < M*8: t[m, 4c..4c+3] = the sum of the `parts` partial t tiles in
// order (tp[j] = t_part + j*M*32), written to t_out (when non-NULL) and split
// into both halves of tsplit[m] (when non-NULL) (m = i/8, c = i%8);
// unit i >= M*8: 16-byte chunk c of U[n] -> both halves of udup[n] (n, c from i - M*8)
__device__ __forceinline__ void lowrank_unit(int64_t i, int64_t nT, const float *__restrict__ t_part, int parts,
                                             float *__restrict__ t_out, float beta, uint16_t *__restrict__ tsplit,
                                             const uint16_t *__restrict__ U, uint16_t *__restrict__ udup)
{
    if (i < nT) {
        const int64_t m = i >> 3, c = i & 7;
        const int64_t M = nT >> 3;
        float4 t4 = *reinterpret_cast<const float4 *>(t_part + m * kRank + 4 * c);
        for (int j = 1; j < parts; ++j) {
            const float4 a = *reinterpret_cast<const float4 *>(t_part + (j * M + m) * kRank + 4 * c);
            t4.x = __fadd_rn(t4.x, a.x);
            t4.y = __fadd_rn(t4.y, a.y);
            t4.z = __fadd_rn(t4.z, a.z);
            t4.w = __fadd_rn(t4.w, a.w);
        }
        if (t_out)
            *reinterpret_cast<float4 *>(t_out + m * kRank + 4 * c) = t4;
        if (!tsplit)
            return;
        const float tv[4] = {t4.x, t4.y, t4.z, t4.w};
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float tt = __fdiv_rn(tv[k], beta);
            hi[k] = f32_to_bf16_bits(tt);
            lo[k] = f32_to_bf16_bits(__fsub_rn(tt, bf16_bits_to_f32(hi[k])));
        }
        *reinterpret_cast<uint2 *>(tsplit + m * 64 + 4 * c) = make_uint2(hi[0] | (hi[1] << 16), hi[2] | (hi[3] << 16));
        *reinterpret_cast<uint2 *>(tsplit + m * 64 + 32 + 4 * c) =
            make_uint2(lo[0] | (lo[1] << 16), lo[2] | (lo[3] << 16));
    } else if (udup) {
        const int64_t j = i - nT;
        const int64_t n = j >> 2, c = j & 3;
        const uint4 u = *reinterpret_cast<const uint4 *>(U + n * kRank + 8 * c);
        *reinterpret_cast<uint4 *>(udup + n * 64 + 8 * c) = u;
        *reinterpret_cast<uint4 *>(udup + n * 64 + 32 + 8 * c) = u;
    }
}

// ---------------------------------------------------------------------------
// NVFP4 block quantisation of H in with global scale g, over rows_pad rows
// (a multiple of 128): rows past `rows` are zero and only their scale bytes
// are written (as 0), which fills the tiled layout's padding.  g comes from
// *g_static when non-NULL, else RN(A / 2688) from *amax, and is stored to
// *g_out (when non-NULL) by thread 0 of block 0.  Each lane owns two whole
// 16-value blocks, so block maxima and scales need no shuffles.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kStreamThreads) nvfp4_quant_kernel(const __grid_constant__ CUtensorMap tm,
                                                                     int64_t rows, int64_t rows_pad, int64_t K,
                                                                     const uint32_t *__restrict__ amax,
                                                                     const float *__restrict__ g_static,
                                                                     float *__restrict__ g_out,
                                                                     uint8_t *__restrict__ codes,
                                                                     uint8_t *__restrict__ sf, LowrankOut lr)
{
    const int lane = threadIdx.x & 31;
    const int q = lane & 7;
    grid_dep_launch();
    // amax (and t) come from the preceding pass: the consumers wait for it before
    // their first block, the producer starts streaming at once
    float g = 0.0f, sixg = 0.0f;
    const int64_t kb_per_row = K / kHad;
    const int64_t C = K / kSfBlock;
    const bool idx32 = rows_pad * kb_per_row <= (int64_t)UINT32_MAX;
    // the forward's low-rank operands (g is final here), done while the first chunks load
    auto lowrank = [&](int c) {
        grid_dep_wait();
        g = g_static ? *g_static : __fdiv_rn(__uint_as_float(*amax), 2688.0f);
        sixg = __fmul_rn(6.0f, g);
        if (g_out && blockIdx.x == 0 && c == 0)
            *g_out = g;
        if (!lr.t_part)
            return;
        const float beta = lowrank_beta(g, lr.g_w);
        const int64_t nT = rows * 8, total = nT + (lr.udup ? lr.N * 4 : 0);
        const int64_t stride = (int64_t)gridDim.x * (32 * kStreamConsumers);
        for (int64_t i = (int64_t)blockIdx.x * (32 * kStreamConsumers) + c; i < total; i += stride)
            lowrank_unit(i, nT, lr.t_part, lr.parts, lr.t_out, beta, lr.tsplit, lr.U, lr.udup);
    };
    stream_blocks<T>(&tm, rows_pad * kb_per_row, nullptr, [&](int64_t b, float (&v)[32], bool valid) {
        fwht256_l32(v, lane);
        if (!valid)
            return;
        const int64_t row = idx32 ? (int64_t)((uint32_t)b / (uint32_t)kb_per_row) : b / kb_per_row;
        const int64_t kb = b - row * kb_per_row;
        uint32_t word[4];
        uint32_t sfc[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float bmax = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; i += 2)
                bmax = fmax3(bmax, fabsf(v[16 * h + i]), fabsf(v[16 * h + i + 1]));
            uint32_t code = 0;
            uint32_t w0 = 0, w1 = 0;
            if (g != 0.0f) {
                code = to_ue4m3(__fdiv_rn(bmax, sixg));
                if (code != 0) {
                    const float inv = __frcp_rn(__fmul_rn(ue4m3_value(code), g));
                    const uint64_t inv2 = f2_pack(inv, inv);
                    float s[16];
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        f2_unpack(f2_mul(f2_pack(v[16 * h + 2 * i], v[16 * h + 2 * i + 1]), inv2), s[2 * i],
                                  s[2 * i + 1]);
                    w0 = to_e2m1x4(s[0], s[1], s[2], s[3]) | (to_e2m1x4(s[4], s[5], s[6], s[7]) << 16);
                    w1 = to_e2m1x4(s[8], s[9], s[10], s[11]) | (to_e2m1x4(s[12], s[13], s[14], s[15]) << 16);
                }
            }
            word[2 * h] = w0;
            word[2 * h + 1] = w1;
            sfc[h] = code;
        }
        if (row < rows && SQ_DCHECK(row * (K / 2) + kb * (kHad / 2) + 16 * q + 16 <= rows * (K / 2), &g_library_status))
            *reinterpret_cast<uint4 *>(codes + row * (K / 2) + kb * (kHad / 2) + 16 * q) =
                make_uint4(word[0], word[1], word[2], word[3]);
        // scale columns 2q, 2q+1 of the block are adjacent bytes of the tiled layout
        if (SQ_DCHECK(sf_offset(row, kb * (kHad / kSfBlock) + 2 * q, C) + 2 <= rows_pad * C, &g_library_status))
            *reinterpret_cast<uint16_t *>(sf + sf_offset(row, kb * (kHad / kSfBlock) + 2 * q, C)) =
            (uint16_t)(sfc[0] | (sfc[1] << 8));
    }, lowrank);
}

// ---------------------------------------------------------------------------
// int4 builder, group 32 or 64.  With the 8-lane Hadamard layout every lane
// holds 32 consecutive rotated values: one whole group of 32 (group index
// 8 * block + lane % 8), or one half of a group of 64 whose other half sits in
// the neighbouring lane (lane ^ 1; group index 4 * block + (lane % 8) / 2).
// Each lane sweeps the 26 scale fractions in registers; for group 64 the two
// lanes of a pair share the absmax and add their half errors.
// ---------------------------------------------------------------------------
// sum of RN((r_i - q_i s)^2) over 32 values, as lane 0 of an xor butterfly over
// strides 16, 8, 4, 2, 1; rp holds the 32 rotated values as pairs (r_2j, r_2j+1).
// q = clamp(rint(r inv), -QMAX, QMAX): |r inv| <= 2 QMAX < 2^22, so adding and
// subtracting 1.5 * 2^23 rounds to the nearest integer, ties to even, exactly
// like rint (and on the FMA pipe, not the conversion unit).  The error is
// fma(-q, s, r): r - q s with one rounding (for int4, q s is exact anyway).
template <int QMAX = 7>
__device__ __forceinline__ float group_sq_error(const uint64_t (&rp)[16], float s, float inv)
{
    uint64_t p[16];
    if (s == 0.0f) {                                   // q = 0: error r^2
#pragma unroll
        for (int j = 0; j < 16; ++j)
            p[j] = f2_mul(rp[j], rp[j]);
    } else {
        constexpr float kRound = 12582912.0f;          // 1.5 * 2^23
        const uint64_t inv2 = f2_pack(inv, inv), nsn = f2_pack(-s, -s);
        const uint64_t rnd = f2_pack(kRound, kRound);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            float t0, t1;
            f2_unpack(f2_add(f2_mul(rp[j], inv2), rnd), t0, t1);
            t0 = fminf(fmaxf(t0, kRound - (float)QMAX), kRound + (float)QMAX);
            t1 = fminf(fmaxf(t1, kRound - (float)QMAX), kRound + (float)QMAX);
            const uint64_t q = f2_sub(f2_pack(t0, t1), rnd);
            const uint64_t e = f2_fma(q, nsn, rp[j]);
            p[j] = f2_mul(e, e);
        }
    }
    // strides 16, 8, 4, 2 are pair strides 8, 4, 2, 1; stride 1 adds the two halves of pair 0
#pragma unroll
    for (int d = 8; d >= 1; d >>= 1)
#pragma unroll
        for (int j = 0; j < d; ++j)
            p[j] = f2_add(p[j], p[j + d]);
    float lo, hi;
    f2_unpack(p[0], lo, hi);
    return __fadd_rn(lo, hi);
}

// the swept scale fractions RN((50 + 2j) / 100), j = 0..25 (folded at compile time, IEEE rounding)
__constant__ float kFrac[26] = {
    50.0f / 100, 52.0f / 100, 54.0f / 100, 56.0f / 100, 58.0f / 100, 60.0f / 100, 62.0f / 100,
    64.0f / 100, 66.0f / 100, 68.0f / 100, 70.0f / 100, 72.0f / 100, 74.0f / 100, 76.0f / 100,
    78.0f / 100, 80.0f / 100, 82.0f / 100, 84.0f / 100, 86.0f / 100, 88.0f / 100, 90.0f / 100,
    92.0f / 100, 94.0f / 100, 96.0f / 100, 98.0f / 100, 100.0f / 100};

template <int G>
__global__ void __launch_bounds__(kStreamThreads, 2) int4_build_kernel(const __grid_constant__ CUtensorMap tm,
                                                                    int64_t blocks, uint8_t *__restrict__ codes,
                                                                    uint16_t *__restrict__ scales,
                                                                    uint8_t *__restrict__ frac)
{
    static_assert(G == 32 || G == 64, "group 32 or 64");
    const int lane = threadIdx.x & 31;
    stream_blocks<float>(&tm, blocks, nullptr, [&](int64_t b, float (&r)[32], bool valid) {
        fwht256_l32(r, lane);
        // group 64: both lanes of a pair run the sweep (shuffles), so no lane leaves before it;
        // blocks past the tensor are zero-filled and only their stores are skipped
        if (G == 32 && !valid)
            return;
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; i += 2)
            a = fmax3(a, fabsf(r[i]), fabsf(r[i + 1]));
        if (G == 64)
            a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
        uint64_t rp[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
            rp[j] = f2_pack(r[2 * j], r[2 * j + 1]);
        float best = 0.0f, best_s = 0.0f;
        uint16_t best_h = 0;
        int best_j = 0;
#pragma unroll 1
        for (int j = 0; j < kFracCount; ++j) {
            const float f = kFrac[j];
            const __half hs = __float2half_rn(__fdiv_rn(__fmul_rn(f, a), 7.0f));
            const float s = __half2float(hs);
            const float inv = s == 0.0f ? 0.0f : __frcp_rn(s);
            float mse = group_sq_error<7>(rp, s, inv);
            if (G == 64)                               // first half + second half (addition commutes)
                mse = __fadd_rn(mse, __shfl_xor_sync(0xffffffffu, mse, 1));
            if (j == 0 || mse < best) {
                best = mse;
                best_j = j;
                best_s = s;
                best_h = __half_as_ushort(hs);
            }
        }
        if (!valid)
            return;
        // codes for the winning scale (same arithmetic as in the sweep)
        const float inv = best_s == 0.0f ? 0.0f : __frcp_rn(best_s);
        uint32_t word[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
            float r0, r1;
            f2_unpack(rp[i >> 1], r0, r1);
            int q0 = 0, q1 = 0;
            if (best_s != 0.0f) {
                q0 = (int)fminf(fmaxf(rintf(__fmul_rn(r0, inv)), -7.0f), 7.0f);
                q1 = (int)fminf(fmaxf(rintf(__fmul_rn(r1, inv)), -7.0f), 7.0f);
            }
            word[i >> 3] |= (((uint32_t)q0 & 0xFu) | (((uint32_t)q1 & 0xFu) << 4)) << (4 * (i & 7));
        }
        const int64_t hidx = 8 * b + (lane & 7);     // flat index of this lane's 32 values
        if (!SQ_DCHECK(hidx < 8 * blocks, &g_library_status))
            return;
        reinterpret_cast<uint4 *>(codes)[hidx] = make_uint4(word[0], word[1], word[2], word[3]);
        if (G == 32 || (lane & 1) == 0) {
            const int64_t gidx = G == 32 ? hidx : hidx >> 1;
            scales[gidx] = best_h;
            if (frac)
                frac[gidx] = (uint8_t)best_j;
        }
    });
}

// ---------------------------------------------------------------------------
// int8 per-row builder (v3.1 int8-residual mode).  One CTA of 256 threads per
// row at a time (persistent over rows).  The row is copied into shared memory
// (16-byte chunk c of each lane's 128-byte piece at slot c ^ lane%8, so the 8
// lanes of a block read 8 different bank groups), rotated in place by 8-lane
// groups (group i takes blocks i, i + 32, ...), and its absmax reduced.  Each
// group then sweeps the 26 scales over its blocks with the values in
// registers: per block, the 32-value butterfly in each lane and a butterfly
// over the 8 lanes (strides 4, 2, 1) give the block's error, stored per
// (fraction, block); 26 threads then add the blocks of their fraction in
// order, and the smallest sum (first on ties) picks the scale.  Finally each
// group quantises its blocks and writes 32 int8 codes per lane.
// ---------------------------------------------------------------------------
constexpr int kI8Threads = 256;
constexpr int kI8MaxK = 16384;

__host__ __device__ constexpr int i8_smem_bytes(int K)
{
    return K * 4 + kFracCount * (K / kHad) * 4 + 3 * kFracCount * 4 + 64;
}

__device__ __forceinline__ int i8_slot(int block, int q, int c)   // float4 index in the shared row
{
    return block * 64 + q * 8 + (c ^ q);
}

__global__ void __launch_bounds__(kI8Threads) int8_build_kernel(const float *__restrict__ R, int64_t N, int K,
                                                                int8_t *__restrict__ codes,
                                                                float *__restrict__ scales,
                                                                uint8_t *__restrict__ frac)
{
    extern __shared__ __align__(16) uint8_t i8_smem[];
    float4 *row = reinterpret_cast<float4 *>(i8_smem);                        // K floats, swizzled
    float *berr = reinterpret_cast<float *>(i8_smem + K * 4);                  // [26][nb] block errors
    float *stab = berr + kFracCount * (K / kHad);                              // [26] scales, [26] errors
    float *etab = stab + kFracCount;
    float *itab = etab + kFracCount;                                           // [26] RN(1 / scale)
    float *red = itab + kFracCount;                                            // [8] warp maxima, choice
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int q = lane & 7;
    const int grp = tid >> 3;                                                  // 8-lane group, 0..31
    const int nb = K / kHad;
    const int iters = (nb + 31) / 32;                                          // blocks per group (max)

    for (int64_t n = blockIdx.x; n < N; n += gridDim.x) {
        // copy the row (float4 f of the row -> block f/64, lane (f/8)%8, chunk f%8)
        const float4 *src = reinterpret_cast<const float4 *>(R + n * K);
        for (int f = tid; f < K / 4; f += kI8Threads)
            row[i8_slot(f >> 6, (f >> 3) & 7, f & 7)] = __ldg(src + f);
        __syncthreads();
        // rotate in place, absmax
        float a = 0.0f;
        for (int it = 0; it < iters; ++it) {
            const int b = grp + 32 * it;
            const bool valid = b < nb;                 // the whole warp runs the shuffles
            float v[32];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float4 x = valid ? row[i8_slot(b, q, c)] : make_float4(0.f, 0.f, 0.f, 0.f);
                v[4 * c] = x.x; v[4 * c + 1] = x.y; v[4 * c + 2] = x.z; v[4 * c + 3] = x.w;
            }
            fwht256_l32(v, lane);
            if (valid) {
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    row[i8_slot(b, q, c)] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
#pragma unroll
                for (int i = 0; i < 32; i += 2)
                    a = fmax3(a, fabsf(v[i]), fabsf(v[i + 1]));
            }
        }
#pragma unroll
        for (int x = 16; x >= 1; x >>= 1)
            a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, x));
        if (lane == 0)
            red[warp] = a;
        __syncthreads();
        if (tid < kFracCount) {
            float m = 0.0f;
            for (int w = 0; w < kI8Threads / 32; ++w)
                m = fmaxf(m, red[w]);
            const float sj = __fdiv_rn(__fmul_rn(kFrac[tid], m), 127.0f);
            stab[tid] = sj;
            itab[tid] = sj == 0.0f ? 0.0f : __frcp_rn(sj);
        }
        __syncthreads();
        // sweep: per block and fraction, the block's error
        for (int it = 0; it < iters; ++it) {
            const int b = grp + 32 * it;
            const bool valid = b < nb;
            uint64_t rp[16];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float4 x = valid ? row[i8_slot(b, q, c)] : make_float4(0.f, 0.f, 0.f, 0.f);
                rp[2 * c] = f2_pack(x.x, x.y);
                rp[2 * c + 1] = f2_pack(x.z, x.w);
            }
#pragma unroll 1
            for (int j = 0; j < kFracCount; ++j) {
                const float sj = stab[j], inv = itab[j];
                float e = group_sq_error<127>(rp, sj, inv);
                e = __fadd_rn(e, __shfl_xor_sync(0xffffffffu, e, 4));
                e = __fadd_rn(e, __shfl_xor_sync(0xffffffffu, e, 2));
                e = __fadd_rn(e, __shfl_xor_sync(0xffffffffu, e, 1));
                if (valid && q == 0)
                    berr[j * nb + b] = e;
            }
        }
        __syncthreads();
        if (tid < kFracCount) {                        // blocks in order, per fraction
            float E = berr[tid * nb];
            for (int b = 1; b < nb; ++b)
                E = __fadd_rn(E, berr[tid * nb + b]);
            etab[tid] = E;
        }
        __syncthreads();
        int best_j = 0;
        {
            float best = etab[0];
            for (int j = 1; j < kFracCount; ++j)
                if (etab[j] < best) {
                    best = etab[j];
                    best_j = j;
                }
        }
        const float s = stab[best_j];
        const float inv = s == 0.0f ? 0.0f : __frcp_rn(s);
        // codes
        for (int it = 0; it < iters; ++it) {
            const int b = grp + 32 * it;
            if (b >= nb)
                break;
            uint32_t w[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float4 x = row[i8_slot(b, q, c)];
                const float xv[4] = {x.x, x.y, x.z, x.w};
                uint32_t word = 0;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    int qi = 0;
                    if (s != 0.0f)
                        qi = (int)fminf(fmaxf(rintf(__fmul_rn(xv[k], inv)), -127.0f), 127.0f);
                    word |= ((uint32_t)qi & 0xFFu) << (8 * k);
                }
                w[c] = word;
            }
            if (!SQ_DCHECK(n < N && (int64_t)b * kHad + 32 * q + 32 <= K, &g_library_status))
                continue;
            uint4 *dst = reinterpret_cast<uint4 *>(codes + n * K + (int64_t)b * kHad + 32 * q);
            dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
            dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
        }
        if (tid == 0) {
            scales[n] = s;
            if (frac)
                frac[n] = (uint8_t)best_j;
        }
        __syncthreads();                               // the shared row is free for the next one
    }
}

// rank-16 low-rank factors widened to rank 32 with zero columns 16..31, so the
// rank-32 forward machinery (t = x lora_down, the low-rank MMA step) adds
// exactly the rank-16 term: src [rows, 16] bf16 -> dst [rows, 32] bf16
__global__ void __launch_bounds__(256) widen_rank16_kernel(const uint4 *__restrict__ src, int64_t rows,
                                                           uint4 *__restrict__ dst)
{
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < rows * 4;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i >> 2, c = i & 3;       // 16-byte chunk c of dst row r
        dst[i] = c < 2 ? __ldg(src + 2 * r + c) : make_uint4(0u, 0u, 0u, 0u);
    }
}

// ---------------------------------------------------------------------------
// Activation pass 1: one read of x for up to three results.
//   amax (optional):   max |H x| over the whole tensor (the activation global
//                      scale's input), from the 4-lane Hadamard transform;
//   xb (optional):     bf16(H x) [M, K], the A operand of the int4 / int8
//                      forward (the same transform, then the exact 1/16 and one
//                      rounding to bf16);
//   t_part (optional): t = x . lora_down on the tcgen05 tensor cores (fp32
//                      accumulation in tensor memory), as `split` partial
//                      [M, 32] tiles, one per range of K, which the consumer
//                      adds in order (t is deterministic for a given shape).
// A CTA owns 128 rows (the MMA's M) and one of `split` ranges of 256-column
// chunks (blockIdx.x = tile * split + range).  One producer warp streams each
// chunk -- the x tile (128 x 256, four TMA boxes of 64 columns, 128-byte
// swizzle) and the lora_down tile (256 x 32, one box, 64-byte swizzle) --
// into a 2-deep ring; sixteen consumer warps each transform eight rows
// (fwht256_q4_unscaled) and release the stage as soon as their rows are in
// registers; one thread issues the chunk's 16 MMAs (M = 128, N = 32, K = 16)
// straight from the stage.
// ---------------------------------------------------------------------------
constexpr int kP1Rows = 128;
constexpr int kP1BoxBytes = kP1Rows * 128;          // 128 rows x 64 bf16
constexpr int kP1XBytes = 4 * kP1BoxBytes;          // 64 KB
constexpr int kP1DBytes = kHad * kRank * 2;         // 16 KB
constexpr int kP1BufBytes = kP1XBytes + kP1DBytes;
constexpr int kP1Stages = 2;
constexpr int kP1Consumers = 16;                    // 8 rows each
constexpr int kP1Threads = 32 * (kP1Consumers + 2);   // + TMA producer warp + MMA warp
constexpr int kP1Smem = kP1Stages * kP1BufBytes + 1024 + 256;   // ring, 1 KB alignment, barriers
constexpr int kP1MaxSplit = 16;
constexpr int kP1SplitSms = 148;                    // K split sized for one CTA per SM of a B200

int act_t_parts(int64_t M, int64_t K)
{
    const int64_t tiles = (M + kP1Rows - 1) / kP1Rows;
    const int64_t nkb = K / kHad;
    int64_t split = kP1SplitSms / (tiles < 1 ? 1 : tiles);
    split = split < 1 ? 1 : split;
    split = split > kP1MaxSplit ? kP1MaxSplit : split;
    split = split > nkb ? nkb : split;
    return (int)split;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

__device__ __forceinline__ void cp_async_commit()
{
    asm volatile("cp.async.commit_group;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// barrier over the first `threads` threads of the CTA (named barrier 1)
__device__ __forceinline__ void bar_sync_named(uint32_t threads)
{
    asm volatile("bar.sync 1, %0;" ::"r"(threads) : "memory");
}

// t = x . lora_down on the tensor cores: per chunk 16 MMAs (M = 128, N = 32,
// K = 16, bf16 -> fp32 in tensor memory).  A is the x stage (K-major, 128B
// swizzle, four boxes of 128 rows); B is the lora_down stage, N-major (32
// values of a k-row are one 64-byte swizzled row).
constexpr uint32_t kP1Idesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(kRank >> 3) << 17) |
                              ((uint32_t)(128 >> 4) << 24);
__device__ __forceinline__ uint64_t p1_bdesc(uint32_t saddr)
{
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1u << 16) | ((uint64_t)(512u >> 4) << 32) |
           ((uint64_t)1u << 46) | ((uint64_t)4u << 61);
}

__global__ void __launch_bounds__(kP1Threads, 1) act_pass1_kernel(const __grid_constant__ CUtensorMap tmx,
                                                                  const __grid_constant__ CUtensorMap tmd,
                                                                  int64_t M, int64_t K, uint32_t *__restrict__ amax,
                                                                  float *__restrict__ t_part, int split,
                                                                  uint16_t *__restrict__ xb,
                                                                  uint32_t *__restrict__ status)
{
    float *const t32 = t_part;                        // non-NULL: this CTA writes partial tile j of t
    extern __shared__ uint8_t p1_raw[];
    uint8_t *p1_smem =
        reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p1_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(p1_smem + kP1Stages * kP1BufBytes);
    const uint32_t full = smem_u32(bars), empty = smem_u32(bars + kP1Stages);
    const uint32_t done = smem_u32(bars + 2 * kP1Stages);                  // every MMA finished
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + 2 * kP1Stages + 1);
    volatile uint32_t *abort_flag = tmem_holder + 1;
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int j = (int)(blockIdx.x % (unsigned)split);       // range of K chunks
    const int64_t m0 = (int64_t)(blockIdx.x / (unsigned)split) * kP1Rows;
    const int nkb = (int)(K / kHad);
    const int kb0 = (int)((int64_t)j * nkb / split);
    const int nch = (int)((int64_t)(j + 1) * nkb / split) - kb0;
    const uint32_t sbase = smem_u32(p1_smem);
    if (tid == 0) {
        for (int st = 0; st < kP1Stages; ++st) {
            mbar_init(full + 8 * st, 1);
            mbar_init(empty + 8 * st, ((amax || xb) ? kP1Consumers : 0) + (t32 ? 1 : 0));
        }
        mbar_init(done, 1);
        *abort_flag = 0u;
        fence_mbar_init();
    }
    if (t32 && warp == kP1Consumers + 1) {
        tmem_alloc(smem_u32(tmem_holder), 32);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = t32 ? *tmem_holder : 0u;
    grid_dep_launch();                                // the quantisation pass may start loading x

    float m = 0.0f;
    if (warp == kP1Consumers) {                       // TMA producer
        if (lane == 0) {
            prefetch_tmap(&tmx);
            if (t32)
                prefetch_tmap(&tmd);
            for (int c = 0; c < nch; ++c) {
                const int st = c % kP1Stages;
                const uint32_t ph = (uint32_t)(c / kP1Stages) & 1u;
                if (!mbar_wait(empty + 8 * st, ph ^ 1u, abort_flag, status))
                    break;
                mbar_arrive_expect_tx(full + 8 * st, t32 ? kP1BufBytes : kP1XBytes);
                const uint32_t xs = sbase + st * kP1BufBytes;
                const int kb = kb0 + c;
#pragma unroll
                for (int b = 0; b < 4; ++b)
                    tma_load_2d(xs + kP1BoxBytes * b, &tmx, kb * kHad + 64 * b, (int32_t)m0, full + 8 * st);
                if (t32)
                    tma_load_2d(xs + kP1XBytes, &tmd, 0, kb * kHad, full + 8 * st);
            }
        }
        __syncwarp();
    } else if (warp == kP1Consumers + 1) {            // MMA issuer: t
        if (t32 && lane == 0) {
            bool ok = true;
            for (int c = 0; c < nch && ok; ++c) {
                const int st = c % kP1Stages;
                const uint32_t ph = (uint32_t)(c / kP1Stages) & 1u;
                if (!mbar_wait(full + 8 * st, ph, abort_flag, status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t xs = sbase + st * kP1BufBytes;
                const uint64_t da = sdesc_sw128(xs), db = p1_bdesc(xs + kP1XBytes);
#pragma unroll
                for (int ks = 0; ks < 16; ++ks)           // k-step: columns 16ks..16ks+15 of the chunk
                    mma_bf16(tmem_base, da + (uint64_t)((ks >> 2) * (kP1BoxBytes >> 4) + (ks & 3) * 2),
                             db + (uint64_t)(ks * 64), kP1Idesc, (c > 0 || ks > 0) ? 1u : 0u);
                tc_commit(empty + 8 * st);
            }
            tc_commit(done);
        }
        __syncwarp();
    } else if (amax || xb) {                          // consumers: Hadamard absmax and / or bf16(H x)
        // lane (q, r) = (lane / 8, lane % 8) holds quarter q of row 8 warp + r: 64 values of box q
        const int q = lane >> 3;
        const int R = 8 * warp + (lane & 7);
        const bool row_live = m0 + R < M;
        for (int c = 0; c < nch; ++c) {
            const int st = c % kP1Stages;
            const uint32_t ph = (uint32_t)(c / kP1Stages) & 1u;
            int ok = 1;
            if (lane == 0)
                ok = mbar_wait(full + 8 * st, ph, abort_flag, status) ? 1 : 0;
            if (__shfl_sync(0xffffffffu, ok, 0) == 0)
                break;
            uint64_t p[32];
            load_row64_bf16_sw128_s1(p1_smem + st * kP1BufBytes + q * kP1BoxBytes, R, p);
            __syncwarp();
            if (lane == 0)
                mbar_arrive(empty + 8 * st);              // the stage's rows are in registers
            fwht256_q4_from_s2(p, lane);
            if (amax) {
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    float lo, hi;
                    f2_unpack(p[i], lo, hi);
                    m = fmax3(m, fabsf(lo), fabsf(hi));
                }
            }
            if (xb && row_live) {                     // bf16(H x): elements 64q .. 64q+63 of the block
                const int64_t col = (int64_t)(kb0 + c) * kHad + 64 * q;
                if (SQ_DCHECK(col + 64 <= K, status)) {
                    uint4 *o = reinterpret_cast<uint4 *>(xb + (m0 + R) * K + col);
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        uint32_t w4[4];
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj) {
                            float lo, hi;
                            f2_unpack(p[4 * k + jj], lo, hi);
                            w4[jj] = f32x2_to_bf16x2_bits(__fmul_rn(lo, 0.0625f), __fmul_rn(hi, 0.0625f));
                        }
                        o[k] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    }
                }
            }
        }
    }
    __syncthreads();                                  // every role's loop is done

    // t rows of this CTA: warp w < 4 reads tensor-memory lanes 32w..32w+31 once every MMA
    // finished and stores its rows of partial tile j (row m0 + 32w + lane, 128 contiguous bytes)
    __shared__ float wmax[kP1Consumers + 2];
    if (t32 && warp < 4) {
        uint32_t tr[32];
        int ok = 1;
        if (lane == 0)
            ok = mbar_wait(done, 0, abort_flag, status) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        tc_fence_after();
        if (ok) {
            tmem_ld_32cols(tmem_base + ((uint32_t)(32 * warp) << 16), tr);
            tmem_wait_ld();
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
                tr[i] = 0u;
        }
        tc_fence_before();
        const int64_t row = m0 + 32 * warp + lane;
        if (row < M && SQ_DCHECK(j < split, status)) {
            float4 *o = reinterpret_cast<float4 *>(t32 + ((int64_t)j * M + row) * kRank);
#pragma unroll
            for (int i = 0; i < 32; i += 4)
                o[i / 4] = make_float4(__uint_as_float(tr[i]), __uint_as_float(tr[i + 1]),
                                       __uint_as_float(tr[i + 2]), __uint_as_float(tr[i + 3]));
        }
    }
    if (amax) {
        m = __fmul_rn(m, 0.0625f);                    // the transform's 1/16, once (exact for a max)
#pragma unroll
        for (int xx = 16; xx >= 1; xx >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, xx));
    }
    if (lane == 0)
        wmax[warp] = m;
    __syncthreads();                                  // tensor memory read, maxima stored
    if (t32 && warp == kP1Consumers + 1)
        tmem_dealloc(tmem_base, 32);
    if (amax && tid == 0) {
        float b = 0.0f;
        for (int w = 0; w < kP1Consumers; ++w)
            b = fmaxf(b, wmax[w]);
        atomic_max_nonneg(amax, b);
    }
}

// ---------------------------------------------------------------------------
// Activation pass 2: NVFP4 block quantisation of H x with the global scale g
// into codes [M, K/2] and the tiled scales (rows_pad = M rounded up to 128;
// rows past M are zero and only their scale bytes are written, as 0, which
// fills the tiled layout's padding).  g comes from *g_static when non-NULL,
// else RN(A / 2688) from *amax, and is stored to *g_out (when non-NULL) by
// thread 0 of block 0.  The forward's low-rank operands (LowrankOut) are
// written first, while the first chunks load.
// Work unit: 64 rows x one 256-column chunk, four TMA boxes of 64 x 64 bf16
// (128-byte swizzle) in a 3-deep ring; consumer warp w takes rows 8w..8w+7 in
// the 4-lane layout, so each lane owns four whole 16-value scale blocks and
// writes 32 code bytes and 4 scale bytes.  The reciprocals RN(1 / RN(value(sf)
// g)) depend only on the scale code: a table of the 126 finite non-zero codes
// is built once per CTA.
// ---------------------------------------------------------------------------
constexpr int kAQRows = 64;
constexpr int kAQBoxBytes = kAQRows * 128;          // 64 rows x 64 bf16
constexpr int kAQBytes = 4 * kAQBoxBytes;           // 32 KB
constexpr int kAQStages = 3;
constexpr int kAQConsumers = 8;
constexpr int kAQThreads = 32 * (kAQConsumers + 1);
constexpr int kAQSmem = kAQStages * kAQBytes + 1024 + 256 + 128 * 4;   // ring, alignment, barriers, table

__global__ void __launch_bounds__(kAQThreads, 2) act_quant_kernel(const __grid_constant__ CUtensorMap tmx,
                                                                  int64_t M, int64_t rows_pad, int64_t K,
                                                                  const uint32_t *__restrict__ amax,
                                                                  const float *__restrict__ g_static,
                                                                  float *__restrict__ g_out,
                                                                  uint8_t *__restrict__ codes,
                                                                  uint8_t *__restrict__ sf, LowrankOut lr,
                                                                  uint32_t *__restrict__ status)
{
    extern __shared__ uint8_t aq_raw[];
    uint8_t *aq_smem =
        reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(aq_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(aq_smem + kAQStages * kAQBytes);
    const uint32_t full = smem_u32(bars), empty = smem_u32(bars + kAQStages);
    volatile uint32_t *abort_flag = reinterpret_cast<uint32_t *>(bars + 2 * kAQStages);
    float *inv_tab = reinterpret_cast<float *>(aq_smem + kAQStages * kAQBytes + 256);
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    grid_dep_launch();                                // the GEMM may start its set-up
    if (tid == 0) {
        for (int st = 0; st < kAQStages; ++st) {
            mbar_init(full + 8 * st, 1);
            mbar_init(empty + 8 * st, kAQConsumers);
        }
        *abort_flag = 0u;
        fence_mbar_init();
    }
    __syncthreads();
    const int64_t nkb = K / kHad;
    const int64_t units = rows_pad / kAQRows * nkb;
    if (warp == kAQConsumers) {                       // TMA producer: x does not depend on pass 1
        if (lane == 0) {
            prefetch_tmap(&tmx);
            int it = 0;
            for (int64_t u = blockIdx.x; u < units; u += gridDim.x, ++it) {
                const int st = it % kAQStages;
                const uint32_t ph = (uint32_t)(it / kAQStages) & 1u;
                if (!mbar_wait(empty + 8 * st, ph ^ 1u, abort_flag, status))
                    break;
                const int64_t rt = u / nkb, kb = u - rt * nkb;
                mbar_arrive_expect_tx(full + 8 * st, kAQBytes);
                const uint32_t xs = smem_u32(aq_smem + st * kAQBytes);
#pragma unroll
                for (int b = 0; b < 4; ++b)
                    tma_load_2d(xs + kAQBoxBytes * b, &tmx, (int32_t)(kb * kHad + 64 * b), (int32_t)(rt * kAQRows),
                                full + 8 * st);
            }
        }
        __syncwarp();
        return;
    }
    // ---- consumers: the global scale, the reciprocal table, the low-rank operands
    grid_dep_wait();                                  // amax and t of pass 1 are final
    const float g = g_static ? *g_static : __fdiv_rn(__uint_as_float(*amax), 2688.0f);
    const float sixg = __fmul_rn(6.0f, g);
    if (g_out && blockIdx.x == 0 && tid == 0)
        *g_out = g;
    // inv_tab[c] = RN(1 / RN(value(c) g)) for the finite non-zero codes 1..126;
    // entry 127 (not a finite code) counts the entries whose /16 would round
    if (tid < 128)
        inv_tab[tid] = 0.0f;
    bar_sync_named(32 * kAQConsumers);
    if (tid >= 1 && tid <= 126 && g != 0.0f) {
        const float inv = __frcp_rn(__fmul_rn(ue4m3_value((uint32_t)tid), g));
        inv_tab[tid] = inv;
        if (__fmul_rn(__fmul_rn(inv, 0.0625f), 16.0f) != inv)
            atomicAdd(&inv_tab[127], 1.0f);
    }
    if (lr.t_part) {
        const float beta = lowrank_beta(g, lr.g_w);
        const int64_t nT = M * 8, total = nT + (lr.udup ? lr.N * 4 : 0);
        const int64_t stride = (int64_t)gridDim.x * (32 * kAQConsumers);
        for (int64_t i = (int64_t)blockIdx.x * (32 * kAQConsumers) + tid; i < total; i += stride)
            lowrank_unit(i, nT, lr.t_part, lr.parts, lr.t_out, beta, lr.tsplit, lr.U, lr.udup);
    }
    bar_sync_named(32 * kAQConsumers);                // the table is complete
    // With A >= 2^-100 (the codec's precondition) and every table entry still exact
    // after a further /16, RN(RN(v / 16) inv) = RN(v (inv / 16)) for every value that
    // can give a non-zero code (v / 16 is then a normal number), and both are a zero of
    // the same sign otherwise: one multiply per value instead of two.
    const bool fold16 = g >= 0x1p-100f / 2688.0f && inv_tab[127] == 0.0f;
    const int q = lane >> 3;
    const int R = 8 * warp + (lane & 7);
    const uint32_t C = (uint32_t)(K / kSfBlock);
    const uint32_t nkb32 = (uint32_t)nkb;
    const uint32_t step_rt = gridDim.x / nkb32, step_kb = gridDim.x % nkb32;
    uint32_t rt = blockIdx.x / nkb32, kb = blockIdx.x % nkb32;
    int it = 0;
    for (int64_t u = blockIdx.x; u < units; u += gridDim.x, ++it) {
        const int st = it % kAQStages;
        const uint32_t ph = (uint32_t)(it / kAQStages) & 1u;
        int ok = 1;
        if (lane == 0)
            ok = mbar_wait(full + 8 * st, ph, abort_flag, status) ? 1 : 0;
        if (__shfl_sync(0xffffffffu, ok, 0) == 0)
            break;
        uint64_t p[32];
        load_row64_bf16_sw128_s1(aq_smem + st * kAQBytes + q * kAQBoxBytes, R, p);
        __syncwarp();
        if (lane == 0)
            mbar_arrive(empty + 8 * st);
        fwht256_q4_from_s2(p, lane);                  // unscaled: v[j] * 16
        const uint32_t row = rt * kAQRows + (uint32_t)R;
        uint32_t word[8];
        uint32_t sfw = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {                 // scale block b: values 16b .. 16b+15 of the quarter
            float a[16];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                f2_unpack(p[8 * b + i], a[2 * i], a[2 * i + 1]);
            const float m0 = fmax3(fabsf(a[0]), fabsf(a[1]), fabsf(a[2]));
            const float m1 = fmax3(fabsf(a[3]), fabsf(a[4]), fabsf(a[5]));
            const float m2 = fmax3(fabsf(a[6]), fabsf(a[7]), fabsf(a[8]));
            const float m3 = fmax3(fabsf(a[9]), fabsf(a[10]), fabsf(a[11]));
            const float m4 = fmax3(fabsf(a[12]), fabsf(a[13]), fabsf(a[14]));
            const float bmax = fmax3(fmax3(m0, m1, m2), fmax3(m3, m4, fabsf(a[15])), 0.0f);
            uint32_t code = 0, w0 = 0, w1 = 0;
            if (g != 0.0f) {
                // max |v / 16| = max |v| / 16 exactly (rounding is monotonic)
                code = to_ue4m3(__fdiv_rn(__fmul_rn(bmax, 0.0625f), sixg));
                if (code != 0) {
                    const float inv = inv_tab[code];
                    float sv[16];
                    if (fold16) {
                        const float i16 = __fmul_rn(inv, 0.0625f);
                        const uint64_t inv2 = f2_pack(i16, i16);
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            f2_unpack(f2_mul(p[8 * b + i], inv2), sv[2 * i], sv[2 * i + 1]);
                    } else {
                        const uint64_t inv2 = f2_pack(inv, inv), s16 = f2_pack(0.0625f, 0.0625f);
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            f2_unpack(f2_mul(f2_mul(p[8 * b + i], s16), inv2), sv[2 * i], sv[2 * i + 1]);
                    }
                    w0 = to_e2m1x4(sv[0], sv[1], sv[2], sv[3]) | (to_e2m1x4(sv[4], sv[5], sv[6], sv[7]) << 16);
                    w1 = to_e2m1x4(sv[8], sv[9], sv[10], sv[11]) |
                         (to_e2m1x4(sv[12], sv[13], sv[14], sv[15]) << 16);
                }
            }
            word[2 * b] = w0;
            word[2 * b + 1] = w1;
            sfw |= code << (8 * b);
        }
        if ((int64_t)row < M && SQ_DCHECK(kb * (kHad / 2) + 32 * q + 32 <= K / 2, status)) {
            uint4 *o = reinterpret_cast<uint4 *>(codes + (size_t)row * (size_t)(K / 2) + kb * (kHad / 2) + 32 * q);
            o[0] = make_uint4(word[0], word[1], word[2], word[3]);
            o[1] = make_uint4(word[4], word[5], word[6], word[7]);
        }
        // scale columns 4q .. 4q+3 of the chunk are four adjacent bytes of the tiled layout
        const uint32_t c4 = kb * (kHad / kSfBlock) / 4 + q;       // (column / 4) of the first of the four
        const size_t off = ((size_t)(row >> 7) * (C >> 2) + c4) * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4;
        if (SQ_DCHECK(off + 4 <= (size_t)rows_pad * C, status))
            *reinterpret_cast<uint32_t *>(sf + off) = sfw;
        kb += step_kb;
        rt += step_rt;
        if (kb >= nkb32) {
            kb -= nkb32;
            ++rt;
        }
    }
}

// ---------------------------------------------------------------------------
// low-rank operands as a kernel of their own (the int4 forward; see
// lowrank_unit).  g_x NULL means beta = 1.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) lowrank_finish_kernel(const float *__restrict__ t_part, int parts, int64_t M,
                                                             const float *__restrict__ g_x,
                                                             const float *__restrict__ g_w,
                                                             uint16_t *__restrict__ tsplit,
                                                             const uint16_t *__restrict__ U, int64_t N,
                                                             uint16_t *__restrict__ udup)
{
    const float beta = g_x ? lowrank_beta(*g_x, g_w) : 1.0f;
    const int64_t nT = M * 8;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nT + N * 4;
         i += (int64_t)gridDim.x * blockDim.x)
        lowrank_unit(i, nT, t_part, parts, nullptr, beta, tsplit, U, udup);
}

// ---------------------------------------------------------------------------
// bf16 reconstruct without the low-rank term (SQ_RECON_RESIDUAL_ONLY, or a
// weight without factors).  Tile = one 256-column block kb x 64 rows.
// Persistent CTAs of 256 threads walk a contiguous range of tiles (kb-major),
// staging the next tile's codes and scales in shared memory by cp.async while
// the current one is computed.
// Phase 1: each lane decodes 32 payload values of a row (an int4 group or half
//   group, two NVFP4 blocks, or 32 int8 codes), runs the 8-lane Hadamard
//   transform and writes bf16(h) to W, or (for the transposed output W^T
//   [K, N]) h into a shared fp32 tile (float4 f of a row stored at f ^ (f >> 3)
//   -- conflict free for both phases).
// Phase 2 (W^T only): thread t owns columns 2(t%128), 2(t%128)+1 and rows
//   32(t/128)..+31 of the tile and writes them as two 64-byte row pieces of W^T.
// The low-rank reconstruct is reconstruct_ws_kernel below.
// ---------------------------------------------------------------------------
constexpr int kRecRows = 64;
constexpr int kRecScaleBytes = kRecRows * 16;             // 1 KB (8 fp16, 4 fp16, 16 ue4m3 or 1 fp32 per row)
constexpr int kRecHBytes = kRecRows * kHad * 4;           // 64 KB

// per payload format (1 int4 g32, 2 NVFP4, 3 int4 g64: 4-bit codes, rank 32;
// 4 int8 per row: 8-bit codes, rank 16)
template <int FMT>
struct RecCfg {
    static constexpr int kRank = FMT == 4 ? 16 : 32;
    static constexpr int kCodeRow = FMT == 4 ? kHad : kHad / 2;             // code bytes per row and block
    static constexpr int kCodeBytes = kRecRows * kCodeRow;                    // 8 or 16 KB
    static constexpr int kUBytes = kRecRows * kRank * 2;                      // 4 or 2 KB
    static constexpr int kStageBytes = kCodeBytes + kRecScaleBytes + kUBytes;
    static constexpr int kUsBytes = kRecRows * kRank * 4;
    static constexpr int kSmemTiled = kRecHBytes + 2 * kStageBytes;             // h tile + two stages (W^T)
    static constexpr int kSmemResidual = 2 * kStageBytes;
};

__device__ __forceinline__ uint64_t pack2(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void unpack2(uint64_t v, float &lo, float &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

// acc = fma(a, b, acc) on two fp32 lanes, each rounded once
__device__ __forceinline__ void fma2(uint64_t &acc, uint64_t a, uint64_t b)
{
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

__device__ __forceinline__ void cp_async8(uint32_t dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

// Stage tile (kb, rows n0..n0+63) into one buffer: codes [64][128 B] (4-bit
// formats) or [64][256 B] (int8), scales [64][16 B] (int4 group 32: the 8 fp16
// group scales; int4 group 64: the 4 fp16 group scales in the first 8 bytes;
// NVFP4: the 16 ue4m3 block scales, gathered from the tiled layout 4 bytes at
// a time; int8: the row's fp32 scale in the first 4 bytes), lora_up
// [64][2 * rank B].  Rows past N are zero filled.
template <int FMT, bool LOWRANK, int NT = 256>
__device__ __forceinline__ void rec_stage(uint32_t buf, const uint8_t *codes, const void *scales, const uint16_t *U,
                                          int64_t N, int64_t K, int64_t kb, int64_t n0, int tid)
{
    using Cfg = RecCfg<FMT>;
    constexpr int kChunksPerRow = Cfg::kCodeRow / 16;
    static_assert(NT >= kRecRows && (kRecRows * kChunksPerRow) % NT == 0, "staging threads");
#pragma unroll
    for (int i = 0; i < kRecRows * kChunksPerRow / NT; ++i) {
        const int e = tid + NT * i;
        const int r = e / kChunksPerRow, c = e % kChunksPerRow;
        const int64_t n = n0 + r;
        const uint8_t *src =
            n < N ? codes + n * (K * Cfg::kCodeRow / kHad) + kb * Cfg::kCodeRow + 16 * c : codes;
        cp_async16(buf + r * Cfg::kCodeRow + 16 * c, src, n < N ? 16u : 0u);
    }
    const uint32_t sbuf = buf + Cfg::kCodeBytes;
    if (FMT == 1) {
        if (tid < kRecRows) {
            const int64_t n = n0 + tid;
            const uint8_t *src = n < N ? reinterpret_cast<const uint8_t *>(scales) + (n * (K / kGroup) + kb * 8) * 2
                                       : reinterpret_cast<const uint8_t *>(scales);
            cp_async16(sbuf + 16 * tid, src, n < N ? 16u : 0u);
        }
    } else if (FMT == 3) {
        if (tid < kRecRows) {                        // 4 scales = 8 bytes, 8-byte aligned (K % 256 == 0)
            const int64_t n = n0 + tid;
            const uint8_t *src = n < N ? reinterpret_cast<const uint8_t *>(scales) + (n * (K / 64) + kb * 4) * 2
                                       : reinterpret_cast<const uint8_t *>(scales);
            cp_async8(sbuf + 16 * tid, src, n < N ? 8u : 0u);
        }
    } else if (FMT == 4) {
        if (tid < kRecRows) {
            const int64_t n = n0 + tid;
            const uint8_t *src = n < N ? reinterpret_cast<const uint8_t *>(scales) + n * 4
                                       : reinterpret_cast<const uint8_t *>(scales);
            cp_async4(sbuf + 16 * tid, src, n < N ? 4u : 0u);
        }
    } else {
        for (int e = tid; e < 4 * kRecRows; e += NT) {
            const int r = e >> 2, j = e & 3;
            const int64_t n = n0 + r;
            const uint8_t *src = n < N ? reinterpret_cast<const uint8_t *>(scales) +
                                             sf_offset(n, kb * (kHad / kSfBlock) + 4 * j, K / kSfBlock)
                                       : reinterpret_cast<const uint8_t *>(scales);
            cp_async4(sbuf + 16 * r + 4 * j, src, n < N ? 4u : 0u);
        }
    }
    if (LOWRANK) {
        constexpr int kUChunks = Cfg::kRank / 8;     // 16-byte chunks of a lora_up row
        for (int e = tid; e < kRecRows * kUChunks; e += NT) {
            const int r = e / kUChunks, c = e % kUChunks;
            const int64_t n = n0 + r;
            const uint16_t *src = n < N ? U + n * Cfg::kRank + 8 * c : U;
            cp_async16(buf + Cfg::kCodeBytes + kRecScaleBytes + r * (2 * Cfg::kRank) + 16 * c, src,
                       n < N ? 16u : 0u);
        }
    }
}

// 32 payload values of staged row r, values 32q..32q+31 of the block (one int4
// group of 32, half of a group of 64, two NVFP4 blocks, or 32 int8 codes)
template <int FMT>
__device__ __forceinline__ void rec_decode(const uint8_t *stage, int r, int q, float g, float (&v)[32])
{
    using Cfg = RecCfg<FMT>;
    const uint8_t *sc = stage + Cfg::kCodeBytes + 16 * r;
    if (FMT == 4) {
        const float s = *reinterpret_cast<const float *>(sc);
        const uint4 c0 = *reinterpret_cast<const uint4 *>(stage + r * Cfg::kCodeRow + 32 * q);
        const uint4 c1 = *reinterpret_cast<const uint4 *>(stage + r * Cfg::kCodeRow + 32 * q + 16);
        const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float q[4];
            int8x4_to_f32(w[j], q);
#pragma unroll
            for (int t = 0; t < 4; ++t)
                v[4 * j + t] = __fmul_rn(q[t], s);
        }
        return;
    }
    const uint4 c = *reinterpret_cast<const uint4 *>(stage + r * Cfg::kCodeRow + 16 * q);
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
    if (FMT == 1 || FMT == 3) {
        const float s = __half2float(*reinterpret_cast<const __half *>(sc + 2 * (FMT == 3 ? q >> 1 : q)));
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float q[8];
            int4x8_to_f32(w[j], q);
#pragma unroll
            for (int t = 0; t < 8; ++t)
                v[8 * j + t] = __fmul_rn(q[t], s);
        }
    } else {
        const uint32_t sf2 = *reinterpret_cast<const uint16_t *>(sc + 2 * q);
        const float d0 = ue4m3_value(sf2 & 0xFFu), d1 = ue4m3_value(sf2 >> 8);
#pragma unroll
        for (int b = 0; b < 16; ++b) {
            const float2 e = e2m1x2_value((w[b >> 2] >> (8 * (b & 3))) & 0xFFu);
            const float d = b < 8 ? d0 : d1;
            v[2 * b] = __fmul_rn(__fmul_rn(e.x, d), g);
            v[2 * b + 1] = __fmul_rn(__fmul_rn(e.y, d), g);
        }
    }
}

template <int FMT, bool TRANS>
__global__ void __launch_bounds__(256, TRANS ? 2 : 3) reconstruct_kernel(const uint8_t *__restrict__ codes,
                                                                      const void *__restrict__ scales,
                                                                      const float *__restrict__ g_w,
                                                                      const uint16_t *__restrict__ U, int64_t N,
                                                                      int64_t K, uint16_t *__restrict__ W)
{
    using Cfg = RecCfg<FMT>;
    extern __shared__ __align__(128) uint8_t rec_smem[];
    float *h = reinterpret_cast<float *>(rec_smem);                                // [64][256] swizzled
    uint8_t *stage0 = rec_smem + (TRANS ? kRecHBytes : 0);
    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const float g = FMT == 2 ? *g_w : 0.0f;
    const int64_t NT = (N + kRecRows - 1) / kRecRows;
    const int64_t T = (K / kHad) * NT;
    const int64_t t_begin = T * blockIdx.x / gridDim.x;
    const int64_t t_end = T * (blockIdx.x + 1) / gridDim.x;
    if (t_begin >= t_end)
        return;
    const uint32_t sbase = smem_u32(stage0);
    rec_stage<FMT, false>(sbase, codes, scales, U, N, K, t_begin / NT, (t_begin % NT) * kRecRows, tid);
    cp_async_commit();

    const int cp = tid & 127;                        // phase 2 (W^T): column pair
    const int rbase = 32 * (tid >> 7);
    const int f = cp >> 1;                           // float4 of h holding columns 2cp, 2cp+1
    const int fo = 2 * (cp & 1);

#pragma unroll 1
    for (int64_t t = t_begin, i = 0; t < t_end; ++t, ++i) {
        const int buf = (int)(i & 1);
        if (t + 1 < t_end)
            rec_stage<FMT, false>(sbase + (buf ^ 1) * Cfg::kStageBytes, codes, scales, U, N, K, (t + 1) / NT,
                                  ((t + 1) % NT) * kRecRows, tid);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();                             // tile t staged; previous tile's phase 2 done
        const int64_t kb = t / NT;
        const int64_t n0 = (t % NT) * kRecRows;
        const uint8_t *st = stage0 + buf * Cfg::kStageBytes;

        // phase 1: h = H(d)
#pragma unroll 1
        for (int pass = 0; pass < 2; ++pass) {
            const int r = 32 * pass + 4 * warp + (lane >> 3);
            const int q = lane & 7;
            float v[32];
            rec_decode<FMT>(st, r, q, g, v);
            fwht256_l32(v, lane);
            if (!TRANS) {                            // row-major: straight to W
                const int64_t n = n0 + r;
                if (n < N && SQ_DCHECK(kb * kHad + 32 * q + 32 <= K, &g_library_status)) {
                    uint4 *o = reinterpret_cast<uint4 *>(W + n * K + kb * kHad + 32 * q);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        uint32_t ww[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            ww[j] = f32x2_to_bf16x2_bits(v[8 * k + 2 * j], v[8 * k + 2 * j + 1]);
                        o[k] = make_uint4(ww[0], ww[1], ww[2], ww[3]);
                    }
                }
            } else {
                float4 *row = reinterpret_cast<float4 *>(h + r * kHad);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int ff = 8 * q + k;
                    row[ff ^ (ff >> 3)] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
                }
            }
        }
        if (!TRANS) {
            __syncthreads();                         // stage buffer free before the next prefetch lands
            continue;
        }
        __syncthreads();                             // h complete

        // phase 2 (W^T [K, N]): rows k0, k0 + 1, columns n0 + rbase .. + 31
        const int64_t k0 = kb * kHad + 2 * cp;
        uint32_t tw0[16], tw1[16];                   // columns k0, k0 + 1 of the 32 rows, bf16 pairs
#pragma unroll
        for (int rr = 0; rr < 32; ++rr) {
            const int r = rbase + rr;
            const float2 hv = *reinterpret_cast<const float2 *>(h + r * kHad + 4 * (f ^ (f >> 3)) + fo);
            const uint32_t b0 = f32_to_bf16_bits(hv.x), b1 = f32_to_bf16_bits(hv.y);
            const int slot = rr >> 1, hi = rr & 1;
            tw0[slot] = hi ? (tw0[slot] | (b0 << 16)) : b0;
            tw1[slot] = hi ? (tw1[slot] | (b1 << 16)) : b1;
        }
        const int64_t nb0 = n0 + rbase;
        if (!SQ_DCHECK(k0 + 1 < K, &g_library_status))
            continue;
        if (nb0 + 32 <= N) {
            uint4 *o0 = reinterpret_cast<uint4 *>(W + k0 * N + nb0);
            uint4 *o1 = reinterpret_cast<uint4 *>(W + (k0 + 1) * N + nb0);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                o0[c] = make_uint4(tw0[4 * c], tw0[4 * c + 1], tw0[4 * c + 2], tw0[4 * c + 3]);
                o1[c] = make_uint4(tw1[4 * c], tw1[4 * c + 1], tw1[4 * c + 2], tw1[4 * c + 3]);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (nb0 + i < N) {
                    W[k0 * N + nb0 + i] = (uint16_t)(tw0[i >> 1] >> (16 * (i & 1)));
                    W[(k0 + 1) * N + nb0 + i] = (uint16_t)(tw1[i >> 1] >> (16 * (i & 1)));
                }
        }
    }
    cp_async_wait<0>();
}

// ---------------------------------------------------------------------------
// bf16 reconstruct with the low-rank term, warp-specialised (W, or W^T for
// TRANS).  Same tiles, same arithmetic and same outputs as reconstruct_kernel,
// but the two phases run in different warps of one CTA per SM and overlap:
//   warps 0-3 (producer): stage tile i + 2 by cp.async while tile i is
//     decoded; decode + Hadamard-transform tile i into h[i % 2] (16 rows per
//     warp), and its lora_up rows into us[i % 2] (fp32);
//   warps 4-11 (consumer): the rank-r fmaf chains of tile i from h[i % 2] and
//     us[i % 2] (thread t: columns 2(t%128), +1 and rows 32(t/128)..+31, as in
//     reconstruct_kernel), W = bf16(RN(L + h)).
// Hand-offs are mbarriers: stage_full[s] (the producer threads' copies landed,
// cp.async.mbarrier.arrive.noinc), stage_free[s] (the producer warps are done
// reading stage s), h_full[b] (h and us of the tile written), h_free[b] (the
// consumer warps are done with it).  Every wait is bounded; on a timeout the
// CTA stops, waits for its copies in flight and sets *status.
// ---------------------------------------------------------------------------
constexpr int kWsP1Warps = 4;
constexpr int kWsP2Warps = 8;
constexpr int kWsP1Threads = 32 * kWsP1Warps;
constexpr int kWsThreads = 32 * (kWsP1Warps + kWsP2Warps);

// lora_up of a tile in fp32 for the consumers: [rows][rank] (W^T), or [rank][rows + 4]
// (W: thread reads of four consecutive rows of one rank are one 16-byte broadcast)
constexpr int kUsTStride = kRecRows + 4;

template <int FMT>
struct RecWsCfg {
    using C = RecCfg<FMT>;
    static constexpr int kUsBytes = C::kRank * kUsTStride * 4 > C::kUsBytes ? C::kRank * kUsTStride * 4 : C::kUsBytes;
    static constexpr int kUsOff = 2 * kRecHBytes;                     // h[2] at 0
    static constexpr int kStageOff = kUsOff + 2 * kUsBytes;           // us[2]
    static constexpr int kBarOff = kStageOff + 2 * C::kStageBytes;    // stage[2]
    static constexpr int kSmem = kBarOff + 8 * 8 + 16;                // 8 mbarriers, abort flag
};

__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint32_t bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

template <int FMT, bool TRANS>
__global__ void __launch_bounds__(kWsThreads, 1) reconstruct_ws_kernel(const uint8_t *__restrict__ codes,
                                                                      const void *__restrict__ scales,
                                                                      const float *__restrict__ g_w,
                                                                      const uint16_t *__restrict__ U,
                                                                      const uint16_t *__restrict__ D, int64_t N,
                                                                      int64_t K, uint16_t *__restrict__ W,
                                                                      uint32_t *__restrict__ status)
{
    using Cfg = RecCfg<FMT>;
    using L = RecWsCfg<FMT>;
    constexpr int kR = Cfg::kRank;
    extern __shared__ __align__(128) uint8_t rec_smem[];
    uint64_t *bars = reinterpret_cast<uint64_t *>(rec_smem + L::kBarOff);
    const uint32_t stage_full = smem_u32(bars), stage_free = smem_u32(bars + 2);
    const uint32_t h_full = smem_u32(bars + 4), h_free = smem_u32(bars + 6);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(bars + 8);
    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(stage_full + 8 * b, kWsP1Threads);
            mbar_init(stage_free + 8 * b, kWsP1Warps);
            mbar_init(h_full + 8 * b, kWsP1Warps);
            mbar_init(h_free + 8 * b, kWsP2Warps);
        }
        *abort_flag = 0u;
        fence_mbar_init();
    }
    __syncthreads();
    const int64_t NT = (N + kRecRows - 1) / kRecRows;
    const int64_t T = (K / kHad) * NT;
    const int64_t t_begin = T * blockIdx.x / gridDim.x;
    const int n_tiles = (int)(T * (blockIdx.x + 1) / gridDim.x - t_begin);
    if (n_tiles <= 0)
        return;

    if (warp < kWsP1Warps) {
        // ------------------------------------------------------------ producer
        const float g = FMT == 2 ? *g_w : 0.0f;
        const uint32_t stage0 = smem_u32(rec_smem + L::kStageOff);
        auto issue = [&](int i) {
            const int64_t t = t_begin + i;
            const int sb = i & 1;
            rec_stage<FMT, true, kWsP1Threads>(stage0 + sb * Cfg::kStageBytes, codes, scales, U, N, K, t / NT,
                                               (t % NT) * kRecRows, tid);
            cp_async_mbar_arrive_noinc(stage_full + 8 * sb);
        };
        issue(0);
        if (n_tiles > 1)
            issue(1);
        for (int i = 0; i < n_tiles; ++i) {
            const int sb = i & 1;
            const uint32_t par = (uint32_t)(i >> 1) & 1u;
            if (!mbar_wait(stage_full + 8 * sb, par, abort_flag, status))
                break;
            if (!mbar_wait(h_free + 8 * sb, par ^ 1u, abort_flag, status))
                break;
            const uint8_t *st = rec_smem + L::kStageOff + sb * Cfg::kStageBytes;
            float *h = reinterpret_cast<float *>(rec_smem + sb * kRecHBytes);
            float *us = reinterpret_cast<float *>(rec_smem + L::kUsOff + sb * L::kUsBytes);
#pragma unroll 1
            for (int pass = 0; pass < kRecRows / (4 * kWsP1Warps); ++pass) {
                const int r = 4 * kWsP1Warps * pass + 4 * warp + (lane >> 3);
                const int q = lane & 7;
                float v[32];
                rec_decode<FMT>(st, r, q, g, v);
                fwht256_l32(v, lane);
                float4 *row = reinterpret_cast<float4 *>(h + r * kHad);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int ff = 8 * q + k;
                    row[ff ^ (ff >> 3)] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
                }
            }
            const uint16_t *ust = reinterpret_cast<const uint16_t *>(st + Cfg::kCodeBytes + kRecScaleBytes);
#pragma unroll
            for (int j = 0; j < kRecRows * kR / kWsP1Threads; ++j) {
                const int e = tid + kWsP1Threads * j;          // element (row e / kR, rank e % kR)
                const float u = bf16_bits_to_f32(ust[e]);
                if (TRANS)
                    us[e] = u;
                else
                    us[(e % kR) * kUsTStride + e / kR] = u;
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(h_full + 8 * sb);
                mbar_arrive(stage_free + 8 * sb);
            }
            if (i + 2 < n_tiles) {                   // every producer warp is done with stage sb
                if (!mbar_wait(stage_free + 8 * sb, par, abort_flag, status))
                    break;
                issue(i + 2);
            }
        }
        cp_async_wait<0>();                          // no copy lands after the CTA exits
        return;
    }

    // ---------------------------------------------------------------- consumer
    if (!TRANS) {
        // W: thread t takes columns k0 = 2 (t % 128), k0 + 1 and rows 32 (t / 128) .. + 31, four
        // rows at a time.  The packed lanes of an fma run over two rows of one column: the
        // column's lora_down value is the duplicated operand (duplicated once per 256-column
        // block, in registers), and the rows' lora_up values come as ready pairs from one
        // 16-byte broadcast load of the transposed us -- no move per fma.  Each (row, column)
        // is still its own chain fma(U[n, r], D[k, r], L) for r = 0, 1, .. in order.
        const int ct = tid - kWsP1Threads;
        const int cp = ct & 127;
        const int rbase = 32 * (ct >> 7);
        const int f = cp >> 1;                       // float4 of h holding columns 2cp, 2cp+1
        const int fo = 2 * (cp & 1);
        uint64_t dd0[kR], dd1[kR];                   // (D[k0, r], D[k0, r]) and (D[k0 + 1, r], D[k0 + 1, r])
        int64_t cur_kb = -1;
#pragma unroll 1
        for (int i = 0; i < n_tiles; ++i) {
            const int sb = i & 1;
            const int64_t t = t_begin + i;
            const int64_t kb = t / NT;
            const int64_t n0 = (t % NT) * kRecRows;
            const int64_t k0 = kb * kHad + 2 * cp;
            if (kb != cur_kb) {
                cur_kb = kb;
                const uint4 *dr0 = reinterpret_cast<const uint4 *>(D + k0 * kR);
                const uint4 *dr1 = reinterpret_cast<const uint4 *>(D + (k0 + 1) * kR);
#pragma unroll
                for (int k = 0; k < kR / 8; ++k) {
                    const uint4 a = __ldg(dr0 + k), b = __ldg(dr1 + k);
                    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float a0 = bf16_bits_to_f32(wa[j] & 0xFFFFu), a1 = bf16_bits_to_f32(wa[j] >> 16);
                        const float b0 = bf16_bits_to_f32(wb[j] & 0xFFFFu), b1 = bf16_bits_to_f32(wb[j] >> 16);
                        dd0[8 * k + 2 * j] = pack2(a0, a0);
                        dd0[8 * k + 2 * j + 1] = pack2(a1, a1);
                        dd1[8 * k + 2 * j] = pack2(b0, b0);
                        dd1[8 * k + 2 * j + 1] = pack2(b1, b1);
                    }
                }
            }
            if (!mbar_wait(h_full + 8 * sb, (uint32_t)(i >> 1) & 1u, abort_flag, status))
                break;
            const float *h = reinterpret_cast<const float *>(rec_smem + sb * kRecHBytes);
            const float *us = reinterpret_cast<const float *>(rec_smem + L::kUsOff + sb * L::kUsBytes);
#pragma unroll 2
            for (int r0 = rbase; r0 < rbase + 32; r0 += 4) {
                // a01 / a23: rows (r0, r0 + 1) / (r0 + 2, r0 + 3) of column k0; b01 / b23 of k0 + 1
                uint64_t a01 = 0ull, a23 = 0ull, b01 = 0ull, b23 = 0ull;
#pragma unroll
                for (int rr = 0; rr < kR; ++rr) {
                    const ulonglong2 u = *reinterpret_cast<const ulonglong2 *>(us + rr * kUsTStride + r0);
                    fma2(a01, u.x, dd0[rr]);
                    fma2(a23, u.y, dd0[rr]);
                    fma2(b01, u.x, dd1[rr]);
                    fma2(b23, u.y, dd1[rr]);
                }
                float La[4], Lb[4];
                unpack2(a01, La[0], La[1]);
                unpack2(a23, La[2], La[3]);
                unpack2(b01, Lb[0], Lb[1]);
                unpack2(b23, Lb[2], Lb[3]);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int r = r0 + j;
                    const int64_t n = n0 + r;
                    const float2 hv = *reinterpret_cast<const float2 *>(h + r * kHad + 4 * (f ^ (f >> 3)) + fo);
                    const float o0 = __fadd_rn(La[j], hv.x);   // W = bf16(RN(L + h))
                    const float o1 = __fadd_rn(Lb[j], hv.y);
                    if (n < N && SQ_DCHECK(k0 + 1 < K, status))
                        *reinterpret_cast<uint32_t *>(W + n * K + k0) = f32x2_to_bf16x2_bits(o0, o1);
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(h_free + 8 * sb);          // h and us of this tile are no longer read
        }
        return;
    }
    const int ct = tid - kWsP1Threads;
    const int cp = ct & 127;
    const int rbase = 32 * (ct >> 7);
    const int f = cp >> 1;                           // float4 of h holding columns 2cp, 2cp+1
    const int fo = 2 * (cp & 1);
    uint64_t d2[kR];
    int64_t cur_kb = -1;
#pragma unroll 1
    for (int i = 0; i < n_tiles; ++i) {
        const int sb = i & 1;
        const int64_t t = t_begin + i;
        const int64_t kb = t / NT;
        const int64_t n0 = (t % NT) * kRecRows;
        const int64_t k0 = kb * kHad + 2 * cp;
        if (kb != cur_kb) {                          // lora_down of this thread's two columns
            cur_kb = kb;
            const uint4 *dr0 = reinterpret_cast<const uint4 *>(D + k0 * kR);
            const uint4 *dr1 = reinterpret_cast<const uint4 *>(D + (k0 + 1) * kR);
#pragma unroll
            for (int k = 0; k < kR / 8; ++k) {
                const uint4 a = __ldg(dr0 + k), b = __ldg(dr1 + k);
                const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    d2[8 * k + 2 * j] = pack2(bf16_bits_to_f32(wa[j] & 0xFFFFu), bf16_bits_to_f32(wb[j] & 0xFFFFu));
                    d2[8 * k + 2 * j + 1] = pack2(bf16_bits_to_f32(wa[j] >> 16), bf16_bits_to_f32(wb[j] >> 16));
                }
            }
        }
        if (!mbar_wait(h_full + 8 * sb, (uint32_t)(i >> 1) & 1u, abort_flag, status))
            break;
        const float *h = reinterpret_cast<const float *>(rec_smem + sb * kRecHBytes);
        const float *us = reinterpret_cast<const float *>(rec_smem + L::kUsOff + sb * L::kUsBytes);
        uint32_t tw0[16], tw1[16];                   // TRANS: columns k0, k0 + 1 of the 32 rows, bf16 pairs
        constexpr int kUnroll = TRANS ? 8 : 1;       // register-indexed pieces need constant indices
#pragma unroll kUnroll
        for (int r0 = rbase; r0 < rbase + 32; r0 += 4) {
            uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
            for (int rr = 0; rr < kR; rr += 4) {
                float4 u4[4];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    u4[j] = *reinterpret_cast<const float4 *>(us + (r0 + j) * kR + rr);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    fma2(acc[j], pack2(u4[j].x, u4[j].x), d2[rr]);
                    fma2(acc[j], pack2(u4[j].y, u4[j].y), d2[rr + 1]);
                    fma2(acc[j], pack2(u4[j].z, u4[j].z), d2[rr + 2]);
                    fma2(acc[j], pack2(u4[j].w, u4[j].w), d2[rr + 3]);
                }
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int r = r0 + j;
                const int64_t n = n0 + r;
                const float2 hv = *reinterpret_cast<const float2 *>(h + r * kHad + 4 * (f ^ (f >> 3)) + fo);
                float L0, L1;
                unpack2(acc[j], L0, L1);
                const float o0 = __fadd_rn(L0, hv.x);  // W = bf16(RN(L + h))
                const float o1 = __fadd_rn(L1, hv.y);
                if (TRANS) {
                    const uint32_t b0 = f32_to_bf16_bits(o0), b1 = f32_to_bf16_bits(o1);
                    const int slot = (r - rbase) >> 1, hi = (r - rbase) & 1;
                    tw0[slot] = hi ? (tw0[slot] | (b0 << 16)) : b0;
                    tw1[slot] = hi ? (tw1[slot] | (b1 << 16)) : b1;
                } else if (n < N && SQ_DCHECK(k0 + 1 < K, status)) {
                    *reinterpret_cast<uint32_t *>(W + n * K + k0) = f32x2_to_bf16x2_bits(o0, o1);
                }
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(h_free + 8 * sb);              // h and us of this tile are no longer read
        if (TRANS) {                                 // W^T [K, N]: rows k0, k0 + 1, columns n0 + rbase .. + 31
            const int64_t nb0 = n0 + rbase;
            if (!SQ_DCHECK(k0 + 1 < K, status)) {
                // index check failed (debug builds): the stores are skipped
            } else if (nb0 + 32 <= N) {
                uint4 *o0 = reinterpret_cast<uint4 *>(W + k0 * N + nb0);
                uint4 *o1 = reinterpret_cast<uint4 *>(W + (k0 + 1) * N + nb0);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    o0[c] = make_uint4(tw0[4 * c], tw0[4 * c + 1], tw0[4 * c + 2], tw0[4 * c + 3]);
                    o1[c] = make_uint4(tw1[4 * c], tw1[4 * c + 1], tw1[4 * c + 2], tw1[4 * c + 3]);
                }
            } else {
#pragma unroll
                for (int i2 = 0; i2 < 32; ++i2)
                    if (nb0 + i2 < N) {
                        W[k0 * N + nb0 + i2] = (uint16_t)(tw0[i2 >> 1] >> (16 * (i2 & 1)));
                        W[(k0 + 1) * N + nb0 + i2] = (uint16_t)(tw1[i2 >> 1] >> (16 * (i2 & 1)));
                    }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// the SQ_CHECK_FINITE scan: n bf16 values (n % 8 == 0), 16 bytes per step; a value whose exponent
// field is all ones (NaN or infinity) sets kStatusNonfinite, once per warp that meets one
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) check_finite_bf16_kernel(const uint4 *__restrict__ x, int64_t n16,
                                                                uint32_t *__restrict__ status)
{
    bool bad = false;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += (int64_t)gridDim.x * blockDim.x) {
        const uint4 v = x[i];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
            bad |= ((w[j] & 0x7F80u) == 0x7F80u) | ((w[j] & 0x7F800000u) == 0x7F800000u);
    }
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0)
        atomicOr(status, kStatusNonfinite);
}

cudaError_t launch_check_finite_bf16(const uint16_t *x, int64_t n, uint32_t *status, int sms, cudaStream_t s)
{
    const int64_t n16 = n / 8;
    const int64_t blocks = (n16 + 255) / 256;
    const int64_t grid = blocks < (int64_t)sms * 4 ? blocks : (int64_t)sms * 4;
    check_finite_bf16_kernel<<<(unsigned)(grid < 1 ? 1 : grid), 256, 0, s>>>(reinterpret_cast<const uint4 *>(x), n16,
                                                                           status);
    return cudaGetLastError();
}

cudaError_t library_status_word(uint32_t **p)
{
    return cudaGetSymbolAddress(reinterpret_cast<void **>(p), g_library_status);
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
static int grid_for(int64_t warp_tasks, int warps_per_block, int sms, int ctas_per_sm)
{
    int64_t want = (warp_tasks + warps_per_block - 1) / warps_per_block;
    int64_t cap = (int64_t)sms * ctas_per_sm;
    if (want > cap)
        want = cap;
    return (int)(want < 1 ? 1 : want);
}

// streamer launch: tensor map over `in` as [rows * K / 32, 32], persistent grid
template <typename T>
static bool stream_map(CUtensorMap *tm, const T *in, int64_t rows, int64_t K)
{
    const bool f32 = sizeof(T) == 4;
    return make_tmap(tm, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (int)sizeof(T), in,
                     32, (uint64_t)(rows * K / 32), 32, 256, f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
}

// shared-memory opt-in, once per device, context and kernel (keyed on the kernel
// itself: kernels with the same signature must not share the flag)
template <typename T, auto k>
static cudaError_t stream_attr()
{
    constexpr int kMaxDev = 64;
    static unsigned long long done_ctx[kMaxDev];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev)
        return cudaErrorInvalidDevice;
    const unsigned long long ctx = current_context_id();
    if (ctx != 0 && done_ctx[dev] == ctx)
        return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, StreamCfg<T>::kSmem);
    if (e == cudaSuccess)
        done_ctx[dev] = ctx;
    return e;
}

static int stream_grid(int64_t blocks, int sms, int per_sm)
{
    const int64_t chunks = (blocks + 31) / 32;
    const int64_t cap = (int64_t)sms * per_sm;
    return (int)(chunks < 1 ? 1 : (chunks < cap ? chunks : cap));
}

template <typename T>
static cudaError_t launch_absmax_rot(const T *in, int64_t rows, int64_t K, uint32_t *amax, int sms, cudaStream_t s)
{
    CUtensorMap tm;
    if (!stream_map(&tm, in, rows, K))
        return cudaErrorInvalidValue;
    cudaError_t e = stream_attr<T, absmax_rot_kernel<T>>();
    if (e != cudaSuccess)
        return e;
    const int64_t blocks = rows * (K / kHad);
    absmax_rot_kernel<T><<<stream_grid(blocks, sms, sizeof(T) == 4 ? 2 : 3), kStreamThreads, StreamCfg<T>::kSmem, s>>>(
        tm, blocks, amax);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_nvfp4_quant(const T *in, int64_t rows, int64_t K, const uint32_t *amax, const float *g_static,
                                      float *g_out, uint8_t *codes, uint8_t *sf, const LowrankOut &lr, int sms,
                                      cudaStream_t s)
{
    CUtensorMap tm;
    if (!stream_map(&tm, in, rows, K))
        return cudaErrorInvalidValue;
    cudaError_t e = stream_attr<T, nvfp4_quant_kernel<T>>();
    if (e != cudaSuccess)
        return e;
    const int64_t rows_pad = (rows + 127) / 128 * 128;
    // dependent launch: the CTAs start (and stream x) while the absmax pass drains
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)stream_grid(rows_pad * (K / kHad), sms, sizeof(T) == 4 ? 2 : 3));
    cfg.blockDim = dim3(kStreamThreads);
    cfg.dynamicSmemBytes = StreamCfg<T>::kSmem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, nvfp4_quant_kernel<T>, tm, rows, rows_pad, K, amax, g_static, g_out, codes, sf,
                              lr);
}

cudaError_t launch_absmax_rot_f32(const float *in, int64_t rows, int64_t K, uint32_t *amax, int sms, cudaStream_t s)
{
    return launch_absmax_rot(in, rows, K, amax, sms, s);
}

cudaError_t launch_absmax_rot_bf16(const uint16_t *in, int64_t rows, int64_t K, uint32_t *amax, int sms,
                                   cudaStream_t s)
{
    return launch_absmax_rot(in, rows, K, amax, sms, s);
}

cudaError_t launch_nvfp4_quant_f32(const float *in, int64_t rows, int64_t K, const uint32_t *amax,
                                   const float *g_static, float *g_out, uint8_t *codes, uint8_t *sf, int sms,
                                   cudaStream_t s)
{
    return launch_nvfp4_quant(in, rows, K, amax, g_static, g_out, codes, sf, LowrankOut{}, sms, s);
}

cudaError_t launch_nvfp4_quant_bf16(const uint16_t *in, int64_t rows, int64_t K, const uint32_t *amax,
                                    const float *g_static, float *g_out, uint8_t *codes, uint8_t *sf,
                                    const LowrankOut &lr, uint32_t *status, int sms, cudaStream_t s)
{
    constexpr int kMaxDev = 64;
    static unsigned long long attr_ctx[kMaxDev];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev)
        return cudaErrorInvalidDevice;
    const unsigned long long ctx = current_context_id();
    if (ctx == 0 || attr_ctx[dev] != ctx) {
        cudaError_t e = cudaFuncSetAttribute(act_quant_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAQSmem);
        if (e != cudaSuccess)
            return e;
        attr_ctx[dev] = ctx;
    }
    CUtensorMap tmx;
    if (!make_tmap(&tmx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, in, (uint64_t)K, (uint64_t)rows, 64, kAQRows,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const int64_t rows_pad = (rows + 127) / 128 * 128;
    const int64_t units = rows_pad / kAQRows * (K / kHad);
    const int64_t cap = 2LL * sms;                   // two CTAs per SM
    // dependent launch: the CTAs start (and stream x) while pass 1 drains
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(units < cap ? units : cap));
    cfg.blockDim = dim3(kAQThreads);
    cfg.dynamicSmemBytes = kAQSmem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, act_quant_kernel, tmx, rows, rows_pad, K, amax, g_static, g_out, codes, sf, lr,
                              status);
}

cudaError_t launch_int4_build(const float *R, int64_t N, int64_t K, int group, uint8_t *codes, uint16_t *scales,
                              uint8_t *frac, int sms, cudaStream_t s)
{
    CUtensorMap tm;
    if (!stream_map(&tm, R, N, K))
        return cudaErrorInvalidValue;
    cudaError_t e = stream_attr<float, int4_build_kernel<32>>();
    if (e != cudaSuccess)
        return e;
    const int64_t blocks = N * K / kHad;
    if (group == 64) {
        e = stream_attr<float, int4_build_kernel<64>>();
        if (e != cudaSuccess)
            return e;
        int4_build_kernel<64><<<stream_grid(blocks, sms, 2), kStreamThreads, StreamCfg<float>::kSmem, s>>>(
            tm, blocks, codes, scales, frac);
    } else {
        int4_build_kernel<32><<<stream_grid(blocks, sms, 2), kStreamThreads, StreamCfg<float>::kSmem, s>>>(
            tm, blocks, codes, scales, frac);
    }
    return cudaGetLastError();
}

cudaError_t launch_int8_build(const float *R, int64_t N, int64_t K, int8_t *codes, float *scales, uint8_t *frac,
                              int sms, cudaStream_t s)
{
    if (K > kI8MaxK)
        return cudaErrorInvalidValue;
    constexpr int kMaxDev = 64;
    static unsigned long long attr_ctx[kMaxDev];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev)
        return cudaErrorInvalidDevice;
    const unsigned long long ctx = current_context_id();
    if (ctx == 0 || attr_ctx[dev] != ctx) {
        cudaError_t e = cudaFuncSetAttribute(int8_build_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             i8_smem_bytes(kI8MaxK));
        if (e != cudaSuccess)
            return e;
        attr_ctx[dev] = ctx;
    }
    // persistent CTAs over rows: only as many as are resident at once (registers and
    // shared memory), so that no CTA waits for a whole earlier CTA's share of rows
    const int smem = i8_smem_bytes((int)K);
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, int8_build_kernel, kI8Threads, smem) != cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    const int64_t want = (int64_t)sms * per_sm;
    const unsigned grid = (unsigned)(N < want ? N : want);
    int8_build_kernel<<<grid, kI8Threads, smem, s>>>(R, N, (int)K, codes, scales, frac);
    return cudaGetLastError();
}

cudaError_t launch_widen_rank16(const uint16_t *src, int64_t rows, uint16_t *dst, int sms, cudaStream_t s)
{
    widen_rank16_kernel<<<grid_for(rows * 4, 256, sms, 4), 256, 0, s>>>(reinterpret_cast<const uint4 *>(src), rows,
                                                                       reinterpret_cast<uint4 *>(dst));
    return cudaGetLastError();
}

cudaError_t launch_act_pass1(const uint16_t *x, int64_t M, int64_t K, const uint16_t *D, uint32_t *amax,
                             float *t_part, uint16_t *xb, uint32_t *status, int sms, cudaStream_t s)
{
    (void)sms;
    constexpr int kMaxDev = 64;
    static unsigned long long attr_ctx[kMaxDev];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev)
        return cudaErrorInvalidDevice;
    const unsigned long long ctx = current_context_id();
    if (ctx == 0 || attr_ctx[dev] != ctx) {
        cudaError_t e = cudaFuncSetAttribute(act_pass1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kP1Smem);
        if (e != cudaSuccess)
            return e;
        attr_ctx[dev] = ctx;
    }
    CUtensorMap tmx, tmd;
    memset(&tmd, 0, sizeof(tmd));
    if (!make_tmap(&tmx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, (uint64_t)K, (uint64_t)M, 64, kP1Rows,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (t_part && !make_tmap(&tmd, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, (uint64_t)kRank, (uint64_t)K, kRank, kHad,
                             CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    const int64_t tiles = (M + kP1Rows - 1) / kP1Rows;
    const int split = act_t_parts(M, K);
    act_pass1_kernel<<<(unsigned)(tiles * split), kP1Threads, kP1Smem, s>>>(tmx, tmd, M, K, amax, t_part, split,
                                                                            xb, status);
    return cudaGetLastError();
}

cudaError_t launch_lowrank_finish(const float *t_part, int parts, int64_t M, const float *g_x, const float *g_w,
                                  uint16_t *tsplit, const uint16_t *U, int64_t N, uint16_t *udup, int sms,
                                  cudaStream_t s)
{
    lowrank_finish_kernel<<<grid_for(M * 8 + N * 4, 256, sms, 4), 256, 0, s>>>(t_part, parts, M, g_x, g_w, tsplit,
                                                                                  U, N, udup);
    return cudaGetLastError();
}

template <int FMT, bool TRANS>
static cudaError_t launch_reconstruct_v(const uint8_t *codes, const void *scales, const float *g_w,
                                        const uint16_t *U, int64_t N, int64_t K, uint16_t *W, int sms,
                                        cudaStream_t s)
{
    using Cfg = RecCfg<FMT>;
    constexpr int kSmem = TRANS ? Cfg::kSmemTiled : Cfg::kSmemResidual;
    constexpr int kMaxDev = 64;
    static unsigned long long attr_ctx[kMaxDev];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev)
        return cudaErrorInvalidDevice;
    const unsigned long long ctx = current_context_id();
    if (TRANS && (ctx == 0 || attr_ctx[dev] != ctx)) {
        cudaError_t e = cudaFuncSetAttribute(reconstruct_kernel<FMT, TRANS>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        if (e != cudaSuccess)
            return e;
        attr_ctx[dev] = ctx;
    }
    const int64_t tiles = (K / kHad) * ((N + kRecRows - 1) / kRecRows);
    const int64_t per_sm = TRANS ? 2 : 3;                    // resident CTAs per SM (registers, shared memory)
    const unsigned grid = (unsigned)(tiles < per_sm * sms ? tiles : per_sm * sms);
    reconstruct_kernel<FMT, TRANS><<<grid, 256, kSmem, s>>>(codes, scales, g_w, U, N, K, W);
    return cudaGetLastError();
}

// the warp-specialised kernel: one CTA of 384 threads per SM
template <int FMT, bool TRANS>
static cudaError_t launch_reconstruct_ws(const uint8_t *codes, const void *scales, const float *g_w,
                                         const uint16_t *U, const uint16_t *D, int64_t N, int64_t K, uint16_t *W,
                                         int sms, cudaStream_t s)
{
    constexpr int kSmem = RecWsCfg<FMT>::kSmem;
    constexpr int kMaxDev = 64;
    static unsigned long long attr_ctx[kMaxDev];
    static uint32_t *status_word[kMaxDev];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev)
        return cudaErrorInvalidDevice;
    const unsigned long long ctx = current_context_id();
    if (ctx == 0 || attr_ctx[dev] != ctx) {
        cudaError_t e = cudaFuncSetAttribute(reconstruct_ws_kernel<FMT, TRANS>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        if (e == cudaSuccess)
            e = library_status_word(&status_word[dev]);
        if (e != cudaSuccess)
            return e;
        attr_ctx[dev] = ctx;
    }
    const int64_t tiles = (K / kHad) * ((N + kRecRows - 1) / kRecRows);
    const unsigned grid = (unsigned)(tiles < sms ? tiles : sms);
    reconstruct_ws_kernel<FMT, TRANS><<<grid, kWsThreads, kSmem, s>>>(codes, scales, g_w, U, D, N, K, W,
                                                                      status_word[dev]);
    return cudaGetLastError();
}

template <int FMT>
static cudaError_t launch_reconstruct_fmt(const uint8_t *codes, const void *scales, const float *g_w,
                                          const uint16_t *U, const uint16_t *D, int64_t N, int64_t K,
                                          int with_lowrank, int transposed, uint16_t *W, int sms, cudaStream_t s)
{
    if (transposed)
        return with_lowrank ? launch_reconstruct_ws<FMT, true>(codes, scales, g_w, U, D, N, K, W, sms, s)
                            : launch_reconstruct_v<FMT, true>(codes, scales, g_w, U, N, K, W, sms, s);
    return with_lowrank ? launch_reconstruct_ws<FMT, false>(codes, scales, g_w, U, D, N, K, W, sms, s)
                        : launch_reconstruct_v<FMT, false>(codes, scales, g_w, U, N, K, W, sms, s);
}

cudaError_t launch_reconstruct(int fmt, const uint8_t *codes, const void *scales, const float *g_w,
                               const uint16_t *U, const uint16_t *D, int64_t N, int64_t K, int with_lowrank,
                               int transposed, uint16_t *W, int sms, cudaStream_t s)
{
    switch (fmt) {
    case 2: return launch_reconstruct_fmt<2>(codes, scales, g_w, U, D, N, K, with_lowrank, transposed, W, sms, s);
    case 3: return launch_reconstruct_fmt<3>(codes, scales, g_w, U, D, N, K, with_lowrank, transposed, W, sms, s);
    case 4: return launch_reconstruct_fmt<4>(codes, scales, g_w, U, D, N, K, with_lowrank, transposed, W, sms, s);
    default: return launch_reconstruct_fmt<1>(codes, scales, g_w, U, D, N, K, with_lowrank, transposed, W, sms, s);
    }
}

}  // namespace sq
