// sq_quant.cu -- HBM-bound kernels of the SquareQ W4 layer: Hadamard-256
// rotation + absmax, NVFP4 block quantisation into the tiled scale layout,
// the int4 group-32 builder with its scale-fraction sweep, the bf16
// activation rotation and int4 dequant of the "dequant-first" forward, the
// low-rank input t = x . lora_down, and the bf16 reconstruct.
//
// All kernels are grid-stride loops over warp-sized tasks, launched with a
// grid that is a multiple of the SM count; loads and stores are contiguous per
// warp.  They follow the SquareQ README, section "SquareQ v3 -- W4", as stated
// operation by operation in include/sq.h.
#include "sq_kernels.h"
#include "sq_device.cuh"

namespace sq {

// ---------------------------------------------------------------------------
// loading one 256-block into the warp layout of fwht256_warp
// ---------------------------------------------------------------------------
__device__ __forceinline__ void load_block(const float *p, int lane, float (&v)[8])
{
    float4 a = __ldg(reinterpret_cast<const float4 *>(p + 4 * lane));
    float4 b = __ldg(reinterpret_cast<const float4 *>(p + 128 + 4 * lane));
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void load_block(const uint16_t *p, int lane, float (&v)[8])
{
    uint2 a = __ldg(reinterpret_cast<const uint2 *>(p + 4 * lane));
    uint2 b = __ldg(reinterpret_cast<const uint2 *>(p + 128 + 4 * lane));
    v[0] = bf16_bits_to_f32(a.x & 0xFFFFu); v[1] = bf16_bits_to_f32(a.x >> 16);
    v[2] = bf16_bits_to_f32(a.y & 0xFFFFu); v[3] = bf16_bits_to_f32(a.y >> 16);
    v[4] = bf16_bits_to_f32(b.x & 0xFFFFu); v[5] = bf16_bits_to_f32(b.x >> 16);
    v[6] = bf16_bits_to_f32(b.y & 0xFFFFu); v[7] = bf16_bits_to_f32(b.y >> 16);
}

// ---------------------------------------------------------------------------
// pass 1: A = max |H in| over a [rows, K] matrix, folded into *amax (u32 bits)
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) absmax_rot_kernel(const T *__restrict__ in, int64_t rows,
                                                         int64_t K, uint32_t *__restrict__ amax)
{
    const int lane = threadIdx.x & 31;
    const int64_t warps_total = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t kb_per_row = K / kHad;
    const int64_t tasks = rows * kb_per_row;
    float m = 0.0f;
    for (int64_t task = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); task < tasks;
         task += warps_total) {
        float v[8];
        load_block(in + task * kHad, lane, v);
        fwht256_warp(v, lane);
#pragma unroll
        for (int i = 0; i < 8; ++i)
            m = fmaxf(m, fabsf(v[i]));
    }
#pragma unroll
    for (int x = 16; x >= 1; x >>= 1)
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, x));
    __shared__ float wmax[32];
    if (lane == 0)
        wmax[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float b = 0.0f;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w)
            b = fmaxf(b, wmax[w]);
        atomic_max_nonneg(amax, b);
    }
}

// ---------------------------------------------------------------------------
// pass 2: NVFP4 block quantisation of H in with global scale g.
// rows_pad >= rows (a multiple of 128): rows past `rows` are zero, and only
// their scale bytes are written (as 0), which fills the tiled layout's padding.
// g comes from *g_static when non-NULL, else RN(A / 2688) from *amax, and is
// stored to *g_out (when non-NULL) by thread 0 of block 0.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) nvfp4_quant_kernel(const T *__restrict__ in, int64_t rows,
                                                          int64_t rows_pad, int64_t K,
                                                          const uint32_t *__restrict__ amax,
                                                          const float *__restrict__ g_static,
                                                          float *__restrict__ g_out,
                                                          uint8_t *__restrict__ codes,
                                                          uint8_t *__restrict__ sf)
{
    const int lane = threadIdx.x & 31;
    const float g = g_static ? *g_static : __fdiv_rn(__uint_as_float(*amax), 2688.0f);
    if (g_out && blockIdx.x == 0 && threadIdx.x == 0)
        *g_out = g;
    const float sixg = __fmul_rn(6.0f, g);
    const int64_t warps_total = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t kb_per_row = K / kHad;
    const int64_t C = K / kSfBlock;
    const int64_t tasks = rows_pad * kb_per_row;
    for (int64_t task = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); task < tasks;
         task += warps_total) {
        const int64_t row = task / kb_per_row;
        const int64_t kb = task - row * kb_per_row;
        float v[8];
        const bool valid = row < rows;
        if (valid) {
            load_block(in + row * K + kb * kHad, lane, v);
            fwht256_warp(v, lane);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                v[i] = 0.0f;
        }
        uint32_t packed[2];
        uint32_t sfc[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            // block of 16 = 4 lanes x 4 values
            float b = fmaxf(fmaxf(fabsf(v[4 * h]), fabsf(v[4 * h + 1])),
                            fmaxf(fabsf(v[4 * h + 2]), fabsf(v[4 * h + 3])));
            b = fmaxf(b, __shfl_xor_sync(0xffffffffu, b, 1));
            b = fmaxf(b, __shfl_xor_sync(0xffffffffu, b, 2));
            uint32_t code = 0;
            uint32_t pk = 0;
            if (g != 0.0f) {
                code = to_ue4m3(__fdiv_rn(b, sixg));
                if (code != 0) {
                    const float den = __fmul_rn(ue4m3_value(code), g);
                    const float inv = __frcp_rn(den);
                    pk = to_e2m1x2(__fmul_rn(v[4 * h], inv), __fmul_rn(v[4 * h + 1], inv)) |
                         (to_e2m1x2(__fmul_rn(v[4 * h + 2], inv), __fmul_rn(v[4 * h + 3], inv)) << 8);
                }
            }
            packed[h] = pk;
            sfc[h] = code;
        }
        if (valid) {
            uint16_t *cp = reinterpret_cast<uint16_t *>(codes + row * (K / 2) + kb * (kHad / 2));
            cp[lane] = (uint16_t)packed[0];
            cp[32 + lane] = (uint16_t)packed[1];   // bytes 64..127 of the block
        }
        if ((lane & 3) == 0) {
            const int64_t c0 = kb * (kHad / kSfBlock) + (lane >> 2);
            sf[sf_offset(row, c0, C)] = (uint8_t)sfc[0];
            sf[sf_offset(row, c0 + 8, C)] = (uint8_t)sfc[1];
        }
    }
}

// ---------------------------------------------------------------------------
// int4 group-32 builder.  A warp takes 4 consecutive 256-blocks (1024 values,
// 32 groups), rotates them, stages them in shared memory and then each lane
// sweeps one whole group of 32 in registers.
// Staging layout: group G, float4 w of the group sits in slot G*8 + (w ^ (G&7))
// so both the rotated writes and the per-group reads are conflict free.
// ---------------------------------------------------------------------------
constexpr int kInt4Warps = 8;

__device__ __forceinline__ float group_sq_error(const float (&r)[32], float s, float inv)
{
    float p[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        float e;
        if (s == 0.0f) {
            e = r[i];
        } else {
            float q = rintf(__fmul_rn(r[i], inv));
            q = fminf(fmaxf(q, -7.0f), 7.0f);
            e = __fsub_rn(r[i], __fmul_rn(q, s));   // q*s is exact
        }
        p[i] = __fmul_rn(e, e);
    }
    // lane 0 of an xor butterfly over strides 16, 8, 4, 2, 1
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1)
#pragma unroll
        for (int i = 0; i < d; ++i)
            p[i] = __fadd_rn(p[i], p[i + d]);
    return p[0];
}

__global__ void __launch_bounds__(kInt4Warps * 32) int4_build_kernel(const float *__restrict__ R,
                                                                     int64_t N, int64_t K,
                                                                     uint8_t *__restrict__ codes,
                                                                     uint16_t *__restrict__ scales,
                                                                     uint8_t *__restrict__ frac)
{
    __shared__ __align__(16) float4 stage[kInt4Warps][256];
    const int lane = threadIdx.x & 31;
    const int wid = threadIdx.x >> 5;
    const int64_t blocks = N * K / kHad;
    const int64_t tasks = (blocks + 3) / 4;
    const int64_t warps_total = (int64_t)gridDim.x * kInt4Warps;
    float4 *st = stage[wid];
    for (int64_t task = (int64_t)blockIdx.x * kInt4Warps + wid; task < tasks; task += warps_total) {
        const int64_t b0 = task * 4;
        const int nb = (int)(blocks - b0 < 4 ? blocks - b0 : 4);
        for (int b = 0; b < nb; ++b) {
            float v[8];
            load_block(R + (b0 + b) * kHad, lane, v);
            fwht256_warp(v, lane);
            const int G0 = 8 * b + (lane >> 3);
            const int G1 = G0 + 4;
            const int w = lane & 7;
            st[G0 * 8 + (w ^ (G0 & 7))] = make_float4(v[0], v[1], v[2], v[3]);
            st[G1 * 8 + (w ^ (G1 & 7))] = make_float4(v[4], v[5], v[6], v[7]);
        }
        __syncwarp();
        const int G = lane;
        if (G < nb * 8) {
            float r[32];
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                float4 q4 = st[G * 8 + (w ^ (G & 7))];
                r[4 * w] = q4.x; r[4 * w + 1] = q4.y; r[4 * w + 2] = q4.z; r[4 * w + 3] = q4.w;
            }
            float a = 0.0f;
#pragma unroll
            for (int i = 0; i < 32; ++i)
                a = fmaxf(a, fabsf(r[i]));
            float best = 0.0f, best_s = 0.0f;
            uint16_t best_h = 0;
            int best_j = 0;
#pragma unroll 1
            for (int j = 0; j < kFracCount; ++j) {
                const float f = __fdiv_rn((float)(50 + 2 * j), 100.0f);
                const __half hs = __float2half_rn(__fdiv_rn(__fmul_rn(f, a), 7.0f));
                const float s = __half2float(hs);
                const float inv = s == 0.0f ? 0.0f : __frcp_rn(s);
                const float mse = group_sq_error(r, s, inv);
                if (j == 0 || mse < best) {
                    best = mse;
                    best_j = j;
                    best_s = s;
                    best_h = __half_as_ushort(hs);
                }
            }
            // codes for the winning scale (same arithmetic as in the sweep)
            const float inv = best_s == 0.0f ? 0.0f : __frcp_rn(best_s);
            uint32_t word[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                int q = 0;
                if (best_s != 0.0f) {
                    float qf = rintf(__fmul_rn(r[i], inv));
                    q = (int)fminf(fmaxf(qf, -7.0f), 7.0f);
                }
                word[i >> 3] |= ((uint32_t)q & 0xFu) << (4 * (i & 7));
            }
            const int64_t gidx = b0 * 8 + G;     // flat group index
            reinterpret_cast<uint4 *>(codes)[gidx] = make_uint4(word[0], word[1], word[2], word[3]);
            scales[gidx] = best_h;
            if (frac)
                frac[gidx] = (uint8_t)best_j;
        }
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------
// int4 forward prologue: xb = bf16(H x), [M, K]
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) rotate_bf16_kernel(const uint16_t *__restrict__ x, int64_t M,
                                                          int64_t K, uint16_t *__restrict__ xb)
{
    const int lane = threadIdx.x & 31;
    const int64_t warps_total = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t tasks = M * (K / kHad);
    for (int64_t task = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); task < tasks;
         task += warps_total) {
        float v[8];
        load_block(x + task * kHad, lane, v);
        fwht256_warp(v, lane);
        uint2 lo, hi;
        lo.x = f32_to_bf16_bits(v[0]) | (f32_to_bf16_bits(v[1]) << 16);
        lo.y = f32_to_bf16_bits(v[2]) | (f32_to_bf16_bits(v[3]) << 16);
        hi.x = f32_to_bf16_bits(v[4]) | (f32_to_bf16_bits(v[5]) << 16);
        hi.y = f32_to_bf16_bits(v[6]) | (f32_to_bf16_bits(v[7]) << 16);
        uint16_t *o = xb + task * kHad;
        *reinterpret_cast<uint2 *>(o + 4 * lane) = lo;
        *reinterpret_cast<uint2 *>(o + 128 + 4 * lane) = hi;
    }
}

// ---------------------------------------------------------------------------
// int4 "dequant-first": wb[n, k] = bf16(q s), 8 values per thread
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) dequant_int4_kernel(const uint32_t *__restrict__ codes,
                                                           const uint16_t *__restrict__ scales,
                                                           int64_t total8, uint4 *__restrict__ wb)
{
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total8;
         i += (int64_t)gridDim.x * blockDim.x) {
        const uint32_t c = __ldg(codes + i);
        const float s = __half2float(__ushort_as_half(__ldg(scales + (i >> 2))));  // 4 words per group
        uint32_t o[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            int q0 = (int)((c >> (8 * p)) & 0xFu);
            int q1 = (int)((c >> (8 * p + 4)) & 0xFu);
            q0 = q0 >= 8 ? q0 - 16 : q0;
            q1 = q1 >= 8 ? q1 - 16 : q1;
            o[p] = f32_to_bf16_bits(__fmul_rn((float)q0, s)) | (f32_to_bf16_bits(__fmul_rn((float)q1, s)) << 16);
        }
        wb[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// ---------------------------------------------------------------------------
// low-rank operand preparation: udup[n] = [U[n, 0:32] | U[n, 0:32]] (bf16
// [N, 64], the B operand of the low-rank MMA step) and dt = lora_down^T
// (bf16 [32, K], for contiguous fragment loads).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) lora_prep_kernel(const uint16_t *__restrict__ U, int64_t N,
                                                        const uint16_t *__restrict__ D, int64_t K,
                                                        uint16_t *__restrict__ udup,
                                                        uint16_t *__restrict__ dt)
{
    const int64_t nU = udup ? N * 64 : 0;
    const int64_t nD = dt ? K * 32 : 0;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nU + nD;
         i += (int64_t)gridDim.x * blockDim.x) {
        if (i < nU) {
            const int64_t n = i >> 6;
            udup[i] = U[n * 32 + (i & 31)];
        } else {
            const int64_t j = i - nU;          // j = r * K + k
            const int64_t r = j / K;
            const int64_t k = j - r * K;
            dt[j] = D[k * 32 + r];
        }
    }
}

// ---------------------------------------------------------------------------
// low-rank input t = x . lora_down (fp32 accumulation) on mma.sync bf16.
// A CTA takes 16 rows; its 8 warps split K and their partial [16, 32] tiles
// are summed in a fixed order.  Output either fp32 t [M, 32], or the split
// form used by the forward's low-rank MMA step: with beta = g_x g_w (1 when
// either is NULL or the product is 0), tt = t / beta, hi = bf16(tt),
// lo = bf16(tt - hi), tsplit[m] = [hi[0:32] | lo[0:32]] (bf16 [M, 64]).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
                 "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};\n"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(256) lowrank_t_kernel(const uint16_t *__restrict__ x, int64_t M, int64_t K,
                                                        const uint16_t *__restrict__ dt,
                                                        const float *__restrict__ g_x,
                                                        const float *__restrict__ g_w,
                                                        float *__restrict__ t_out,
                                                        uint16_t *__restrict__ tsplit)
{
    __shared__ float part[8][16][33];
    const int lane = threadIdx.x & 31;
    const int wid = threadIdx.x >> 5;
    const int gq = lane >> 2;       // groupID
    const int tq = lane & 3;        // thread in group
    const int64_t m0 = (int64_t)blockIdx.x * 16;
    const int64_t kslice = K / 8;
    const int64_t kbeg = wid * kslice;
    const int64_t r0 = m0 + gq, r1 = m0 + gq + 8;
    const uint32_t *x0 = reinterpret_cast<const uint32_t *>(x + (r0 < M ? r0 : 0) * K);
    const uint32_t *x1 = reinterpret_cast<const uint32_t *>(x + (r1 < M ? r1 : 0) * K);
    const uint32_t mask0 = r0 < M ? 0xffffffffu : 0u;
    const uint32_t mask1 = r1 < M ? 0xffffffffu : 0u;
    float c[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i)
            c[nt][i] = 0.0f;
    for (int64_t k0 = kbeg; k0 < kbeg + kslice; k0 += 16) {
        const int64_t ka = (k0 + 2 * tq) >> 1;      // 32-bit word index
        uint32_t a[4];
        a[0] = __ldg(x0 + ka) & mask0;
        a[1] = __ldg(x1 + ka) & mask1;
        a[2] = __ldg(x0 + ka + 4) & mask0;
        a[3] = __ldg(x1 + ka + 4) & mask1;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            const uint32_t *drow = reinterpret_cast<const uint32_t *>(dt + (int64_t)(8 * nt + gq) * K);
            const uint32_t b0 = __ldg(drow + ka);
            const uint32_t b1 = __ldg(drow + ka + 4);
            mma_bf16_16816(c[nt], a, b0, b1);
        }
    }
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
        part[wid][gq][8 * nt + 2 * tq] = c[nt][0];
        part[wid][gq][8 * nt + 2 * tq + 1] = c[nt][1];
        part[wid][gq + 8][8 * nt + 2 * tq] = c[nt][2];
        part[wid][gq + 8][8 * nt + 2 * tq + 1] = c[nt][3];
    }
    __syncthreads();
    float beta = 1.0f;
    if (g_x && g_w) {
        const float b = __fmul_rn(*g_x, *g_w);
        beta = b == 0.0f ? 1.0f : b;
    }
    for (int e = threadIdx.x; e < 16 * 32; e += blockDim.x) {
        const int row = e >> 5, col = e & 31;
        const int64_t m = m0 + row;
        if (m >= M)
            continue;
        float s = 0.0f;
#pragma unroll
        for (int w = 0; w < 8; ++w)
            s = __fadd_rn(s, part[w][row][col]);
        if (t_out)
            t_out[m * 32 + col] = s;
        if (tsplit) {
            const float tt = __fdiv_rn(s, beta);
            const uint32_t hi = f32_to_bf16_bits(tt);
            const uint32_t lo = f32_to_bf16_bits(__fsub_rn(tt, bf16_bits_to_f32(hi)));
            tsplit[m * 64 + col] = (uint16_t)hi;
            tsplit[m * 64 + 32 + col] = (uint16_t)lo;
        }
    }
}

// ---------------------------------------------------------------------------
// bf16 reconstruct.  CTA = (256-column block kb, 128-row chunk); lora_down for
// the block is staged transposed in shared memory as fp32, each warp walks 16
// rows: d from the payload, H256 over the block, the rank-32 fma chain, bf16.
// ---------------------------------------------------------------------------
constexpr int kReconRows = 128;
constexpr int kDtPitch = 260;   // floats per staged row (16-byte aligned, fewer bank conflicts)

__global__ void __launch_bounds__(256) reconstruct_kernel(int fmt, const uint8_t *__restrict__ codes,
                                                          const void *__restrict__ scales,
                                                          const float *__restrict__ g_w,
                                                          const uint16_t *__restrict__ U,
                                                          const uint16_t *__restrict__ D, int64_t N,
                                                          int64_t K, int with_lowrank,
                                                          uint16_t *__restrict__ W)
{
    extern __shared__ __align__(16) float dts[];   // [32][kDtPitch]
    const int lane = threadIdx.x & 31;
    const int wid = threadIdx.x >> 5;
    const int64_t kb = blockIdx.x;
    const int64_t C = K / kSfBlock;
    if (with_lowrank) {
        const uint16_t *Dk = D + kb * kHad * kRank;
        for (int i = threadIdx.x; i < kHad * kRank; i += blockDim.x)
            dts[(i & 31) * kDtPitch + (i >> 5)] = bf16_bits_to_f32(Dk[i]);
    }
    __syncthreads();
    const float g = fmt == 2 ? *g_w : 0.0f;
    const int64_t n_end_c = (int64_t)(blockIdx.y + 1) * kReconRows;
    const int64_t n_end = N < n_end_c ? N : n_end_c;
    for (int64_t n = (int64_t)blockIdx.y * kReconRows + wid; n < n_end; n += 8) {
        const uint8_t *crow = codes + n * (K / 2) + kb * (kHad / 2);
        const uint32_t c0 = *reinterpret_cast<const uint16_t *>(crow + 2 * lane);
        const uint32_t c1 = *reinterpret_cast<const uint16_t *>(crow + 64 + 2 * lane);
        float v[8];
        if (fmt == 1) {
            const uint16_t *srow = reinterpret_cast<const uint16_t *>(scales) + n * (K / kGroup) + kb * 8;
            const float s0 = __half2float(__ushort_as_half(srow[lane >> 3]));
            const float s1 = __half2float(__ushort_as_half(srow[4 + (lane >> 3)]));
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                int q0 = (int)((c0 >> (4 * i)) & 0xFu);
                int q1 = (int)((c1 >> (4 * i)) & 0xFu);
                q0 = q0 >= 8 ? q0 - 16 : q0;
                q1 = q1 >= 8 ? q1 - 16 : q1;
                v[i] = __fmul_rn((float)q0, s0);
                v[4 + i] = __fmul_rn((float)q1, s1);
            }
        } else {
            const uint8_t *sf = reinterpret_cast<const uint8_t *>(scales);
            const int64_t cc = kb * (kHad / kSfBlock) + (lane >> 2);
            const float d0 = ue4m3_value(sf[sf_offset(n, cc, C)]);
            const float d1 = ue4m3_value(sf[sf_offset(n, cc + 8, C)]);
            const float2 e00 = e2m1x2_value(c0 & 0xFFu), e01 = e2m1x2_value(c0 >> 8);
            const float2 e10 = e2m1x2_value(c1 & 0xFFu), e11 = e2m1x2_value(c1 >> 8);
            const float e[8] = {e00.x, e00.y, e01.x, e01.y, e10.x, e10.y, e11.x, e11.y};
#pragma unroll
            for (int i = 0; i < 8; ++i)
                v[i] = __fmul_rn(__fmul_rn(e[i], i < 4 ? d0 : d1), g);
        }
        fwht256_warp(v, lane);
        if (with_lowrank) {
            float u[kRank];
            const uint4 *up = reinterpret_cast<const uint4 *>(U + n * kRank);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 w = __ldg(up + q);
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    u[8 * q + 2 * p] = bf16_bits_to_f32(ww[p] & 0xFFFFu);
                    u[8 * q + 2 * p + 1] = bf16_bits_to_f32(ww[p] >> 16);
                }
            }
            float L[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int r = 0; r < kRank; ++r) {
                const float4 a = *reinterpret_cast<const float4 *>(dts + r * kDtPitch + 4 * lane);
                const float4 b = *reinterpret_cast<const float4 *>(dts + r * kDtPitch + 128 + 4 * lane);
                L[0] = __fmaf_rn(u[r], a.x, L[0]);
                L[1] = __fmaf_rn(u[r], a.y, L[1]);
                L[2] = __fmaf_rn(u[r], a.z, L[2]);
                L[3] = __fmaf_rn(u[r], a.w, L[3]);
                L[4] = __fmaf_rn(u[r], b.x, L[4]);
                L[5] = __fmaf_rn(u[r], b.y, L[5]);
                L[6] = __fmaf_rn(u[r], b.z, L[6]);
                L[7] = __fmaf_rn(u[r], b.w, L[7]);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i)
                v[i] = __fadd_rn(L[i], v[i]);
        }
        uint2 lo, hi;
        lo.x = f32_to_bf16_bits(v[0]) | (f32_to_bf16_bits(v[1]) << 16);
        lo.y = f32_to_bf16_bits(v[2]) | (f32_to_bf16_bits(v[3]) << 16);
        hi.x = f32_to_bf16_bits(v[4]) | (f32_to_bf16_bits(v[5]) << 16);
        hi.y = f32_to_bf16_bits(v[6]) | (f32_to_bf16_bits(v[7]) << 16);
        uint16_t *o = W + n * K + kb * kHad;
        *reinterpret_cast<uint2 *>(o + 4 * lane) = lo;
        *reinterpret_cast<uint2 *>(o + 128 + 4 * lane) = hi;
    }
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

cudaError_t launch_absmax_rot_f32(const float *in, int64_t rows, int64_t K, uint32_t *amax, int sms,
                                  cudaStream_t s)
{
    absmax_rot_kernel<float><<<grid_for(rows * (K / kHad), 8, sms, 8), 256, 0, s>>>(in, rows, K, amax);
    return cudaGetLastError();
}

cudaError_t launch_absmax_rot_bf16(const uint16_t *in, int64_t rows, int64_t K, uint32_t *amax, int sms,
                                   cudaStream_t s)
{
    absmax_rot_kernel<uint16_t><<<grid_for(rows * (K / kHad), 8, sms, 8), 256, 0, s>>>(in, rows, K, amax);
    return cudaGetLastError();
}

cudaError_t launch_nvfp4_quant_f32(const float *in, int64_t rows, int64_t K, const uint32_t *amax,
                                   const float *g_static, float *g_out, uint8_t *codes, uint8_t *sf,
                                   int sms, cudaStream_t s)
{
    const int64_t rows_pad = (rows + 127) / 128 * 128;
    nvfp4_quant_kernel<float><<<grid_for(rows_pad * (K / kHad), 8, sms, 8), 256, 0, s>>>(
        in, rows, rows_pad, K, amax, g_static, g_out, codes, sf);
    return cudaGetLastError();
}

cudaError_t launch_nvfp4_quant_bf16(const uint16_t *in, int64_t rows, int64_t K, const uint32_t *amax,
                                    const float *g_static, float *g_out, uint8_t *codes, uint8_t *sf,
                                    int sms, cudaStream_t s)
{
    const int64_t rows_pad = (rows + 127) / 128 * 128;
    nvfp4_quant_kernel<uint16_t><<<grid_for(rows_pad * (K / kHad), 8, sms, 8), 256, 0, s>>>(
        in, rows, rows_pad, K, amax, g_static, g_out, codes, sf);
    return cudaGetLastError();
}

cudaError_t launch_int4_build(const float *R, int64_t N, int64_t K, uint8_t *codes, uint16_t *scales,
                              uint8_t *frac, int sms, cudaStream_t s)
{
    const int64_t tasks = (N * K / kHad + 3) / 4;
    int4_build_kernel<<<grid_for(tasks, kInt4Warps, sms, 4), kInt4Warps * 32, 0, s>>>(R, N, K, codes,
                                                                                      scales, frac);
    return cudaGetLastError();
}

cudaError_t launch_rotate_bf16(const uint16_t *x, int64_t M, int64_t K, uint16_t *xb, int sms, cudaStream_t s)
{
    rotate_bf16_kernel<<<grid_for(M * (K / kHad), 8, sms, 8), 256, 0, s>>>(x, M, K, xb);
    return cudaGetLastError();
}

cudaError_t launch_dequant_int4(const uint8_t *codes, const uint16_t *scales, int64_t N, int64_t K,
                                uint16_t *wb, int sms, cudaStream_t s)
{
    const int64_t total8 = N * K / 8;
    dequant_int4_kernel<<<grid_for(total8, 256, sms, 8), 256, 0, s>>>(
        reinterpret_cast<const uint32_t *>(codes), scales, total8, reinterpret_cast<uint4 *>(wb));
    return cudaGetLastError();
}

cudaError_t launch_lora_prep(const uint16_t *U, int64_t N, const uint16_t *D, int64_t K, uint16_t *udup,
                             uint16_t *dt, int sms, cudaStream_t s)
{
    const int64_t total = (udup ? N * 64 : 0) + (dt ? K * 32 : 0);
    lora_prep_kernel<<<grid_for(total, 256, sms, 4), 256, 0, s>>>(U, N, D, K, udup, dt);
    return cudaGetLastError();
}

cudaError_t launch_lowrank_t(const uint16_t *x, int64_t M, int64_t K, const uint16_t *dt, const float *g_x,
                             const float *g_w, float *t_out, uint16_t *tsplit, cudaStream_t s)
{
    const int64_t grid = (M + 15) / 16;
    lowrank_t_kernel<<<(unsigned)grid, 256, 0, s>>>(x, M, K, dt, g_x, g_w, t_out, tsplit);
    return cudaGetLastError();
}

cudaError_t launch_reconstruct(int fmt, const uint8_t *codes, const void *scales, const float *g_w,
                               const uint16_t *U, const uint16_t *D, int64_t N, int64_t K, int with_lowrank,
                               uint16_t *W, cudaStream_t s)
{
    // 32 x 260 floats = 33,280 bytes of dynamic shared memory: under the 48 KB default
    const int smem = with_lowrank ? kRank * kDtPitch * (int)sizeof(float) : 0;
    dim3 grid((unsigned)(K / kHad), (unsigned)((N + kReconRows - 1) / kReconRows));
    reconstruct_kernel<<<grid, 256, smem, s>>>(fmt, codes, scales, g_w, U, D, N, K, with_lowrank, W);
    return cudaGetLastError();
}

}  // namespace sq
