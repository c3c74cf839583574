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
#include "sq_ptx.cuh"

namespace sq {

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
// may shuffle).  total_blocks may exceed the tensor (zero blocks).
template <typename T, typename F>
__device__ __forceinline__ void stream_blocks(const CUtensorMap *tm, int64_t total_blocks, uint32_t *status, F &&f)
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
    float m = 0.0f;
    stream_blocks<T>(&tm, blocks, nullptr, [&](int64_t, float (&v)[32], bool) {
        fwht256_l32(v, lane);
#pragma unroll
        for (int i = 0; i < 32; ++i)
            m = fmaxf(m, fabsf(v[i]));
    });
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
                                                                     uint8_t *__restrict__ sf)
{
    const int lane = threadIdx.x & 31;
    const int q = lane & 7;
    const float g = g_static ? *g_static : __fdiv_rn(__uint_as_float(*amax), 2688.0f);
    if (g_out && blockIdx.x == 0 && threadIdx.x == 0)
        *g_out = g;
    const float sixg = __fmul_rn(6.0f, g);
    const int64_t kb_per_row = K / kHad;
    const int64_t C = K / kSfBlock;
    stream_blocks<T>(&tm, rows_pad * kb_per_row, nullptr, [&](int64_t b, float (&v)[32], bool valid) {
        fwht256_l32(v, lane);
        if (!valid)
            return;
        const int64_t row = b / kb_per_row;
        const int64_t kb = b - row * kb_per_row;
        uint32_t word[4];
        uint32_t sfc[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float bmax = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i)
                bmax = fmaxf(bmax, fabsf(v[16 * h + i]));
            uint32_t code = 0;
            uint32_t w0 = 0, w1 = 0;
            if (g != 0.0f) {
                code = to_ue4m3(__fdiv_rn(bmax, sixg));
                if (code != 0) {
                    const float inv = __frcp_rn(__fmul_rn(ue4m3_value(code), g));
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        w0 |= to_e2m1x2(__fmul_rn(v[16 * h + 2 * i], inv), __fmul_rn(v[16 * h + 2 * i + 1], inv))
                              << (8 * i);
                        w1 |= to_e2m1x2(__fmul_rn(v[16 * h + 8 + 2 * i], inv),
                                        __fmul_rn(v[16 * h + 8 + 2 * i + 1], inv))
                              << (8 * i);
                    }
                }
            }
            word[2 * h] = w0;
            word[2 * h + 1] = w1;
            sfc[h] = code;
        }
        if (row < rows)
            *reinterpret_cast<uint4 *>(codes + row * (K / 2) + kb * (kHad / 2) + 16 * q) =
                make_uint4(word[0], word[1], word[2], word[3]);
        // scale columns 2q, 2q+1 of the block are adjacent bytes of the tiled layout
        *reinterpret_cast<uint16_t *>(sf + sf_offset(row, kb * (kHad / kSfBlock) + 2 * q, C)) =
            (uint16_t)(sfc[0] | (sfc[1] << 8));
    });
}

// ---------------------------------------------------------------------------
// int4 group-32 builder.  With the 8-lane Hadamard layout every lane holds one
// whole group of 32 rotated values and sweeps the 26 scale fractions in
// registers (group index = 8 * block + lane % 8).
// ---------------------------------------------------------------------------
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

__global__ void __launch_bounds__(kStreamThreads) int4_build_kernel(const __grid_constant__ CUtensorMap tm,
                                                                    int64_t blocks, uint8_t *__restrict__ codes,
                                                                    uint16_t *__restrict__ scales,
                                                                    uint8_t *__restrict__ frac)
{
    const int lane = threadIdx.x & 31;
    stream_blocks<float>(&tm, blocks, nullptr, [&](int64_t b, float (&r)[32], bool valid) {
        fwht256_l32(r, lane);
        if (!valid)
            return;
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
        const int64_t gidx = 8 * b + (lane & 7);     // flat group index
        reinterpret_cast<uint4 *>(codes)[gidx] = make_uint4(word[0], word[1], word[2], word[3]);
        scales[gidx] = best_h;
        if (frac)
            frac[gidx] = (uint8_t)best_j;
    });
}

// ---------------------------------------------------------------------------
// int4 forward prologue: xb = bf16(H x), [M, K]
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kStreamThreads) rotate_bf16_kernel(const __grid_constant__ CUtensorMap tm,
                                                                     int64_t blocks, uint16_t *__restrict__ xb)
{
    const int lane = threadIdx.x & 31;
    stream_blocks<uint16_t>(&tm, blocks, nullptr, [&](int64_t b, float (&v)[32], bool valid) {
        fwht256_l32(v, lane);
        if (!valid)
            return;
        uint4 *o = reinterpret_cast<uint4 *>(xb + b * kHad + 32 * (lane & 7));
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                w[j] = f32_to_bf16_bits(v[8 * i + 2 * j]) | (f32_to_bf16_bits(v[8 * i + 2 * j + 1]) << 16);
            o[i] = make_uint4(w[0], w[1], w[2], w[3]);
        }
    });
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
// Activation pass 1: one read of x for two results.
//   amax (optional): max |H x| over the whole tensor (the activation global
//                    scale's input), from the 8-lane Hadamard transform;
//   t32 (optional):  t = x . lora_down, fp32 [M, 32], on mma.sync bf16 tensor
//                    cores (fp32 accumulation; each CTA sums its partials in a
//                    fixed order, so t is deterministic).
// A CTA owns 16 rows and walks K in 256-column chunks; the x chunk (16 x 256)
// and the lora_down chunk (256 x 32) are staged in shared memory by cp.async,
// double buffered.  Warps 0-3 transform rows 4w..4w+3, warps 4-7 run k-steps
// 4(w-4)..4(w-4)+3 of the chunk for all 32 outputs.
// x tile: 16-byte chunk c of row r sits at c ^ ((c >> 2) & 7) ^ (r & 7), which
// keeps both the transform's per-row reads and ldmatrix conflict free; D tile:
// chunk c of k-row k sits at c ^ ((k >> 1) & 3).
// ---------------------------------------------------------------------------
constexpr int kP1Rows = 16;
constexpr int kP1XBytes = kP1Rows * kHad * 2;      // 8 KB
constexpr int kP1DBytes = kHad * kRank * 2;        // 16 KB
constexpr int kP1BufBytes = kP1XBytes + kP1DBytes;
constexpr int kP1Smem = 2 * kP1BufBytes;           // 48 KB

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

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
                 "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};\n"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t p1_xoff(int r, int c)
{
    return (uint32_t)(r * 512 + 16 * (c ^ ((c >> 2) & 7) ^ (r & 7)));
}

__device__ __forceinline__ uint32_t p1_doff(int k, int c)
{
    return (uint32_t)(k * 64 + 16 * (c ^ ((k >> 1) & 3)));
}

__global__ void __launch_bounds__(256) act_pass1_kernel(const uint16_t *__restrict__ x, int64_t M, int64_t K,
                                                        const uint16_t *__restrict__ D,
                                                        uint32_t *__restrict__ amax, float *__restrict__ t32)
{
    extern __shared__ __align__(128) uint8_t p1_smem[];
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int64_t m0 = (int64_t)blockIdx.x * kP1Rows;
    const int nkb = (int)(K / kHad);
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(p1_smem);

    auto issue = [&](int kb, int buf) {
        const uint32_t xs = sbase + buf * kP1BufBytes;
        const uint32_t ds = xs + kP1XBytes;
#pragma unroll
        for (int i = 0; i < 2; ++i) {                 // x: 16 rows x 32 chunks
            const int e = tid + 256 * i;
            const int r = e >> 5, c = e & 31;
            const int64_t row = m0 + r;
            const bool ok = row < M;
            const uint16_t *src = x + (ok ? row : 0) * K + (int64_t)kb * kHad + 8 * c;
            cp_async16(xs + p1_xoff(r, c), src, ok ? 16u : 0u);
        }
        if (t32) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {             // D: 256 k-rows x 4 chunks
                const int e = tid + 256 * i;
                const int k = e >> 2, c = e & 3;
                cp_async16(ds + p1_doff(k, c), D + ((int64_t)kb * kHad + k) * kRank + 8 * c, 16u);
            }
        }
        cp_async_commit();
    };

    float m = 0.0f;
    float acc[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i)
            acc[nt][i] = 0.0f;

    issue(0, 0);
    for (int kb = 0; kb < nkb; ++kb) {
        const int buf = kb & 1;
        if (kb + 1 < nkb) {
            issue(kb + 1, buf ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const uint32_t xs = sbase + buf * kP1BufBytes;
        const uint32_t ds = xs + kP1XBytes;
        if (warp < 4) {
            if (amax) {
                const int r = 4 * warp + (lane >> 3);
                const int q = lane & 7;
                float v[32];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint4 a = *reinterpret_cast<const uint4 *>(p1_smem + (p1_xoff(r, 4 * q + i) +
                                                                                 buf * kP1BufBytes));
                    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        v[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
                        v[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
                    }
                }
                fwht256_l32(v, lane);
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    m = fmaxf(m, fabsf(v[i]));
            }
        } else if (t32) {
            const int w4 = warp - 4;
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const int ks = 4 * w4 + s;            // k-step: columns 16ks..16ks+15 of the chunk
                // A 16x16: matrices (rows 0-7 | 8-15) x (k 0-7 | 8-15); lane provides row (lane & 15)
                uint32_t a[4];
                const int ar = lane & 15;
                const int ac = 2 * ks + (lane >> 4);
                ldmatrix_x4(xs + p1_xoff(ar, ac), a);
                // B: (k 0-7 | 8-15) x (n-tile pair), transposed load of row-major D
#pragma unroll
                for (int np = 0; np < 2; ++np) {
                    uint32_t b[4];
                    const int bk = 16 * ks + (lane & 7) + 8 * ((lane >> 3) & 1);
                    const int bc = 2 * np + (lane >> 4);
                    ldmatrix_x4_trans(ds + p1_doff(bk, bc), b);
                    mma_bf16_16816(acc[2 * np], a, b[0], b[1]);
                    mma_bf16_16816(acc[2 * np + 1], a, b[2], b[3]);
                }
            }
        }
        __syncthreads();
    }

    if (amax) {
#pragma unroll
        for (int xx = 16; xx >= 1; xx >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, xx));
    }
    // partial t tiles of warps 4-7 and the absmax reduce through the (now idle) smem
    float *part = reinterpret_cast<float *>(p1_smem);          // [4][16][33]
    float *wmax = part + 4 * 16 * 33;                           // [8]
    if (warp >= 4 && t32) {
        const int w4 = warp - 4;
        const int g = lane >> 2, tq = lane & 3;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            part[(w4 * 16 + g) * 33 + 8 * nt + 2 * tq] = acc[nt][0];
            part[(w4 * 16 + g) * 33 + 8 * nt + 2 * tq + 1] = acc[nt][1];
            part[(w4 * 16 + g + 8) * 33 + 8 * nt + 2 * tq] = acc[nt][2];
            part[(w4 * 16 + g + 8) * 33 + 8 * nt + 2 * tq + 1] = acc[nt][3];
        }
    }
    if (lane == 0)
        wmax[warp] = m;
    __syncthreads();
    if (amax && tid == 0) {
        float b = 0.0f;
        for (int w = 0; w < 4; ++w)
            b = fmaxf(b, wmax[w]);
        atomic_max_nonneg(amax, b);
    }
    if (t32) {
        for (int e = tid; e < kP1Rows * kRank; e += 256) {
            const int r = e >> 5, col = e & 31;
            if (m0 + r >= M)
                continue;
            float v = 0.0f;
#pragma unroll
            for (int w = 0; w < 4; ++w)
                v = __fadd_rn(v, part[(w * 16 + r) * 33 + col]);
            t32[(m0 + r) * kRank + col] = v;
        }
    }
}

// ---------------------------------------------------------------------------
// low-rank operands of the forward's extra MMA step.  With beta = g_x g_w (1
// when either pointer is NULL or the product is 0): tt = t / beta,
// tsplit[m] = [bf16(tt) | bf16(tt - bf16(tt))] (bf16 [M, 64]), and
// udup[n] = [U[n] | U[n]] (bf16 [N, 64]).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) lowrank_finish_kernel(const float *__restrict__ t32, int64_t M,
                                                             const float *__restrict__ g_x,
                                                             const float *__restrict__ g_w,
                                                             uint16_t *__restrict__ tsplit,
                                                             const uint16_t *__restrict__ U, int64_t N,
                                                             uint16_t *__restrict__ udup)
{
    float beta = 1.0f;
    if (g_x && g_w) {
        const float b = __fmul_rn(*g_x, *g_w);
        beta = b == 0.0f ? 1.0f : b;
    }
    const int64_t nT = M * kRank, nU = N * kRank;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nT + nU;
         i += (int64_t)gridDim.x * blockDim.x) {
        if (i < nT) {
            const int64_t m = i >> 5, col = i & 31;
            const float tt = __fdiv_rn(t32[i], beta);
            const uint32_t hi = f32_to_bf16_bits(tt);
            const uint32_t lo = f32_to_bf16_bits(__fsub_rn(tt, bf16_bits_to_f32(hi)));
            tsplit[m * 64 + col] = (uint16_t)hi;
            tsplit[m * 64 + 32 + col] = (uint16_t)lo;
        } else {
            const int64_t j = i - nT;
            const int64_t n = j >> 5, col = j & 31;
            const uint16_t u = U[j];
            udup[n * 64 + col] = u;
            udup[n * 64 + 32 + col] = u;
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

// streamer launch: tensor map over `in` as [rows * K / 32, 32], persistent grid
template <typename T>
static bool stream_map(CUtensorMap *tm, const T *in, int64_t rows, int64_t K)
{
    const bool f32 = sizeof(T) == 4;
    return make_tmap(tm, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (int)sizeof(T), in,
                     32, (uint64_t)(rows * K / 32), 32, 256, f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
}

// shared-memory opt-in, once per device and kernel
template <typename T, typename Kern>
static cudaError_t stream_attr(Kern k)
{
    constexpr int kMaxDev = 64;
    static bool done[kMaxDev];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev)
        return cudaErrorInvalidDevice;
    if (done[dev])
        return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, StreamCfg<T>::kSmem);
    if (e == cudaSuccess)
        done[dev] = true;
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
    cudaError_t e = stream_attr<T>(absmax_rot_kernel<T>);
    if (e != cudaSuccess)
        return e;
    const int64_t blocks = rows * (K / kHad);
    absmax_rot_kernel<T><<<stream_grid(blocks, sms, sizeof(T) == 4 ? 2 : 3), kStreamThreads, StreamCfg<T>::kSmem, s>>>(
        tm, blocks, amax);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_nvfp4_quant(const T *in, int64_t rows, int64_t K, const uint32_t *amax, const float *g_static,
                                      float *g_out, uint8_t *codes, uint8_t *sf, int sms, cudaStream_t s)
{
    CUtensorMap tm;
    if (!stream_map(&tm, in, rows, K))
        return cudaErrorInvalidValue;
    cudaError_t e = stream_attr<T>(nvfp4_quant_kernel<T>);
    if (e != cudaSuccess)
        return e;
    const int64_t rows_pad = (rows + 127) / 128 * 128;
    nvfp4_quant_kernel<T><<<stream_grid(rows_pad * (K / kHad), sms, sizeof(T) == 4 ? 2 : 3), kStreamThreads,
                            StreamCfg<T>::kSmem, s>>>(tm, rows, rows_pad, K, amax, g_static, g_out, codes, sf);
    return cudaGetLastError();
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
    return launch_nvfp4_quant(in, rows, K, amax, g_static, g_out, codes, sf, sms, s);
}

cudaError_t launch_nvfp4_quant_bf16(const uint16_t *in, int64_t rows, int64_t K, const uint32_t *amax,
                                    const float *g_static, float *g_out, uint8_t *codes, uint8_t *sf, int sms,
                                    cudaStream_t s)
{
    return launch_nvfp4_quant(in, rows, K, amax, g_static, g_out, codes, sf, sms, s);
}

cudaError_t launch_int4_build(const float *R, int64_t N, int64_t K, uint8_t *codes, uint16_t *scales,
                              uint8_t *frac, int sms, cudaStream_t s)
{
    CUtensorMap tm;
    if (!stream_map(&tm, R, N, K))
        return cudaErrorInvalidValue;
    cudaError_t e = stream_attr<float>(int4_build_kernel);
    if (e != cudaSuccess)
        return e;
    const int64_t blocks = N * K / kHad;
    int4_build_kernel<<<stream_grid(blocks, sms, 2), kStreamThreads, StreamCfg<float>::kSmem, s>>>(tm, blocks, codes,
                                                                                                   scales, frac);
    return cudaGetLastError();
}

cudaError_t launch_rotate_bf16(const uint16_t *x, int64_t M, int64_t K, uint16_t *xb, int sms, cudaStream_t s)
{
    CUtensorMap tm;
    if (!stream_map(&tm, x, M, K))
        return cudaErrorInvalidValue;
    cudaError_t e = stream_attr<uint16_t>(rotate_bf16_kernel);
    if (e != cudaSuccess)
        return e;
    const int64_t blocks = M * (K / kHad);
    rotate_bf16_kernel<<<stream_grid(blocks, sms, 3), kStreamThreads, StreamCfg<uint16_t>::kSmem, s>>>(tm, blocks, xb);
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

cudaError_t launch_act_pass1(const uint16_t *x, int64_t M, int64_t K, const uint16_t *D, uint32_t *amax,
                             float *t32, cudaStream_t s)
{
    const int64_t grid = (M + kP1Rows - 1) / kP1Rows;
    act_pass1_kernel<<<(unsigned)grid, 256, kP1Smem, s>>>(x, M, K, D, amax, t32);
    return cudaGetLastError();
}

cudaError_t launch_lowrank_finish(const float *t32, int64_t M, const float *g_x, const float *g_w,
                                  uint16_t *tsplit, const uint16_t *U, int64_t N, uint16_t *udup, int sms,
                                  cudaStream_t s)
{
    lowrank_finish_kernel<<<grid_for((M + N) * kRank, 256, sms, 4), 256, 0, s>>>(t32, M, g_x, g_w, tsplit, U, N,
                                                                                  udup);
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
