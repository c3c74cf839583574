// sq_gemm.cu -- persistent, warp-specialised tcgen05 GEMM of the W4 forward:
//
//   y[M, N] = beta * ( A B^T + Tsplit Udup^T )            (fp32 out)
//
//   NVFP4 path: A = e2m1 activation codes [M, K/2] with ue4m3 block-16 scales,
//               B = e2m1 weight codes [N, K/2] with ue4m3 scales (tiled layout),
//               block-scaled MMA (kind::mxf4nvf4.block16), beta = g_x * g_w.
//   int4 / int8 path: A = bf16(H x) [M, K] by TMA; B = bf16(q s) by TMA from a
//               ring of R slots of 256 rows in global memory (L2-resident),
//               which the kernel's own dequantising warps fill from the 4- or
//               8-bit payload, each 256-row tile of W once (not once per M
//               tile); kind::f16, beta = 1.
//   bf16 path:  A and B bf16 by TMA (the input gradient's GEMM).
//   Low-rank:   Tsplit [M, 64] = [hi | lo] bf16 split of t / beta, Udup [N, 64]
//               = [U | U]; one extra kind::f16 K-step into the same accumulator
//               adds (t / beta) U^T, so the epilogue only scales by beta.
//
// (SquareQ README: the op-level parity paragraph of the FP4 forward names the
// block-scaled GEMM and its epilogue; the "Residual codecs" paragraph makes the
// int4 codec dequant-first.)
//
// CTA tile 128 x 256, one CTA per SM, 6 warps (+4 scale warps on the NVFP4 path,
// +4 dequantising warps on the int4 / int8 paths):
//   warps 0-3  epilogue: tcgen05.ld of their 32 accumulator lanes, scale,
//              128B-swizzled staging in shared memory, TMA store;
//   warp 4     TMA producer (tiles of A, B, the scale factors, the low-rank
//              operands) into a ring of shared-memory stages;
//   warp 5     tensor-memory allocator and the single MMA-issuing thread;
//   warps 6-9  (NVFP4) move each MMA's ue4m3 scale factors from shared memory
//              into tensor memory with tcgen05.st, one 32-lane sub-partition
//              per warp, so the tensor pipe spends no cycles on copies;
//              (int4 / int8) write this CTA's share of each W tile its cluster
//              multiplies into the ring (see "W ring" below), from the start of
//              the kernel (they read only the weight payload, not the outputs of
//              the preceding kernels).
// Tensor memory (512 columns).  NVFP4: two accumulator slots at columns 0 and
// 64 that overlap in columns 64..255, and four 48-column scale-factor buffers
// at 320..511 (four stages of scale factors between the scale warps and the
// MMAs that read them).  The epilogue takes the overlapping 192 columns of a
// tile first -- four chunks into registers, two of them parked in its staging
// buffers, then the last two -- and releases the MMA thread, which starts the
// next tile while the rest drains: accumulator double buffering in 320
// columns.  bf16 / int4 / int8 (no scale factors): two disjoint slots, [0, 256)
// and [256, 512); the epilogue drains its slot chunk by chunk and releases it
// for the tile after next, so the MMAs never wait for it.
#include <cuda.h>

#include "sq_device.cuh"
#include "sq_kernels.h"
#include "sq_ptx.cuh"

namespace sq {

constexpr int BM = 256;                        // cluster tile: two CTAs x 128 rows
constexpr int BN = 256;
constexpr int kRowsPerCta = 128;
constexpr int kRowBytes = 128;                 // every stage holds 128-byte rows (one swizzle atom)
constexpr int kABytes = kRowsPerCta * kRowBytes;   // 16 KB: this CTA's 128 rows of A
constexpr int kBBytes = 128 * kRowBytes;           // 16 KB: this CTA's half (128 rows) of B
constexpr int kMmaPerStage = 4;                // K = 64 (fp4) or 16 (bf16) per MMA, 32 bytes of the row each
constexpr int kSfaBytes = kMmaPerStage * 512;  // one 512-byte chunk (128 rows x 4 scales) per MMA
constexpr int kSfbBytes = 2 * kSfaBytes;       // both 128-row halves of B (every CTA needs all 256)
constexpr int kEpiWarps = 4;
constexpr int kStagingBytes = 32 * 128;        // one warp's 32 rows x 32 fp32
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccSlot1 = 64;             // NVFP4: accumulator slots [0, 256) and [64, 320)
constexpr uint32_t kAccSlot1Full = 256;        // bf16 / int4 / int8: slots [0, 256) and [256, 512)
constexpr int kOverlapChunks = 6;              // 32-column chunks shared by the two slots
constexpr uint32_t kSfCol = 320;               // ring of four scale-factor buffers, one stage (4 MMAs) each
constexpr uint32_t kSfBufCols = 48;            // SFB for MMA k at +8k (256 rows), SFA at +32+4k (128 rows)
constexpr uint32_t kSfBufs = 4;

// instruction descriptors: M = 256 (the CTA pair), N = 256, K-major A and B
constexpr uint32_t kIdescBf16 = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                ((uint32_t)(BM >> 4) << 24);           // f32 accum, bf16 x bf16
constexpr uint32_t kIdescNvfp4 = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                 ((uint32_t)(BM >> 4) << 24);          // e2m1 x e2m1, ue4m3 scales

template <int MODE>
struct GemmCfg {
    static constexpr bool FP4 = MODE == kGemmNvfp4;
    static constexpr bool DQ = MODE == kGemmInt4G32 || MODE == kGemmInt4G64 || MODE == kGemmInt8;
    static constexpr int kStages = FP4 ? 5 : 6;
    static constexpr int kScaleWarps = FP4 ? 4 : 0;              // warps 6..9 fill the scale-factor buffers
    static constexpr int kDqWarps = DQ ? 4 : 0;                  // warps 6..9 fill the W ring
    static constexpr int kThreads = 32 * (6 + kScaleWarps + kDqWarps);
    static constexpr int kStageBytes = kABytes + kBBytes + (FP4 ? kSfaBytes + kSfbBytes : 0);
    static constexpr int kKPerStage = FP4 ? 256 : 64;            // K values per stage
    static constexpr int kStagingOff = kStages * kStageBytes;
    static constexpr int kBarOff = kStagingOff + kEpiWarps * 2 * kStagingBytes;
    // full[s], empty[s], sfdata[s], acc_full[2], acc_empty[2], drain
    static constexpr int kNumBars = 3 * kStages + 5;
    static constexpr int kSmemBytes = kBarOff + 8 * kNumBars + 16 + 1024;   // + holder, flag, verdict, alignment
};

struct GemmArgs {
    const uint8_t *sfa;      // NVFP4: tiled activation scales
    const uint8_t *sfb;      // NVFP4: tiled weight scales
    const float *g_x;        // NVFP4: activation global scale (device)
    const float *g_w;        // NVFP4: weight global scale (device)
    const uint8_t *bq;       // int4 / int8: weight codes ([N, K/2] or [N, K])
    const void *bscale;      // int4: fp16 group scales [N, K/G]; int8: fp32 row scales [N]
    uint16_t *wring;         // int4 / int8: W ring, [ring_slots * 256, K] bf16
    uint32_t *ring_ready;    // [ring_slots] shares written (2 per tile: both CTAs), zero at launch
    uint32_t *ring_done;     // [ring_slots] tiles whose B loads have all landed, zero at launch
    int ring_slots;
    uint32_t *status;        // device status word
    int M, N, K;
    int lora;                // 1: add the low-rank K-step
    int out_bf16;            // 1: y is bf16 (RNE of the fp32 result), else fp32
};

// warp-uniform bounded wait on a local barrier: lane 0 polls, the verdict is broadcast
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile uint32_t *abort_flag,
                                          uint32_t *status, int lane)
{
    int ok = 1;
    if (lane == 0)
        ok = mbar_wait(bar, parity, abort_flag, status) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

__device__ __forceinline__ bool warp_wait_cluster(uint32_t bar, uint32_t parity, volatile uint32_t *abort_flag,
                                                  uint32_t *status, int lane)
{
    int ok = 1;
    if (lane == 0)
        ok = mbar_wait_cluster(bar, parity, abort_flag, status) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// scale one 32-row x 32-column accumulator chunk into 128B-swizzled staging
// buffer sb of the warp (the caller made sure the buffer is free)
// one warp's 32 rows x 32 columns of y, scaled by beta, into staging buffer sb in the layout of
// the y tensor map: fp32 rows of 128 bytes with the 128-byte swizzle, or (ybf) bf16 rows of 64
// bytes with the 64-byte swizzle (16-byte piece j of row r at j ^ ((r >> 1) & 3))
__device__ __forceinline__ void stage_chunk(const uint32_t (&r)[32], float beta, uint8_t *staging, int sb, int lane,
                                            bool ybf)
{
    uint8_t *buf = staging + sb * kStagingBytes;
    if (ybf) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t p[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                p[i] = f32x2_to_bf16x2_bits(__fmul_rn(__uint_as_float(r[8 * j + 2 * i]), beta),
                                            __fmul_rn(__uint_as_float(r[8 * j + 2 * i + 1]), beta));
            *reinterpret_cast<uint4 *>(buf + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) =
                make_uint4(p[0], p[1], p[2], p[3]);
        }
        return;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float4 o;
        o.x = __fmul_rn(__uint_as_float(r[4 * j + 0]), beta);
        o.y = __fmul_rn(__uint_as_float(r[4 * j + 1]), beta);
        o.z = __fmul_rn(__uint_as_float(r[4 * j + 2]), beta);
        o.w = __fmul_rn(__uint_as_float(r[4 * j + 3]), beta);
        *reinterpret_cast<float4 *>(buf + lane * 128 + ((j ^ (lane & 7)) << 4)) = o;
    }
}

// TMA-store staging buffer sb (written by the whole warp) to y at (x, y)
__device__ __forceinline__ void issue_store(uint8_t *staging, int sb, int lane, const CUtensorMap *tmY, int x, int y)
{
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d(tmY, smem_u32(staging + sb * kStagingBytes), x, y);
        bulk_commit_group();
    }
}

// stage + store a chunk through buffer sb, once at most one earlier store is pending
__device__ __forceinline__ void store_chunk(const uint32_t (&r)[32], float beta, uint8_t *staging, int sb, int lane,
                                            const CUtensorMap *tmY, int x, int y, bool ybf)
{
    if (lane == 0)
        bulk_wait_group_read1();
    __syncwarp();
    stage_chunk(r, beta, staging, sb, lane, ybf);
    issue_store(staging, sb, lane, tmY, x, y);
}

// ---------------------------------------------------------------------------
// W ring (int4 / int8 paths).  Every one of the m_tiles clusters that multiply
// W tile nt (256 rows of W) writes 1/m_tiles of its rows as bf16(q s) into slot
// nt % R of a ring in global memory and counts its share in ring_ready[slot]
// (release); each of them waits for all 2 m_tiles shares (acquire) before its
// TMA loads of B from the slot, and counts the tile in ring_done[slot] once its
// MMAs are done (its epilogue starts), which frees the slot for tile nt + R.  So W is dequantised
// once per 256-row tile instead of once per (M tile, N tile), the GEMM's B
// operand moves by TMA as on the bf16 path, and the ring (R x 256 x K bf16,
// about 3 MB a slot at K = 6144) stays in L2 and in a workspace of fixed size.
// The values are those of the stand-alone dequantisation:
//   int4: bf16(q s), rounded once, formed in bf16x2 arithmetic from the split
//         s = s_hi + s_lo (dq_int4x8);
//   int8: q s is rounded to fp32 and then to bf16, as the int8 codec defines.
// (SquareQ README, "Residual codecs": the residual codecs are dequant-first.)
// Bit for bit the same for every finite scale.
// ---------------------------------------------------------------------------
// bf16x2 arithmetic, each lane rounded once (round to nearest even)
__device__ __forceinline__ uint32_t bf2_sub(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ uint32_t bf2_mul(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ uint32_t bf2_fma(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t r;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
    return r;
}

// eight int4 codes (value i in nibble i) times the scale s = s_hi + s_lo -> 8 bf16
// values, in bf16x2 arithmetic with no conversion instruction.  s_hi = bf16(s) and
// s_lo = s - s_hi are both exact in bf16 (an fp16 scale has 11 significant bits), q
// (the code byte placed under the exponent of 128, minus 136) is exact, q s_lo is
// exact (at most 7 bits), and one fma forms bf16(q s_hi + q s_lo) = bf16(q s) with a
// single rounding -- the stand-alone dequantisation's value, zero signs included.
__device__ __forceinline__ uint4 dq_int4x8(uint32_t w, uint32_t shi2, uint32_t slo2)
{
    const uint32_t x = w ^ 0x88888888u;                 // q + 8 in every nibble
    const uint32_t lo = x & 0x0F0F0F0Fu, hi = (x >> 4) & 0x0F0F0F0Fu;
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        // halves (value 2j, value 2j + 1) = bf16 128 + (q + 8): byte j of lo / hi under 0x43
        const uint32_t v = (__byte_perm(lo, hi, (4u + j) << 8 | (uint32_t)j) & 0x00FF00FFu) | 0x43004300u;
        const uint32_t q = bf2_sub(v, 0x43084308u);     // - 136: exact
        o[j] = bf2_fma(q, shi2, bf2_mul(q, slo2));
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// four int8 codes (value i in byte i) times the fp32 scale pair s2 -> 4 bf16 values (2 words)
__device__ __forceinline__ void dq_int8x4(uint32_t w, uint64_t s2, uint32_t &o0, uint32_t &o1)
{
    const uint32_t x = w ^ 0x80808080u;                 // q + 128 in every byte, under 2^23
    const uint64_t off = f2_pack(8388736.0f, 8388736.0f);
    const uint64_t a01 = f2_pack(__uint_as_float(__byte_perm(x, 0x4B000000u, 0x7650u)),
                                 __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7651u)));
    const uint64_t a23 = f2_pack(__uint_as_float(__byte_perm(x, 0x4B000000u, 0x7652u)),
                                 __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7653u)));
    float p0, p1, p2, p3;
    f2_unpack(f2_mul(f2_sub(a01, off), s2), p0, p1);
    f2_unpack(f2_mul(f2_sub(a23, off), s2), p2, p3);
    o0 = f32x2_to_bf16x2_bits(p0, p1);
    o1 = f32x2_to_bf16x2_bits(p2, p3);
}

// the payload of the 32 values 32 kc .. 32 kc + 31 of row n of W (one group-32 scale,
// one 16-byte load for int4; two for int8), and bf16(q s) of them (64 bytes)
struct DqRaw {
    uint4 c0, c1;            // int4: 32 codes in c0; int8: 32 codes in c0, c1
    uint32_t s;              // int4: fp16 scale bits; int8: fp32 scale bits
};

template <int MODE>
__device__ __forceinline__ DqRaw dq_load(const GemmArgs &a, int n, int kc)
{
    DqRaw d;
    if (MODE == kGemmInt8) {
        const uint4 *p = reinterpret_cast<const uint4 *>(a.bq + (int64_t)n * a.K) + 2 * kc;
        d.c0 = __ldg(p);
        d.c1 = __ldg(p + 1);
        d.s = __ldg(reinterpret_cast<const uint32_t *>(a.bscale) + n);
    } else {
        constexpr int gs = MODE == kGemmInt4G32 ? 32 : 64;
        d.c0 = __ldg(reinterpret_cast<const uint4 *>(a.bq + (int64_t)n * (a.K / 2)) + kc);
        d.c1 = make_uint4(0u, 0u, 0u, 0u);
        d.s = __ldg(reinterpret_cast<const uint16_t *>(a.bscale) + (int64_t)n * (a.K / gs) + (32 * kc) / gs);
    }
    return d;
}

template <int MODE>
__device__ __forceinline__ void dq_convert_store(const DqRaw &d, uint4 *dst)
{
    if (MODE == kGemmInt8) {
        const float sf = __uint_as_float(d.s);
        const uint64_t s2 = f2_pack(sf, sf);
        const uint32_t w[8] = {d.c0.x, d.c0.y, d.c0.z, d.c0.w, d.c1.x, d.c1.y, d.c1.z, d.c1.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint4 o;
            dq_int8x4(w[2 * j], s2, o.x, o.y);
            dq_int8x4(w[2 * j + 1], s2, o.z, o.w);
            dst[j] = o;
        }
        return;
    }
    const float sf = __half2float(__ushort_as_half((uint16_t)d.s));
    const uint32_t shi = __bfloat16_as_ushort(__float2bfloat16_rn(sf));
    const uint32_t slo = __bfloat16_as_ushort(__float2bfloat16_rn(__fsub_rn(sf, __uint_as_float(shi << 16))));
    const uint32_t shi2 = shi | (shi << 16), slo2 = slo | (slo << 16);
    const uint32_t w[4] = {d.c0.x, d.c0.y, d.c0.z, d.c0.w};
#pragma unroll
    for (int j = 0; j < 4; ++j)
        dst[j] = dq_int4x8(w[j], shi2, slo2);
}

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GemmCfg<MODE>::kThreads, 1)
    sq_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmT, const __grid_constant__ CUtensorMap tmU,
                   const __grid_constant__ CUtensorMap tmY, const GemmArgs args)
{
    using Cfg = GemmCfg<MODE>;
    constexpr bool FP4 = Cfg::FP4;
    constexpr bool DQ = Cfg::DQ;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kBarOff);
    const uint32_t bar_full = smem_u32(bars);                          // leader: both CTAs' stage ready
    const uint32_t bar_empty = bar_full + 8 * Cfg::kStages;            // each CTA: its stage may be refilled
    const uint32_t bar_sfdata = bar_empty + 8 * Cfg::kStages;          // each CTA: its scale tiles landed
    const uint32_t bar_acc_full = bar_sfdata + 8 * Cfg::kStages;       // each CTA: accumulator ready
    // leader: (NVFP4) the overlap drained in both CTAs / (else) slot s drained in both CTAs
    const uint32_t bar_acc_empty = bar_acc_full + 16;
    const uint32_t bar_drain = bar_acc_empty + 16;                     // leader: every MMA finished
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + Cfg::kNumBars);
    volatile uint32_t *abort_flag = tmem_holder + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();      // 0 = leader (issues the pair's MMAs)
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        for (int st = 0; st < Cfg::kStages; ++st) {
            // leader's expect_tx (both CTAs' bytes) + every scale or dequantising warp of both CTAs
            mbar_init(bar_full + 8 * st, 1 + 2 * Cfg::kScaleWarps);
            mbar_init(bar_empty + 8 * st, 1 + Cfg::kScaleWarps);        // MMA commit + scale warps
            mbar_init(bar_sfdata + 8 * st, 1);
        }
        mbar_init(bar_acc_full, 1);
        mbar_init(bar_acc_full + 8, 1);
        mbar_init(bar_acc_empty, 2 * kEpiWarps);
        mbar_init(bar_acc_empty + 8, 2 * kEpiWarps);
        mbar_init(bar_drain, 1);
        *abort_flag = 0u;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc2(smem_u32(tmem_holder), kTmemCols);
        tmem_relinquish2();
    }
    if (warp == 4 && lane == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        prefetch_tmap(&tmT);
        prefetch_tmap(&tmU);
        prefetch_tmap(&tmY);
    }
    tc_fence_before();
    cluster_sync();                               // barriers of both CTAs initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    // operands written by the preceding kernels are visible after this; the W ring
    // writers read only the weight payload and start at once
    if (!(DQ && warp >= 6))
        grid_dep_wait();

    const int m_tiles = (args.M + BM - 1) / BM;
    const int n_tiles = (args.N + BN - 1) / BN;
    const int tiles = m_tiles * n_tiles;
    const int cluster_id = blockIdx.x >> 1;
    const int clusters = gridDim.x >> 1;
    const int k_stages = args.K / Cfg::kKPerStage;
    const int lora_stages = args.lora ? 1 : 0;                // [t_hi | t_lo] x [U | U]
    const int stages_per_tile = k_stages + lora_stages;
    const int sf_chunks_per_row_tile = args.K / 64;          // 512-byte chunks per 128-row tile
    const int m_rows_pad = (args.M + 127) / 128 * 128;

    if (warp == 4) {
        // ------------------------------------------------------------ producer (both CTAs)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            bool next_ready = false;                                      // (int4 / int8) probed early
            for (int tile = cluster_id; tile < tiles && ok; tile += clusters) {
                const int mt = tile % m_tiles, nt = tile / m_tiles;
                const int m0 = mt * BM + (int)rank * kRowsPerCta;         // this CTA's rows of A / y
                const int nh = nt * BN + (int)rank * 128;                 // this CTA's half of B
                const bool sfa_ok = m0 < m_rows_pad;
                const bool sfb_hi = (nt * BN + 128) < args.N;
                // int4 / int8: this CTA's half of W tile nt sits in ring slot nt % R once all
                // 2 * m_tiles shares of this use of the slot are written
                const int ring_row = DQ ? (nt % args.ring_slots) * BN + (int)rank * 128 : 0;
                if (DQ) {
                    const uint32_t need = (uint32_t)(nt / args.ring_slots + 1) * (uint32_t)m_tiles * 2u;
                    if (!next_ready &&
                        !gwait_geq(args.ring_ready + nt % args.ring_slots, need, abort_flag, args.status)) {
                        ok = false;
                        break;
                    }
                    next_ready = false;
                    fence_proxy_async_global();                // the TMA reads below see those stores
                }
                for (int ks = 0; ks < stages_per_tile; ++ks) {
                    if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1u, abort_flag, args.status)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sbase = smem + stage * Cfg::kStageBytes;
                    const uint32_t fb = bar_full + 8 * stage;            // counted on the leader's copy
                    const uint32_t sA = smem_u32(sbase), sB = smem_u32(sbase + kABytes);
                    const uint32_t sd = bar_sfdata + 8 * stage;
                    if (leader)
                        mbar_arrive_expect_tx(fb, 2 * (kABytes + kBBytes));
                    if (ks < lora_stages) {
                        tma_load_2d_pair(sA, &tmT, 0, m0, fb);
                        tma_load_2d_pair(sB, &tmU, 0, nh, fb);
                        if (FP4)
                            mbar_arrive(sd);                              // keeps the scale warps in step
                    } else {
                        const int kk = ks - lora_stages;
                        if (FP4) {
                            tma_load_2d_pair(sA, &tmA, kk * kRowBytes, m0, fb);
                            tma_load_2d_pair(sB, &tmB, kk * kRowBytes, nh, fb);
                            const uint32_t sSfa = smem_u32(sbase + kABytes + kBBytes);
                            const uint32_t sSfb = sSfa + kSfaBytes;
                            const int64_t chunk = (int64_t)kk * kMmaPerStage;
                            const uint32_t sf_bytes = (sfa_ok ? kSfaBytes : 0) + (sfb_hi ? kSfbBytes : kSfaBytes);
                            mbar_arrive_expect_tx(sd, sf_bytes);
                            if (sfa_ok)
                                bulk_load(sSfa,
                                          args.sfa + ((int64_t)(m0 / 128) * sf_chunks_per_row_tile + chunk) * 512,
                                          kSfaBytes, sd);
                            bulk_load(sSfb, args.sfb + ((int64_t)(2 * nt) * sf_chunks_per_row_tile + chunk) * 512,
                                      kSfaBytes, sd);
                            if (sfb_hi)
                                bulk_load(sSfb + kSfaBytes,
                                          args.sfb + ((int64_t)(2 * nt + 1) * sf_chunks_per_row_tile + chunk) * 512,
                                          kSfaBytes, sd);
                        } else {
                            tma_load_2d_pair(sA, &tmA, kk * 64, m0, fb);
                            tma_load_2d_pair(sB, &tmB, kk * 64, DQ ? ring_row : nh, fb);
                        }
                    }
                    if (DQ && ks == stages_per_tile / 2) {     // one acquire probe for the next tile,
                        const int nn = (tile + clusters) / m_tiles;   // so its start rarely waits
                        next_ready = tile + clusters < tiles &&
                                     ld_acquire_gpu(args.ring_ready + nn % args.ring_slots) >=
                                         (uint32_t)(nn / args.ring_slots + 1) * (uint32_t)m_tiles * 2u;
                    }
                    if (++stage == Cfg::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // let every load that was issued land (and be consumed) before the CTA exits
            for (int st = 0; st < Cfg::kStages; ++st) {
                (void)mbar_wait(bar_empty + 8 * stage, phase ^ 1u, abort_flag, args.status);
                if (++stage == Cfg::kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer (leader)
        // One thread issues every MMA of the pair, so its per-stage work is kept to a
        // few adds: shared-memory descriptors are built once and advanced by the
        // stage offset (the start-address field holds address / 16).
        if (leader && lane == 0) {
            const uint32_t s0 = smem_u32(smem);
            const uint64_t dA0 = sdesc_sw128(s0);                      // stage 0, A, k = 0
            const uint64_t dB0 = sdesc_sw128(s0 + kABytes);
            constexpr uint32_t kStage16 = Cfg::kStageBytes >> 4;
            int stage = 0;
            uint32_t off16 = 0;
            uint32_t phase = 0;
            int count = 0;
            uint32_t sfbuf = 0;
            uint32_t sf = tmem_base + kSfCol;
            bool ok = true;
            for (int tile = cluster_id; tile < tiles && ok; tile += clusters, ++count) {
                const uint32_t acc = tmem_base + ((count & 1) ? (FP4 ? kAccSlot1 : kAccSlot1Full) : 0u);
                if (FP4) {        // the overlap of the previous tile's slot has been drained
                    if (count > 0 &&
                        !mbar_wait_cluster(bar_acc_empty, (uint32_t)((count - 1) & 1), abort_flag, args.status))
                        break;
                } else {          // tile count - 2 (same slot) has left tensor memory
                    if (count >= 2 && !mbar_wait_cluster(bar_acc_empty + 8 * (count & 1),
                                                         (uint32_t)(((count >> 1) - 1) & 1), abort_flag, args.status))
                        break;
                }
                for (int ks = 0; ks < stages_per_tile; ++ks) {
                    if (!mbar_wait_cluster(bar_full + 8 * stage, phase, abort_flag, args.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t a = dA0 + off16, b = dB0 + off16;
                    if (ks < lora_stages) {
#pragma unroll
                        for (int k = 0; k < kMmaPerStage; ++k)
                            mma2_bf16(acc, a + 2 * k, b + 2 * k, kIdescBf16, k > 0 ? 1u : 0u);
                    } else if (FP4) {
                        // the scale factors of stage g sit in tensor-memory buffer g % 3 of both
                        // CTAs; full[] above already counted the scale warps that stored them
#pragma unroll
                        for (int k = 0; k < kMmaPerStage; ++k)
                            mma2_nvfp4(acc, a + 2 * k, b + 2 * k, kIdescNvfp4, sf + 32 + 4 * k, sf + 8 * k,
                                       (ks > 0 || k > 0) ? 1u : 0u);
                    } else {
#pragma unroll
                        for (int k = 0; k < kMmaPerStage; ++k)
                            mma2_bf16(acc, a + 2 * k, b + 2 * k, kIdescBf16, (ks > 0 || k > 0) ? 1u : 0u);
                    }
                    tc_commit2_both(bar_empty + 8 * stage);
                    if (++stage == Cfg::kStages) {
                        stage = 0;
                        off16 = 0;
                        phase ^= 1u;
                    } else {
                        off16 += kStage16;
                    }
                    if (++sfbuf == kSfBufs) {             // scale buffer of the next stage
                        sfbuf = 0;
                        sf = tmem_base + kSfCol;
                    } else {
                        sf += kSfBufCols;
                    }
                }
                if (ok)
                    tc_commit2_both(bar_acc_full + 8 * (count & 1));
            }
            // all issued MMAs must finish before tensor memory is released
            tc_commit2_local(bar_drain);
            (void)mbar_wait(bar_drain, 0, abort_flag, args.status);
        }
        __syncwarp();
    } else if (DQ && warp >= 6) {
        // ------------------------------------------------------------ W ring writers (int4 / int8, both CTAs)
        // For each tile (mt, nt) of the cluster, in order: the cluster writes share mt
        // of the m_tiles shares (rows 256 mt / m_tiles ..) of W tile nt into ring slot
        // nt % R, this CTA one half of it, once the slot's previous tile (nt - R) has
        // been loaded by all of its m_tiles clusters.  The writers run ahead of the
        // cluster's own MMAs; every wait points at an earlier W tile, so the chain ends.
        // Only thread 0 waits (bounded) and every writer thread then meets it at named
        // barrier 1, so the four warps always take the same way out.
        constexpr int kBatch = 4;                                   // 32-value chunks in flight per thread
        const int tid = threadIdx.x - 6 * 32;                      // 0..127
        const int R = args.ring_slots;
        const int kc32 = args.K / 32;                               // 32-value chunks per row
        volatile uint32_t *verdict = tmem_holder + 2;
        for (int tile = cluster_id; tile < tiles; tile += clusters) {
            const int mt = tile % m_tiles, nt = tile / m_tiles;
            const int slot = nt % R;
            const int lo = (BN * mt) / m_tiles, hi = (BN * (mt + 1)) / m_tiles;
            const int mid = lo + (hi - lo) / 2;
            const int r0 = rank ? mid : lo, r1 = rank ? hi : mid;
            if (tid == 0)
                *verdict = gwait_geq(args.ring_done + slot, (uint32_t)(nt / R) * (uint32_t)m_tiles, abort_flag,
                                     args.status)
                               ? 1u
                               : 0u;
            named_barrier_sync(1, 128);
            if (*verdict == 0u)
                break;
            const int total = (r1 - r0) * kc32;
            for (int c0 = tid; c0 < total; c0 += kBatch * 128) {
                DqRaw raw[kBatch];
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    const int c = c0 + 128 * u;
                    const int rr = r0 + c / kc32, n = nt * BN + rr;
                    if (c < total && n < args.N)
                        raw[u] = dq_load<MODE>(args, n, c - (rr - r0) * kc32);
                }
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    const int c = c0 + 128 * u;
                    const int rr = r0 + c / kc32, n = nt * BN + rr;
                    if (c < total) {
                        uint4 *dst = reinterpret_cast<uint4 *>(args.wring + ((int64_t)slot * BN + rr) * args.K) +
                                     4 * (c - (rr - r0) * kc32);
                        if (n < args.N) {
                            dq_convert_store<MODE>(raw[u], dst);
                        } else {
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                dst[j] = make_uint4(0u, 0u, 0u, 0u);
                        }
                    }
                }
            }
            fence_proxy_async_global();                             // for the TMA loads of other SMs
            named_barrier_sync(1, 128);                             // the four writer warps are done
            if (tid == 0)
                red_release_gpu_add(args.ring_ready + slot, 1u);
        }
    } else if (FP4 && warp >= 6) {
        // ------------------------------------------------------------ scale warps (NVFP4, both CTAs)
        // Warp w owns tensor-memory lanes 32*(w%4)..+31 of its CTA.  For stage g it
        // copies line `lane` of the four SFA chunks (this CTA's rows 32*j + lane) into 4
        // columns per MMA and line `lane` of the eight SFB chunks (rows 128*h + 32*j +
        // lane) into 8 columns per MMA -- the layout tcgen05.cp .32x128b.warpx4 would
        // produce -- in buffer g % 3, with one store round, and then arrives on the
        // leader's full[] barrier of the stage.  Buffer g % 3 is free once the MMAs of
        // stage g - 3 are done, i.e. once that stage's empty[] barrier completed.
        const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
        const uint32_t full_leader = mapa_shared(bar_full, 0);
        int stage = 0;
        uint32_t phase = 0;
        int lstage = 0;                 // ring position and phase of stage g - 3
        uint32_t lphase = 0;
        uint32_t sfbuf = 0;
        int g = 0;
        bool ok = true;
        for (int tile = cluster_id; tile < tiles && ok; tile += clusters) {
            for (int ks = 0; ks < stages_per_tile && ok; ++ks, ++g) {
                if (!warp_wait(bar_sfdata + 8 * stage, phase, abort_flag, args.status, lane)) {
                    ok = false;
                    break;
                }
                uint4 sfa[kMmaPerStage], sfb0[kMmaPerStage], sfb1[kMmaPerStage];
                const bool scaled = ks >= lora_stages;
                if (scaled) {
                    const uint8_t *sSfa = smem + stage * Cfg::kStageBytes + kABytes + kBBytes;
                    const uint8_t *sSfb = sSfa + kSfaBytes;
#pragma unroll
                    for (int k = 0; k < kMmaPerStage; ++k) {
                        sfa[k] = *reinterpret_cast<const uint4 *>(sSfa + 512 * k + 16 * lane);
                        sfb0[k] = *reinterpret_cast<const uint4 *>(sSfb + 512 * k + 16 * lane);
                        sfb1[k] = *reinterpret_cast<const uint4 *>(sSfb + kSfaBytes + 512 * k + 16 * lane);
                    }
                }
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(bar_empty + 8 * stage);
                if (g >= (int)kSfBufs) {
                    if (scaled && !warp_wait(bar_empty + 8 * lstage, lphase, abort_flag, args.status, lane)) {
                        ok = false;
                        break;
                    }
                    if (++lstage == Cfg::kStages) {
                        lstage = 0;
                        lphase ^= 1u;
                    }
                }
                if (scaled) {
                    tc_fence_after();
                    const uint32_t sf = tmem_base + lane_base + kSfCol + kSfBufCols * sfbuf;
#pragma unroll
                    for (int k = 0; k < kMmaPerStage; ++k) {
                        const uint32_t a4[4] = {sfa[k].x, sfa[k].y, sfa[k].z, sfa[k].w};
                        const uint32_t b8[8] = {sfb0[k].x, sfb0[k].y, sfb0[k].z, sfb0[k].w,
                                                sfb1[k].x, sfb1[k].y, sfb1[k].z, sfb1[k].w};
                        tmem_st_8cols(sf + 8 * k, b8);
                        tmem_st_4cols(sf + 32 + 4 * k, a4);
                    }
                    tmem_wait_st();
                    tc_fence_before();
                }
                __syncwarp();
                if (lane == 0)
                    mbar_arrive_cluster(full_leader + 8 * stage);
                if (++sfbuf == kSfBufs)
                    sfbuf = 0;
                if (++stage == Cfg::kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        float beta = 1.0f;
        if (FP4) {
            const float b = __fmul_rn(*args.g_x, *args.g_w);
            beta = b == 0.0f ? 1.0f : b;
        }
        const uint32_t acc_empty_leader = mapa_shared(bar_acc_empty, 0);
        const bool ybf = args.out_bf16 != 0;
        uint8_t *staging = smem + Cfg::kStagingOff + warp * 2 * kStagingBytes;
        int count = 0;
        if constexpr (!FP4) {
            // Disjoint slots: the MMAs of the next tile run in the other slot, so this
            // one drains at leisure, chunk by chunk (the load of chunk q + 1 overlaps
            // the staging and store of chunk q), and is released once all of it has
            // left tensor memory -- in time for the tile after next.
            for (int tile = cluster_id; tile < tiles; tile += clusters, ++count) {
                const int mt = tile % m_tiles, nt = tile / m_tiles;
                const int m0 = mt * BM + (int)rank * kRowsPerCta;
                const int n0 = nt * BN;
                const int slot = count & 1;
                if (!warp_wait(bar_acc_full + 8 * slot, (uint32_t)((count >> 1) & 1), abort_flag, args.status,
                               lane))
                    break;
                if (DQ && leader && warp == 0 && lane == 0)   // the tile's MMAs are done with its W
                    red_release_gpu_add(args.ring_done + nt % args.ring_slots, 1u);
                tc_fence_after();
                const uint32_t acc = tmem_base + ((uint32_t)(32 * warp) << 16) + (slot ? kAccSlot1Full : 0u);
                const bool rows_live = m0 + 32 * warp < args.M;   // skip stores wholly below the matrix
                const int ytop = m0 + 32 * warp;
                uint32_t ra[32], rb[32];
                tmem_ld_32cols(acc, ra);
                tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 8; q += 2) {
                    tmem_ld_32cols(acc + 32 * (q + 1), rb);
                    if (rows_live)
                        store_chunk(ra, beta, staging, 0, lane, &tmY, n0 + 32 * q, ytop, ybf);
                    tmem_wait_ld();
                    if (q + 2 < 8)
                        tmem_ld_32cols(acc + 32 * (q + 2), ra);
                    if (rows_live)
                        store_chunk(rb, beta, staging, 1, lane, &tmY, n0 + 32 * (q + 1), ytop, ybf);
                    tmem_wait_ld();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive_cluster(acc_empty_leader + 8 * slot);
            }
        } else
        for (int tile = cluster_id; tile < tiles; tile += clusters, ++count) {
            const int mt = tile % m_tiles, nt = tile / m_tiles;
            const int m0 = mt * BM + (int)rank * kRowsPerCta;
            const int n0 = nt * BN;
            const int slot = count & 1;
            if (!warp_wait(bar_acc_full + 8 * slot, (uint32_t)((count >> 1) & 1), abort_flag, args.status, lane))
                break;
            tc_fence_after();
            const uint32_t acc = tmem_base + ((uint32_t)(32 * warp) << 16) + (slot ? kAccSlot1 : 0u);
            const bool rows_live = m0 + 32 * warp < args.M;       // skip stores wholly below the matrix
            // The six chunks this slot shares with the other one leave tensor memory
            // first: four into registers, two of those parked in the (now free)
            // staging buffers, then the last two; then the leader may start the next
            // tile.  Chunk q of the tile is column block (first + q) % 8.
            const int first = slot ? 0 : 8 - kOverlapChunks;   // slot 0 shares its last 6 chunks
            const int ytop = m0 + 32 * warp;
            if (lane == 0)
                bulk_wait_group_read0();                       // both staging buffers free
            __syncwarp();
            uint32_t r0[32], r1[32], r2[32], r3[32];
            tmem_ld_32cols(acc + 32 * ((first + 0) & 7), r0);
            tmem_ld_32cols(acc + 32 * ((first + 1) & 7), r1);
            tmem_ld_32cols(acc + 32 * ((first + 2) & 7), r2);
            tmem_ld_32cols(acc + 32 * ((first + 3) & 7), r3);
            tmem_wait_ld();
            stage_chunk(r0, beta, staging, 0, lane, ybf);
            stage_chunk(r1, beta, staging, 1, lane, ybf);
            tmem_ld_32cols(acc + 32 * ((first + 4) & 7), r0);
            tmem_ld_32cols(acc + 32 * ((first + 5) & 7), r1);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive_cluster(acc_empty_leader);
            if (rows_live) {
                issue_store(staging, 0, lane, &tmY, n0 + 32 * ((first + 0) & 7), ytop);
                issue_store(staging, 1, lane, &tmY, n0 + 32 * ((first + 1) & 7), ytop);
                store_chunk(r2, beta, staging, 0, lane, &tmY, n0 + 32 * ((first + 2) & 7), ytop, ybf);
                store_chunk(r3, beta, staging, 1, lane, &tmY, n0 + 32 * ((first + 3) & 7), ytop, ybf);
                store_chunk(r0, beta, staging, 0, lane, &tmY, n0 + 32 * ((first + 4) & 7), ytop, ybf);
                store_chunk(r1, beta, staging, 1, lane, &tmY, n0 + 32 * ((first + 5) & 7), ytop, ybf);
            }
            tmem_ld_32cols(acc + 32 * ((first + 6) & 7), r2);
            tmem_ld_32cols(acc + 32 * ((first + 7) & 7), r3);
            tmem_wait_ld();
            if (rows_live) {
                store_chunk(r2, beta, staging, 0, lane, &tmY, n0 + 32 * ((first + 6) & 7), ytop, ybf);
                store_chunk(r3, beta, staging, 1, lane, &tmY, n0 + 32 * ((first + 7) & 7), ytop, ybf);
            }
        }
        if (lane == 0)
            bulk_wait_group_all();
        __syncwarp();
    }

    tc_fence_before();
    cluster_sync();                               // no CTA leaves while its peer may still signal it
    tc_fence_after();
    if (warp == 5)
        tmem_dealloc2(tmem_base, kTmemCols);
}

// ---------------------------------------------------------------------------
// host side: tensor maps and launch
// ---------------------------------------------------------------------------
typedef CUresult (*PFN_encodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                    const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                    CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                    CUtensorMapFloatOOBfill);

static PFN_encodeTiled encode_fn()
{
    static PFN_encodeTiled fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_encodeTiled>(p);
    }
    return fn;
}

// 2D row-major tensor [rows, inner] of `esize`-byte elements, box [box_rows, box_inner]
bool make_tmap(CUtensorMap *m, CUtensorMapDataType dt, int esize, const void *base, uint64_t inner,
               uint64_t rows, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw)
{
    PFN_encodeTiled fn = encode_fn();
    if (!fn)
        return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * (uint64_t)esize};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// persistent grid: as many CTA pairs as can be resident at once (not every SM
// can pair up inside its GPC), each walking the tile list.  The shared-memory
// opt-in and the occupancy query run once per CUDA context and kernel (a new
// context loads the device code again, without the attribute).
template <int MODE>
static cudaError_t launch_mode(const CUtensorMap &tA, const CUtensorMap &tB, const CUtensorMap &tT,
                               const CUtensorMap &tU, const CUtensorMap &tY, const GemmArgs &a, int tiles, int sms,
                               cudaStream_t stream)
{
    using Cfg = GemmCfg<MODE>;
    constexpr int kMaxDev = 64;
    static unsigned long long ctx_seen[kMaxDev];
    static int resident_pairs[kMaxDev];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev)
        return cudaErrorInvalidDevice;
    const unsigned long long ctx = current_context_id();
    if (ctx == 0 || ctx_seen[dev] != ctx) {
        cudaError_t e =
            cudaFuncSetAttribute(sq_gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
        if (e != cudaSuccess)
            return e;
        cudaLaunchConfig_t q = {};
        q.gridDim = dim3(2 * (sms / 2));
        q.blockDim = dim3(Cfg::kThreads);
        q.dynamicSmemBytes = Cfg::kSmemBytes;
        int resident = 0;
        e = cudaOccupancyMaxActiveClusters(&resident, sq_gemm_kernel<MODE>, &q);
        (void)cudaGetLastError();
        resident_pairs[dev] = (e == cudaSuccess && resident > 0 && resident < sms / 2) ? resident : sms / 2;
        ctx_seen[dev] = ctx;
    }
    const int pairs = resident_pairs[dev];
    const int grid = 2 * (tiles < pairs ? tiles : pairs);        // clusters of two CTAs
    // dependent launch: the set-up (barriers, tensor memory, descriptor prefetch) overlaps
    // the end of the preceding kernel; the kernel waits for its results before loading
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(Cfg::kThreads);
    cfg.dynamicSmemBytes = Cfg::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, sq_gemm_kernel<MODE>, tA, tB, tT, tU, tY, a);
}

cudaError_t launch_gemm(const GemmLaunch &g, int sms, cudaStream_t stream)
{
    CUtensorMap tA, tB, tT, tU, tY;
    const bool fp4 = g.mode == kGemmNvfp4;
    const bool dq = g.mode == kGemmInt4G32 || g.mode == kGemmInt4G64 || g.mode == kGemmInt8;
    if (!fp4 && !dq && g.mode != kGemmBf16)
        return cudaErrorInvalidValue;
    bool ok = true;
    if (fp4) {
        ok &= make_tmap(&tA, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, g.a, (uint64_t)g.K / 2, (uint64_t)g.M, 128, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B);
        ok &= make_tmap(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, g.b, (uint64_t)g.K / 2, (uint64_t)g.N, 128, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B);
    } else {
        ok &= make_tmap(&tA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.a, (uint64_t)g.K, (uint64_t)g.M, 64, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B);
        // (int4 / int8: B comes from the W ring)
        if (dq && (!g.wring || !g.ring_ctr || g.ring_slots < 1))
            return cudaErrorInvalidValue;
        ok &= make_tmap(&tB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dq ? (const void *)g.wring : g.b, (uint64_t)g.K,
                        dq ? (uint64_t)g.ring_slots * BN : (uint64_t)g.N, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    }
    const bool lora = g.tsplit && g.udup;
    // without a low-rank step the maps below are never used; point them at A/B
    ok &= make_tmap(&tT, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, lora ? (const void *)g.tsplit : g.a, 64,
                    (uint64_t)g.M, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= make_tmap(&tU, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, lora ? (const void *)g.udup : g.a, 64,
                    lora ? (uint64_t)g.N : (uint64_t)g.M, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    if (g.out_bf16)
        ok &= make_tmap(&tY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.y, (uint64_t)g.N, (uint64_t)g.M, 32, 32,
                        CU_TENSOR_MAP_SWIZZLE_64B);
    else
        ok &= make_tmap(&tY, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, g.y, (uint64_t)g.N, (uint64_t)g.M, 32, 32,
                        CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok)
        return cudaErrorInvalidValue;
    GemmArgs a;
    a.sfa = g.sfa;
    a.sfb = g.sfb;
    a.g_x = g.g_x;
    a.g_w = g.g_w;
    a.bq = dq ? reinterpret_cast<const uint8_t *>(g.b) : nullptr;
    a.bscale = dq ? g.b_scales : nullptr;
    a.wring = dq ? g.wring : nullptr;
    a.ring_ready = dq ? g.ring_ctr : nullptr;
    a.ring_done = dq ? g.ring_ctr + g.ring_slots : nullptr;
    a.ring_slots = dq ? g.ring_slots : 1;
    a.status = g.status;
    a.M = (int)g.M;
    a.N = (int)g.N;
    a.K = (int)g.K;
    a.lora = lora ? 1 : 0;
    a.out_bf16 = g.out_bf16 ? 1 : 0;
    const int tiles = (int)(((g.M + BM - 1) / BM) * ((g.N + BN - 1) / BN));
    switch (g.mode) {
    case kGemmNvfp4:
        return launch_mode<kGemmNvfp4>(tA, tB, tT, tU, tY, a, tiles, sms, stream);
    case kGemmInt4G32:
        return launch_mode<kGemmInt4G32>(tA, tB, tT, tU, tY, a, tiles, sms, stream);
    case kGemmInt4G64:
        return launch_mode<kGemmInt4G64>(tA, tB, tT, tU, tY, a, tiles, sms, stream);
    case kGemmInt8:
        return launch_mode<kGemmInt8>(tA, tB, tT, tU, tY, a, tiles, sms, stream);
    default:
        return launch_mode<kGemmBf16>(tA, tB, tT, tU, tY, a, tiles, sms, stream);
    }
}

}  // namespace sq
