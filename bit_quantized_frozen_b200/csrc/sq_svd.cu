// sq_svd.cu -- SVD init of the rank-32 low-rank branch (SquareQ README, the
// "Low-rank branch" paragraph: a bf16 branch of rank 32 from the weight's SVD):
//
//   W [N, K] fp32  ->  lora_up   = bf16(U sqrt(sigma))  [N, 32]
//                      lora_down = bf16(V sqrt(sigma))  [K, 32]
//                      R = RN(W - L) [N, K],  L = the reconstruct's rank-32 fmaf chain
//
// The singular subspace comes from subspace iteration started at a caller-supplied
// block Omega [K, 32]:
//
//   V = orth(Omega);  repeat iters times { U = orth(W V);  Z = W^T U;  V = orth(Z) except the last time }
//
// With B = the last Z = W^T U, W ~ U B^T.  The Gram B^T B is factored R^T R (Cholesky) and a
// one-sided Jacobi iteration on the columns of R gives the rotation X with R X = Q S (Q orthogonal,
// S = the singular values of B), so that W ~ (U X) S (B X S^-1)^T and
// up = U X S^(1/2), down = B X S^(-1/2).  orth(A) is CholeskyQR: twice for the final U, once for
// the blocks in between.
//
// Work split: the products with W (the only steps that touch [N, K]) and the Grams of the [rows, 32]
// blocks are grids over all SMs; the 32 x 32 steps (Cholesky, triangular inverse, Jacobi) run in
// one warp with fp64 values in registers -- lane c holds column c -- and warp shuffles.  Every sum
// over rows or splits is taken in a fixed order, so the result depends only on the shape and Omega.
#include <cuda_runtime.h>

#include <cstdint>

#include "sq_device.cuh"
#include "sq_kernels.h"

namespace sq {

constexpr int kSvdRank = 32;
constexpr int kSvdTile = 128;          // rows of W (W V) or columns of W (W^T U) per CTA
constexpr int kSvdChunk = 32;          // depth of one shared-memory stage of the products
constexpr int kGramRows = 512;         // rows per partial Gram (the last one may be shorter)
constexpr int kGramSub = 128;          // rows per shared-memory sub-tile of a partial Gram
constexpr int kJacobiMaxSweeps = 30;
constexpr double kJacobiSkip = 1e-15;  // pairs whose cosine is below this are left alone
constexpr double kJacobiTol = 1e-13;   // a sweep whose largest cosine is below this ends the iteration
constexpr unsigned kFull = 0xffffffffu;
constexpr int kSvdTargetCtas = 1024;   // product grids are split until they reach this many CTAs
constexpr int kSvdMaxSplits = 16;

// two fp32 values as one 64-bit operand of the packed f32x2 instructions, and back
__device__ __forceinline__ uint64_t svd_pack2(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void svd_unpack2(uint64_t v, float &lo, float &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

// acc[j][p] += w[j] * (v[2p], v[2p+1]) for 4 rows j and 4 output pairs p: 16 fma.rn.f32x2, each two
// independent fmaf roundings
__device__ __forceinline__ void svd_fma_4x8(uint64_t (&acc)[4][4], const float (&w)[4], const float4 va,
                                           const float4 vb)
{
    const uint64_t v2[4] = {svd_pack2(va.x, va.y), svd_pack2(va.z, va.w), svd_pack2(vb.x, vb.y),
                            svd_pack2(vb.z, vb.w)};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint64_t w2 = svd_pack2(w[j], w[j]);
#pragma unroll
        for (int p = 0; p < 4; ++p)
            asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc[j][p]) : "l"(w2), "l"(v2[p]));
    }
}

// ---------------------------------------------------------------------------
// Yp[s, n, :] = sum over k in split s of W[n, k] V[k, :], for the 128 rows n of the CTA.
// Grid (N / 128, S), 128 threads.  Warp w owns outputs 8w..8w+7; lane l rows l, l+32, l+64, l+96.
// A stage holds 128 rows x 32 columns of W (row pitch 33 words: the 32 lanes' rows fall in 32
// different banks) and the matching 32 rows of V (read as 16-byte broadcasts).  The next stage is
// loaded into registers while the current one is multiplied.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kSvdTile) svd_wv_kernel(const float *__restrict__ W, int64_t N, int64_t K,
                                                          int64_t k_per_split, const float *__restrict__ V,
                                                          float *__restrict__ Yp)
{
    __shared__ float Ws[kSvdTile][kSvdChunk + 1];
    __shared__ __align__(16) float Vs[kSvdChunk][kSvdRank];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t n0 = (int64_t)blockIdx.x * kSvdTile;
    const int64_t kbeg = (int64_t)blockIdx.y * k_per_split, kend = kbeg + k_per_split;
    const float *wsrc = W + (n0 + warp) * K + lane;    // row warp + 4i, column lane of a stage
    float wr[kSvdTile / 4], vr[kSvdChunk * kSvdRank / kSvdTile];
    auto load = [&](int64_t k0) {
#pragma unroll
        for (int i = 0; i < kSvdTile / 4; ++i)
            wr[i] = wsrc[(int64_t)(4 * i) * K + k0];
#pragma unroll
        for (int i = 0; i < kSvdChunk * kSvdRank / kSvdTile; ++i)
            vr[i] = V[k0 * kSvdRank + tid + kSvdTile * i];
    };
    uint64_t acc[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int p = 0; p < 4; ++p)
            acc[j][p] = 0ull;
    load(kbeg);
    for (int64_t k0 = kbeg; k0 < kend; k0 += kSvdChunk) {
        __syncthreads();                               // the previous stage's reads are done
#pragma unroll
        for (int i = 0; i < kSvdTile / 4; ++i)
            Ws[warp + 4 * i][lane] = wr[i];
#pragma unroll
        for (int i = 0; i < kSvdChunk * kSvdRank / kSvdTile; ++i)
            (&Vs[0][0])[tid + kSvdTile * i] = vr[i];
        __syncthreads();
        if (k0 + kSvdChunk < kend)
            load(k0 + kSvdChunk);
#pragma unroll 8
        for (int k = 0; k < kSvdChunk; ++k) {
            float w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                w[j] = Ws[lane + 32 * j][k];
            svd_fma_4x8(acc, w, *reinterpret_cast<const float4 *>(&Vs[k][8 * warp]),
                        *reinterpret_cast<const float4 *>(&Vs[k][8 * warp + 4]));
        }
    }
    float *out = Yp + (int64_t)blockIdx.y * N * kSvdRank;
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            float lo, hi;
            svd_unpack2(acc[j][p], lo, hi);
            out[(n0 + lane + 32 * j) * kSvdRank + 8 * warp + 2 * p] = lo;
            out[(n0 + lane + 32 * j) * kSvdRank + 8 * warp + 2 * p + 1] = hi;
        }
}

// ---------------------------------------------------------------------------
// Zp[s, k, :] = sum over rows n of split s of W[n, k] U[n, :], for the 128 columns k of the CTA.
// Grid (K / 128, S), 128 threads.  Warp w owns outputs 8w..8w+7; lane l columns l, l+32, l+64,
// l+96.  A stage holds 32 rows x 128 columns of W and the matching 32 rows of U; the next stage
// is loaded into registers while the current one is multiplied.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kSvdTile) svd_wtu_kernel(const float *__restrict__ W, int64_t K,
                                                           int64_t n_per_split, const float *__restrict__ U,
                                                           float *__restrict__ Zp)
{
    __shared__ float Ws[kSvdChunk][kSvdTile];
    __shared__ __align__(16) float Us[kSvdChunk][kSvdRank];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t k0 = (int64_t)blockIdx.x * kSvdTile;
    const int64_t nbeg = (int64_t)blockIdx.y * n_per_split, nend = nbeg + n_per_split;
    float wr[kSvdChunk], ur[kSvdChunk * kSvdRank / kSvdTile];
    auto load = [&](int64_t n0) {
#pragma unroll
        for (int r = 0; r < kSvdChunk; ++r)
            wr[r] = W[(n0 + r) * K + k0 + tid];
#pragma unroll
        for (int i = 0; i < kSvdChunk * kSvdRank / kSvdTile; ++i)
            ur[i] = U[n0 * kSvdRank + tid + kSvdTile * i];
    };
    uint64_t acc[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int p = 0; p < 4; ++p)
            acc[j][p] = 0ull;
    load(nbeg);
    for (int64_t n0 = nbeg; n0 < nend; n0 += kSvdChunk) {
        __syncthreads();
#pragma unroll
        for (int r = 0; r < kSvdChunk; ++r)
            Ws[r][tid] = wr[r];
#pragma unroll
        for (int i = 0; i < kSvdChunk * kSvdRank / kSvdTile; ++i)
            (&Us[0][0])[tid + kSvdTile * i] = ur[i];
        __syncthreads();
        if (n0 + kSvdChunk < nend)
            load(n0 + kSvdChunk);
#pragma unroll 8
        for (int r = 0; r < kSvdChunk; ++r) {
            float w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                w[j] = Ws[r][lane + 32 * j];
            svd_fma_4x8(acc, w, *reinterpret_cast<const float4 *>(&Us[r][8 * warp]),
                        *reinterpret_cast<const float4 *>(&Us[r][8 * warp + 4]));
        }
    }
    float *out = Zp + (int64_t)blockIdx.y * K * kSvdRank;
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            float lo, hi;
            svd_unpack2(acc[j][p], lo, hi);
            out[(k0 + lane + 32 * j) * kSvdRank + 8 * warp + 2 * p] = lo;
            out[(k0 + lane + 32 * j) * kSvdRank + 8 * warp + 2 * p + 1] = hi;
        }
}

// out[i] = P[0][i] + P[1][i] + ... + P[S-1][i] in that order, i < rows * 32
__global__ void __launch_bounds__(256) svd_sum_splits_kernel(const float *__restrict__ P, int splits, int64_t rows,
                                                             float *__restrict__ out)
{
    const int64_t total = rows * kSvdRank;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        float z = P[i];
        for (int s = 1; s < splits; ++s)
            z = __fadd_rn(z, P[(int64_t)s * total + i]);
        out[i] = z;
    }
}

// ---------------------------------------------------------------------------
// partial Grams of A [rows, 32] (rows a multiple of 128): Gp[c][i][j] = sum over rows
// 512c .. min(512c + 511, rows - 1) of a_i a_j in fp64 (each fp32 product is exact in fp64).
// Grid ceil(rows / 512), 256 threads.  Lane l of warp w owns the 4 x 4 block b = 8w + l % 8
// (entries 4 (b / 8) .. +3 by 4 (b % 8) .. +3) over the rows r with r % 4 == l / 8 of each
// 128-row shared-memory sub-tile, in order; the four row groups of a block sit in lanes l, l + 8,
// l + 16, l + 24 and are added by two xor shuffles, ((g0 + g1) + (g2 + g3)) -- a fixed order.
// Each lane converts 8 fp32 values per row for 16 products.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) svd_gram_kernel(const float *__restrict__ A, int64_t rows,
                                                       double *__restrict__ Gp)
{
    __shared__ __align__(16) float As[kGramSub * kSvdRank];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = 8 * warp + (lane & 7), g = lane >> 3;
    const int bi = 4 * (b >> 3), bj = 4 * (b & 7);
    const int64_t r0 = (int64_t)blockIdx.x * kGramRows;
    const int64_t r1 = r0 + kGramRows < rows ? r0 + kGramRows : rows;
    double acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
            acc[i][j] = 0.0;
    for (int64_t rs = r0; rs < r1; rs += kGramSub) {
        __syncthreads();                               // the previous sub-tile's reads are done
        const float4 *src = reinterpret_cast<const float4 *>(A + rs * kSvdRank);
#pragma unroll
        for (int e = 0; e < kGramSub * kSvdRank / 4 / 256; ++e)
            reinterpret_cast<float4 *>(As)[tid + 256 * e] = src[tid + 256 * e];
        __syncthreads();
#pragma unroll 4
        for (int r = g; r < kGramSub; r += 4) {
            const float4 x = *reinterpret_cast<const float4 *>(&As[r * kSvdRank + bi]);
            const float4 y = *reinterpret_cast<const float4 *>(&As[r * kSvdRank + bj]);
            const double xi[4] = {(double)x.x, (double)x.y, (double)x.z, (double)x.w};
            const double yj[4] = {(double)y.x, (double)y.y, (double)y.z, (double)y.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    acc[i][j] = fma(xi[i], yj[j], acc[i][j]);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            acc[i][j] += __shfl_xor_sync(kFull, acc[i][j], 8);
            acc[i][j] += __shfl_xor_sync(kFull, acc[i][j], 16);
        }
    if (g == 0) {
        double *out = Gp + (int64_t)blockIdx.x * (kSvdRank * kSvdRank);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j)
                out[(bi + i) * kSvdRank + bj + j] = acc[i][j];
    }
}

// ---------------------------------------------------------------------------
// One-warp 32 x 32 steps.  Lane c holds column c of a matrix in 32 fp64 registers; every
// register index is a compile-time constant (the loops are unrolled), values move between
// lanes by shuffles only.
// ---------------------------------------------------------------------------
// G = sum of the C partial Grams in order, by all 256 threads (entry e = t + 256 q, four chains
// per thread, the loads of four partials in flight), written over partial 0 (each entry is
// read and written by its own thread only).
__device__ __forceinline__ void svd_sum_grams(double *__restrict__ Gp, int C)
{
    const int t = threadIdx.x;
    double g[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
        g[q] = Gp[t + 256 * q];
    int c = 1;
    for (; c + 4 <= C; c += 4) {
        double v[4][4];
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
            for (int q = 0; q < 4; ++q)
                v[b][q] = Gp[(int64_t)(c + b) * (kSvdRank * kSvdRank) + t + 256 * q];
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
            for (int q = 0; q < 4; ++q)
                g[q] += v[b][q];
    }
    for (; c < C; ++c)
#pragma unroll
        for (int q = 0; q < 4; ++q)
            g[q] += Gp[(int64_t)c * (kSvdRank * kSvdRank) + t + 256 * q];
#pragma unroll
    for (int q = 0; q < 4; ++q)
        Gp[t + 256 * q] = g[q];
}

// Cholesky G = R^T R (R upper triangular), right-looking.  In: g = column `lane` of G (destroyed).
// Out: r = column `lane` of R (r[i] = R[i][lane], zero below the diagonal) and inv = 1 / R[lane][lane]
// (0 for a dead pivot); a pivot d gives R[j][j] = d rsqrt(d) and row j of R = G[j][.] rsqrt(d).  A
// pivot that is not positive (a rank-deficient block, e.g. a zero weight) is a bit of the returned
// mask; its row of R is zero except R[j][j] = dead_diag.
__device__ __forceinline__ uint32_t svd_chol_warp(double (&g)[kSvdRank], double (&r)[kSvdRank], double &inv,
                                                  int lane, double dead_diag)
{
    double diag0 = 0.0;                                // G[lane][lane] before any update
#pragma unroll
    for (int i = 0; i < kSvdRank; ++i)
        if (i == lane)
            diag0 = g[i];
    uint32_t dead = 0u;
#pragma unroll
    for (int j = 0; j < kSvdRank; ++j) {
        const double d = __shfl_sync(kFull, g[j], j);
        const double d0 = __shfl_sync(kFull, diag0, j);
        const bool dj = !(d > 1e-300 * (1.0 + d0));
        dead |= dj ? (1u << j) : 0u;
        const double ij = dj ? 0.0 : rsqrt(d);
        const double rjj = dj ? dead_diag : d * ij;
        double rjc = 0.0;
        if (lane == j) {
            rjc = rjj;
            inv = ij;
        } else if (lane > j && !dj) {
            rjc = g[j] * ij;
        }
        r[j] = rjc;
#pragma unroll
        for (int i = j + 1; i < kSvdRank; ++i) {       // G[i][lane] -= R[j][i] R[j][lane]
            const double rji = __shfl_sync(kFull, rjc, i);
            g[i] = fma(-rji, rjc, g[i]);
        }
    }
    return dead;
}

// Rinv = R^-1 (fp32, row-major 32 x 32): lane c solves R x = e_c by back substitution, dividing by
// the pivots through their reciprocals (inv of lane i); the rows of dead pivots are zero, so the
// matching columns of the orthonormalised block are zero.
__device__ __forceinline__ void svd_rinv_warp(const double (&r)[kSvdRank], double inv, uint32_t dead, int lane,
                                              float *__restrict__ Rinv)
{
    double x[kSvdRank];
#pragma unroll
    for (int i = kSvdRank - 1; i >= 0; --i) {
        double v = (i == lane) ? 1.0 : 0.0;
#pragma unroll
        for (int k = i + 1; k < kSvdRank; ++k)
            v = fma(-__shfl_sync(kFull, r[i], k), x[k], v);   // R[i][k] is lane k's r[i]
        const double ii = __shfl_sync(kFull, inv, i);
        x[i] = ((dead >> i) & 1u) ? 0.0 : v * ii;
    }
#pragma unroll
    for (int i = 0; i < kSvdRank; ++i)
        Rinv[i * kSvdRank + lane] = (float)x[i];
}

// One-sided Jacobi on the columns of R (lane c holds column c): rotations J accumulate in X until
// the columns of R X are orthogonal; their squared norms are the eigenvalues of R^T R.  Each sweep
// runs 31 rounds of 16 disjoint pairs (round-robin: lane 31 meets lane `round`, lane c != round
// meets (2 round - c) mod 31).  Both lanes of a pair form the same three dot products in the same
// order, so they take the same rotation: for a_pp, a_qq, a_pq the tangent
// t = sgn(z) / (|z| + sqrt(z^2 + 1)), z = (a_qq - a_pp) / (2 a_pq), c = 1 / sqrt(t^2 + 1), s = t c,
// and columns p < q become c p - s q and s p + c q.  Output: the eigenvalues in descending order
// (So) and the matching columns of X (Xo, row-major 32 x 32).
__device__ __forceinline__ void svd_jacobi_warp(double (&r)[kSvdRank], int lane, double *__restrict__ Xo,
                                                double *__restrict__ So)
{
    double v[kSvdRank];
#pragma unroll
    for (int i = 0; i < kSvdRank; ++i)
        v[i] = (i == lane) ? 1.0 : 0.0;
    for (int sweep = 0; sweep < kJacobiMaxSweeps; ++sweep) {
        double off = 0.0;
        for (int round = 0; round < kSvdRank - 1; ++round) {
            const int partner = lane == kSvdRank - 1 ? round
                                : lane == round     ? kSvdRank - 1
                                                    : (2 * round - lane + 2 * (kSvdRank - 1)) % (kSvdRank - 1);
            const bool lower = lane < partner;
            double a[2] = {0.0, 0.0}, b[2] = {0.0, 0.0}, g[2] = {0.0, 0.0};   // even / odd i
#pragma unroll
            for (int i = 0; i < kSvdRank; ++i) {
                const double p = __shfl_sync(kFull, r[i], partner);
                a[i & 1] = fma(r[i], r[i], a[i & 1]);
                b[i & 1] = fma(p, p, b[i & 1]);
                g[i & 1] = fma(r[i], p, g[i & 1]);
            }
            const double an = a[0] + a[1], bn = b[0] + b[1], gn = g[0] + g[1];
            const double app = lower ? an : bn, aqq = lower ? bn : an;
            const double prod = app * aqq, g2 = gn * gn;
            double c = 1.0, s = 0.0;
            if (g2 > kJacobiSkip * kJacobiSkip * prod) {   // cosine of the pair above kJacobiSkip
                off = fmax(off, g2 / prod);
                const double z = (aqq - app) / (2.0 * gn);
                const double t = (z >= 0.0 ? 1.0 : -1.0) / (fabs(z) + sqrt(fma(z, z, 1.0)));
                c = rsqrt(fma(t, t, 1.0));
                s = t * c;
            }
            const double sp = lower ? -s : s;          // own column c x + (-s or +s) partner
#pragma unroll
            for (int i = 0; i < kSvdRank; ++i) {
                const double p = __shfl_sync(kFull, r[i], partner);
                r[i] = fma(sp, p, c * r[i]);
            }
#pragma unroll
            for (int i = 0; i < kSvdRank; ++i) {
                const double p = __shfl_sync(kFull, v[i], partner);
                v[i] = fma(sp, p, c * v[i]);
            }
        }
#pragma unroll
        for (int x = 16; x >= 1; x >>= 1)
            off = fmax(off, __shfl_xor_sync(kFull, off, x));
        if (off <= kJacobiTol * kJacobiTol)            // off holds squared cosines
            break;
    }
    double s2 = 0.0;
#pragma unroll
    for (int i = 0; i < kSvdRank; ++i)
        s2 = fma(r[i], r[i], s2);
    int rank = 0;                                      // position in descending order (ties: lane order)
#pragma unroll
    for (int j = 0; j < kSvdRank; ++j) {
        const double o = __shfl_sync(kFull, s2, j);
        rank += (o > s2 || (o == s2 && j < lane)) ? 1 : 0;
    }
#pragma unroll
    for (int i = 0; i < kSvdRank; ++i)
        Xo[i * kSvdRank + rank] = v[i];
    So[rank] = s2;
}

// EIG = false: Rinv = (Cholesky factor of G)^-1.  EIG = true: eigen-decomposition of G.
// 256 threads sum the partial Grams; warp 0 then runs the 32 x 32 step, lane c on column c.
template <bool EIG>
__global__ void __launch_bounds__(256) svd_small_kernel(double *__restrict__ Gp, int C, float *__restrict__ Rinv,
                                                        double *__restrict__ Xo, double *__restrict__ So)
{
    svd_sum_grams(Gp, C);
    __syncthreads();                                   // G (over partial 0) is complete and visible
    if (threadIdx.x >= 32)
        return;
    const int lane = threadIdx.x;
    double g[kSvdRank], r[kSvdRank], inv = 0.0;
#pragma unroll
    for (int i = 0; i < kSvdRank; ++i)
        g[i] = Gp[i * kSvdRank + lane];
    const uint32_t dead = svd_chol_warp(g, r, inv, lane, EIG ? 0.0 : 1.0);
    if (EIG)
        svd_jacobi_warp(r, lane, Xo, So);
    else
        svd_rinv_warp(r, inv, dead, lane, Rinv);
}

// A[row, :] <- A[row, :] Rinv (Rinv upper triangular, fp32), one row per thread, 64 rows per CTA
__global__ void __launch_bounds__(64) svd_apply_kernel(float *__restrict__ A, int64_t rows,
                                                       const float *__restrict__ Rinv)
{
    __shared__ float Rs[kSvdRank][kSvdRank];
    for (int e = threadIdx.x; e < kSvdRank * kSvdRank; e += blockDim.x)
        (&Rs[0][0])[e] = Rinv[e];
    __syncthreads();
    const int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (row >= rows)
        return;
    float4 *a_row = reinterpret_cast<float4 *>(A + row * kSvdRank);
    float a[kSvdRank];
#pragma unroll
    for (int i = 0; i < kSvdRank / 4; ++i) {
        const float4 v = a_row[i];
        a[4 * i] = v.x; a[4 * i + 1] = v.y; a[4 * i + 2] = v.z; a[4 * i + 3] = v.w;
    }
    float o[kSvdRank];
#pragma unroll
    for (int j = 0; j < kSvdRank; ++j) {
        float acc = 0.0f;
#pragma unroll
        for (int i = 0; i <= j; ++i)
            acc = fmaf(a[i], Rs[i][j], acc);
        o[j] = acc;
    }
#pragma unroll
    for (int i = 0; i < kSvdRank / 4; ++i)
        a_row[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
}

// up[n, :] = bf16(U[n, :] X S^(1/4)) for rows n < N, then down[k, :] = bf16(B[k, :] X S^(-1/4))
// for the next K rows (S = eigenvalues of B^T B = sigma^2, so S^(1/4) = sigma^(1/2)); a zero
// sigma gives a zero column of down.  Only the first RO columns (the RO largest sigma) are
// written: up [N, RO], down [K, RO].  One row per thread.
template <int RO>
__global__ void __launch_bounds__(256) svd_factors_kernel(const float *__restrict__ U, const float *__restrict__ B,
                                                          int64_t N, int64_t K, const double *__restrict__ Xd,
                                                          const double *__restrict__ Sd, uint16_t *__restrict__ up,
                                                          uint16_t *__restrict__ down)
{
    __shared__ float X[kSvdRank][kSvdRank];
    __shared__ float sc_up[kSvdRank], sc_down[kSvdRank];
    for (int e = threadIdx.x; e < kSvdRank * kSvdRank; e += blockDim.x)
        X[e >> 5][e & 31] = (float)Xd[e];
    if (threadIdx.x < kSvdRank) {
        const double sig = sqrt(Sd[threadIdx.x]);
        const double h = sqrt(sig);
        sc_up[threadIdx.x] = (float)h;
        sc_down[threadIdx.x] = sig > 0.0 ? (float)(1.0 / h) : 0.0f;
    }
    __syncthreads();
    const int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (row >= N + K)
        return;
    const bool is_up = row < N;
    const float *src = is_up ? U + row * kSvdRank : B + (row - N) * kSvdRank;
    uint16_t *dst = is_up ? up + row * RO : down + (row - N) * RO;
    const float *sc = is_up ? sc_up : sc_down;
    float a[kSvdRank];
#pragma unroll
    for (int i = 0; i < kSvdRank; ++i)
        a[i] = src[i];
#pragma unroll
    for (int j = 0; j < RO; ++j) {
        float s = 0.0f;
#pragma unroll
        for (int i = 0; i < kSvdRank; ++i)
            s = fmaf(a[i], X[i][j], s);
        dst[j] = (uint16_t)f32_to_bf16_bits(s * sc[j]);
    }
}

// ---------------------------------------------------------------------------
// R[n, k] = RN(W[n, k] - L[n, k]), L = fmaf chain over r = 0..RO-1 of up[n, r] down[k, r] from 0
// (the reconstruct's chain; RO = 32, or 16 for the int8 mode).  Grid (K / 256, m): CTA (kb, j) owns columns 256 kb .. +255 and the
// 64-row tiles j, j + m, ... .  Thread t owns columns 256 kb + 2 (t % 128) and +1 (both chains
// advance in one fma.rn.f32x2: two independent fmaf roundings) of rows 32 (t / 128) .. +31 of each
// tile; lora_down of its two columns is staged once (coalesced, through shared memory) and stays
// in registers, the tile's lora_up rows are read as 16-byte shared-memory broadcasts.  R may alias
// W (each element is read before it is written, by the same thread).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void svd_bf16x8(const uint4 v, float (&f)[8])
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

constexpr int kResRows = 8;            // rows of W whose loads a residual thread keeps in flight

template <int RO>
__global__ void __launch_bounds__(256, 2) svd_residual_kernel(const float *W, int64_t N, int64_t K,
                                                           const uint16_t *__restrict__ up,
                                                           const uint16_t *__restrict__ down, float *R)
{
    constexpr int kPieces = RO / 8;                    // 16-byte pieces of a factor row
    __shared__ float ds[256][RO + 1];
    __shared__ __align__(16) float us[64 * RO];
    const int tid = threadIdx.x;
    const int cp = tid & 127, rbase = 32 * (tid >> 7);
    const int64_t k = (int64_t)blockIdx.x * 256 + 2 * cp;
    const uint4 *dsrc = reinterpret_cast<const uint4 *>(down + (int64_t)blockIdx.x * 256 * RO);
#pragma unroll
    for (int i = 0; i < kPieces; ++i) {                // 256 columns x RO bf16
        const int e = tid + 256 * i;
        float f[8];
        svd_bf16x8(dsrc[e], f);
#pragma unroll
        for (int q = 0; q < 8; ++q)
            ds[e / kPieces][8 * (e % kPieces) + q] = f[q];
    }
    __syncthreads();
    uint64_t d2[RO];
#pragma unroll
    for (int r = 0; r < RO; ++r)
        d2[r] = svd_pack2(ds[2 * cp][r], ds[2 * cp + 1][r]);
    const int64_t NT = N / 64;
    for (int64_t nt = blockIdx.y; nt < NT; nt += gridDim.y) {
        const int64_t n0 = nt * 64;
        __syncthreads();                               // the previous tile's reads of us are done
        if (tid < 64 * kPieces) {                      // 64 rows x RO bf16
            float f[8];
            svd_bf16x8(reinterpret_cast<const uint4 *>(up + n0 * RO)[tid], f);
            *reinterpret_cast<float4 *>(&us[8 * tid]) = make_float4(f[0], f[1], f[2], f[3]);
            *reinterpret_cast<float4 *>(&us[8 * tid + 4]) = make_float4(f[4], f[5], f[6], f[7]);
        }
        __syncthreads();
        for (int nb = rbase; nb < rbase + 32; nb += kResRows) {
            float2 w[kResRows];                        // the block's W values, all loads in flight
#pragma unroll
            for (int i = 0; i < kResRows; ++i)
                w[i] = *reinterpret_cast<const float2 *>(W + (n0 + nb + i) * K + k);
            uint64_t acc[kResRows];
#pragma unroll
            for (int i = 0; i < kResRows; ++i)
                acc[i] = 0ull;
#pragma unroll
            for (int r4 = 0; r4 < RO; r4 += 4) {
#pragma unroll
                for (int i = 0; i < kResRows; ++i) {
                    const float4 u = *reinterpret_cast<const float4 *>(&us[(nb + i) * RO + r4]);
                    const float uv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        asm("fma.rn.f32x2 %0, %1, %2, %0;"
                            : "+l"(acc[i]) : "l"(svd_pack2(uv[q], uv[q])), "l"(d2[r4 + q]));
                }
            }
#pragma unroll
            for (int i = 0; i < kResRows; ++i) {
                float L0, L1;
                svd_unpack2(acc[i], L0, L1);
                *reinterpret_cast<float2 *>(R + (n0 + nb + i) * K + k) =
                    make_float2(__fsub_rn(w[i].x, L0), __fsub_rn(w[i].y, L1));
            }
        }
    }
}

// ---------------------------------------------------------------------------
// host orchestration
// ---------------------------------------------------------------------------
static size_t up256(size_t v)
{
    return (v + 255) / 256 * 256;
}

static int64_t max64(int64_t a, int64_t b)
{
    return a > b ? a : b;
}

// splits s in {1, 2, 4, 8, 16} of the reduction dimension `depth` (each part a multiple of 32
// deep) until the grid of `tiles` x s CTAs reaches the target
static int svd_splits(int64_t tiles, int64_t depth)
{
    int s = 1;
    while (s < kSvdMaxSplits && tiles * s < kSvdTargetCtas && depth % (kSvdChunk * 2 * s) == 0)
        s *= 2;
    return s;
}

// rows of the split partials: the larger of the two products' splits x rows
static int64_t svd_partial_rows(int64_t N, int64_t K)
{
    return max64(svd_splits(N / kSvdTile, K) * N, svd_splits(K / kSvdTile, N) * K);
}

size_t svd_workspace_bytes(int64_t N, int64_t K)
{
    const int64_t rows = max64(N, K);
    return up256((size_t)N * kSvdRank * 4) + up256((size_t)K * kSvdRank * 4) +
           up256((size_t)svd_partial_rows(N, K) * kSvdRank * 4) +
           up256((size_t)((rows + kGramRows - 1) / kGramRows) * kSvdRank * kSvdRank * 8) +
           up256(kSvdRank * kSvdRank * 4) + up256(kSvdRank * kSvdRank * 8) + up256(kSvdRank * 8);
}

struct SvdWs {
    float *Y, *V, *P, *Rinv;
    double *Gp, *X, *S;
};

#define SVD_STEP(name)                                   \
    do {                                                 \
        cudaError_t e_ = cudaPeekAtLastError();          \
        if (e_ != cudaSuccess) {                         \
            *stage = name;                               \
            return e_;                                   \
        }                                                \
    } while (0)

// orth(A): CholeskyQR, `passes` times (two for the final U, which must be orthonormal to fp32
// accuracy; one for the blocks in between, which only carry the subspace to the next product)
static cudaError_t svd_orth(float *A, int64_t rows, int passes, const SvdWs &w, cudaStream_t s, const char **stage)
{
    const int C = (int)((rows + kGramRows - 1) / kGramRows);
    for (int pass = 0; pass < passes; ++pass) {
        svd_gram_kernel<<<(unsigned)C, 256, 0, s>>>(A, rows, w.Gp);
        SVD_STEP("svd gram");
        svd_small_kernel<false><<<1, 256, 0, s>>>(w.Gp, C, w.Rinv, nullptr, nullptr);
        SVD_STEP("svd cholesky");
        svd_apply_kernel<<<(unsigned)((rows + 63) / 64), 64, 0, s>>>(A, rows, w.Rinv);
        SVD_STEP("svd apply");
    }
    return cudaSuccess;
}

static cudaError_t svd_sum(const float *P, int splits, int64_t rows, float *out, int sms, cudaStream_t s,
                           const char **stage)
{
    const int64_t blocks = (rows * kSvdRank + 255) / 256;
    const int64_t grid = blocks < (int64_t)sms * 8 ? blocks : (int64_t)sms * 8;
    svd_sum_splits_kernel<<<(unsigned)grid, 256, 0, s>>>(P, splits, rows, out);
    SVD_STEP("svd split sum");
    return cudaSuccess;
}

cudaError_t launch_svd_init(const float *W, int64_t N, int64_t K, const float *omega, int iters, int rank,
                            uint16_t *up, uint16_t *down, float *R, void *ws, int sms, cudaStream_t s,
                            const char **stage)
{
    const int64_t rows = max64(N, K);
    uint8_t *p = reinterpret_cast<uint8_t *>(ws);
    SvdWs w;
    w.Y = reinterpret_cast<float *>(p);
    p += up256((size_t)N * kSvdRank * 4);
    w.V = reinterpret_cast<float *>(p);
    p += up256((size_t)K * kSvdRank * 4);
    w.P = reinterpret_cast<float *>(p);
    p += up256((size_t)svd_partial_rows(N, K) * kSvdRank * 4);
    w.Gp = reinterpret_cast<double *>(p);
    p += up256((size_t)((rows + kGramRows - 1) / kGramRows) * kSvdRank * kSvdRank * 8);
    w.Rinv = reinterpret_cast<float *>(p);
    p += up256(kSvdRank * kSvdRank * 4);
    w.X = reinterpret_cast<double *>(p);
    p += up256(kSvdRank * kSvdRank * 8);
    w.S = reinterpret_cast<double *>(p);

    *stage = "svd start block copy";
    cudaError_t e = cudaMemcpyAsync(w.V, omega, (size_t)K * kSvdRank * 4, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess)
        return e;
    if ((e = svd_orth(w.V, K, 1, w, s, stage)) != cudaSuccess)
        return e;
    const int sv = svd_splits(N / kSvdTile, K), sz = svd_splits(K / kSvdTile, N);
    for (int it = 0; it < iters; ++it) {
        svd_wv_kernel<<<dim3((unsigned)(N / kSvdTile), (unsigned)sv), kSvdTile, 0, s>>>(W, N, K, K / sv, w.V, w.P);
        SVD_STEP("svd W V");
        if ((e = svd_sum(w.P, sv, N, w.Y, sms, s, stage)) != cudaSuccess)
            return e;
        if ((e = svd_orth(w.Y, N, it + 1 < iters ? 1 : 2, w, s, stage)) != cudaSuccess)
            return e;
        svd_wtu_kernel<<<dim3((unsigned)(K / kSvdTile), (unsigned)sz), kSvdTile, 0, s>>>(W, K, N / sz, w.Y, w.P);
        SVD_STEP("svd W^T U");
        if ((e = svd_sum(w.P, sz, K, w.V, sms, s, stage)) != cudaSuccess)
            return e;
        if (it + 1 < iters && (e = svd_orth(w.V, K, 1, w, s, stage)) != cudaSuccess)
            return e;
    }
    // B = W^T U is in w.V; the eigen-decomposition of its Gram gives the rotation and sigma^2
    const int CK = (int)((K + kGramRows - 1) / kGramRows);
    svd_gram_kernel<<<(unsigned)CK, 256, 0, s>>>(w.V, K, w.Gp);
    SVD_STEP("svd gram");
    svd_small_kernel<true><<<1, 256, 0, s>>>(w.Gp, CK, nullptr, w.X, w.S);
    SVD_STEP("svd jacobi");
    if (rank == 16)
        svd_factors_kernel<16><<<(unsigned)((N + K + 255) / 256), 256, 0, s>>>(w.Y, w.V, N, K, w.X, w.S, up, down);
    else
        svd_factors_kernel<32><<<(unsigned)((N + K + 255) / 256), 256, 0, s>>>(w.Y, w.V, N, K, w.X, w.S, up, down);
    SVD_STEP("svd factors");
    const int64_t kbs = K / 256, nts = N / 64;
    int64_t m = ((int64_t)sms * 2) / kbs;              // one wave of two CTAs per SM
    m = m < 1 ? 1 : (m > nts ? nts : m);
    if (rank == 16)
        svd_residual_kernel<16><<<dim3((unsigned)kbs, (unsigned)m), 256, 0, s>>>(W, N, K, up, down, R);
    else
        svd_residual_kernel<32><<<dim3((unsigned)kbs, (unsigned)m), 256, 0, s>>>(W, N, K, up, down, R);
    SVD_STEP("svd residual");
    return cudaSuccess;
}

}  // namespace sq
