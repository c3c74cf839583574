// sq_svd.cu -- SVD init of the rank-32 low-rank branch (SquareQ README,
// "Low-rank branch: rank-32 SVD of the weight, always on, bf16"):
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
// up = U X S^(1/2), down = B X S^(-1/2).  orth(A) is CholeskyQR applied twice.
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
constexpr int kGramRows = 128;         // rows per partial Gram
constexpr int kJacobiMaxSweeps = 30;
constexpr double kJacobiSkip = 1e-15;  // pairs whose cosine is below this are left alone
constexpr double kJacobiTol = 1e-13;   // a sweep whose largest cosine is below this ends the iteration
constexpr unsigned kFull = 0xffffffffu;
constexpr int kSvdTargetCtas = 512;    // product grids are split until they reach this many CTAs

// ---------------------------------------------------------------------------
// Yp[s, n, :] = sum over k in split s of W[n, k] V[k, :], for the 128 rows n of the CTA.
// Grid (N / 128, S), 128 threads.  Warp w owns outputs 8w..8w+7; lane l rows l, l+32, l+64, l+96.
// A stage holds 128 rows x 32 columns of W (row pitch 33 words: the 32 lanes' rows fall in 32
// different banks) and the matching 32 rows of V (read as broadcasts).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kSvdTile) svd_wv_kernel(const float *__restrict__ W, int64_t N, int64_t K,
                                                          int64_t k_per_split, const float *__restrict__ V,
                                                          float *__restrict__ Yp)
{
    __shared__ float Ws[kSvdTile][kSvdChunk + 1];
    __shared__ float Vs[kSvdChunk][kSvdRank];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t n0 = (int64_t)blockIdx.x * kSvdTile;
    const int64_t kbeg = (int64_t)blockIdx.y * k_per_split;
    float acc[4][8];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int o = 0; o < 8; ++o)
            acc[j][o] = 0.0f;
    for (int64_t k0 = kbeg; k0 < kbeg + k_per_split; k0 += kSvdChunk) {
#pragma unroll 8
        for (int i = 0; i < kSvdTile / 4; ++i) {          // row warp + 4i, column lane
            const int r = warp + 4 * i;
            Ws[r][lane] = W[(n0 + r) * K + k0 + lane];
        }
#pragma unroll
        for (int i = 0; i < kSvdChunk * kSvdRank / kSvdTile; ++i) {
            const int e = tid + kSvdTile * i;
            Vs[e >> 5][e & 31] = V[(k0 + (e >> 5)) * kSvdRank + (e & 31)];
        }
        __syncthreads();
#pragma unroll 4
        for (int k = 0; k < kSvdChunk; ++k) {
            float w[4], v[8];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                w[j] = Ws[lane + 32 * j][k];
#pragma unroll
            for (int o = 0; o < 8; ++o)
                v[o] = Vs[k][8 * warp + o];
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int o = 0; o < 8; ++o)
                    acc[j][o] = fmaf(w[j], v[o], acc[j][o]);
        }
        __syncthreads();
    }
    float *out = Yp + (int64_t)blockIdx.y * N * kSvdRank;
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int o = 0; o < 8; ++o)
            out[(n0 + lane + 32 * j) * kSvdRank + 8 * warp + o] = acc[j][o];
}

// ---------------------------------------------------------------------------
// Zp[s, k, :] = sum over rows n of split s of W[n, k] U[n, :], for the 128 columns k of the CTA.
// Grid (K / 128, S), 128 threads.  Warp w owns outputs 8w..8w+7; lane l columns l, l+32, l+64,
// l+96.  A stage holds 32 rows x 128 columns of W and the matching 32 rows of U.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kSvdTile) svd_wtu_kernel(const float *__restrict__ W, int64_t K,
                                                           int64_t n_per_split, const float *__restrict__ U,
                                                           float *__restrict__ Zp)
{
    __shared__ float Ws[kSvdChunk][kSvdTile];
    __shared__ float Us[kSvdChunk][kSvdRank];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t k0 = (int64_t)blockIdx.x * kSvdTile;
    const int64_t nbeg = (int64_t)blockIdx.y * n_per_split;
    float acc[4][8];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int o = 0; o < 8; ++o)
            acc[j][o] = 0.0f;
    for (int64_t n0 = nbeg; n0 < nbeg + n_per_split; n0 += kSvdChunk) {
#pragma unroll 8
        for (int r = 0; r < kSvdChunk; ++r)
            Ws[r][tid] = W[(n0 + r) * K + k0 + tid];
#pragma unroll
        for (int i = 0; i < kSvdChunk * kSvdRank / kSvdTile; ++i) {
            const int e = tid + kSvdTile * i;
            Us[e >> 5][e & 31] = U[(n0 + (e >> 5)) * kSvdRank + (e & 31)];
        }
        __syncthreads();
#pragma unroll 4
        for (int r = 0; r < kSvdChunk; ++r) {
            float w[4], u[8];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                w[j] = Ws[r][lane + 32 * j];
#pragma unroll
            for (int o = 0; o < 8; ++o)
                u[o] = Us[r][8 * warp + o];
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int o = 0; o < 8; ++o)
                    acc[j][o] = fmaf(w[j], u[o], acc[j][o]);
        }
        __syncthreads();
    }
    float *out = Zp + (int64_t)blockIdx.y * K * kSvdRank;
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int o = 0; o < 8; ++o)
            out[(k0 + lane + 32 * j) * kSvdRank + 8 * warp + o] = acc[j][o];
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
// partial Grams of A [rows, 32]: Gp[c][i][j] = sum over rows 128c..128c+127 (in order) of
// a_i a_j, fp64 (each fp32 product is exact in fp64).  Grid rows / 128, 256 threads; thread t
// owns entries (t / 8, 4 (t % 8) .. +3).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) svd_gram_kernel(const float *__restrict__ A, double *__restrict__ Gp)
{
    __shared__ float As[kGramRows][kSvdRank + 1];
    const int tid = threadIdx.x;
    const int64_t r0 = (int64_t)blockIdx.x * kGramRows;
    for (int e = tid; e < kGramRows * kSvdRank; e += 256)
        As[e >> 5][e & 31] = A[(r0 + (e >> 5)) * kSvdRank + (e & 31)];
    __syncthreads();
    const int i = tid >> 3, j0 = 4 * (tid & 7);
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (int r = 0; r < kGramRows; ++r) {
        const double a = (double)As[r][i];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            acc[j] = fma(a, (double)As[r][j0 + j], acc[j]);
    }
    double *g = Gp + (int64_t)blockIdx.x * (kSvdRank * kSvdRank) + i * kSvdRank + j0;
#pragma unroll
    for (int j = 0; j < 4; ++j)
        g[j] = acc[j];
}

// ---------------------------------------------------------------------------
// One-warp 32 x 32 steps.  Lane c holds column c of a matrix in 32 fp64 registers; every
// register index is a compile-time constant (the loops are unrolled), values move between
// lanes by shuffles only.
// ---------------------------------------------------------------------------
// G = sum of the C partial Grams in order; lane c gets column c
__device__ __forceinline__ void svd_load_gram(const double *__restrict__ Gp, int C, int lane, double (&g)[kSvdRank])
{
#pragma unroll
    for (int i = 0; i < kSvdRank; ++i)
        g[i] = Gp[i * kSvdRank + lane];
    for (int c = 1; c < C; ++c) {
        const double *p = Gp + (int64_t)c * (kSvdRank * kSvdRank) + lane;
#pragma unroll
        for (int i = 0; i < kSvdRank; ++i)
            g[i] += p[i * kSvdRank];
    }
}

// Cholesky G = R^T R (R upper triangular), right-looking.  In: g = column `lane` of G (destroyed).
// Out: r = column `lane` of R (r[i] = R[i][lane], zero below the diagonal).  A pivot that is not
// positive (a rank-deficient block, e.g. a zero weight) is a bit of the returned mask; its row of
// R is zero except R[j][j] = dead_diag.
__device__ __forceinline__ uint32_t svd_chol_warp(double (&g)[kSvdRank], double (&r)[kSvdRank], int lane,
                                                  double dead_diag)
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
        const double rjj = dj ? dead_diag : sqrt(d);
        double rjc = 0.0;
        if (lane == j)
            rjc = rjj;
        else if (lane > j && !dj)
            rjc = g[j] / rjj;
        r[j] = rjc;
#pragma unroll
        for (int i = j + 1; i < kSvdRank; ++i) {       // G[i][lane] -= R[j][i] R[j][lane]
            const double rji = __shfl_sync(kFull, rjc, i);
            g[i] = fma(-rji, rjc, g[i]);
        }
    }
    return dead;
}

// Rinv = R^-1 (fp32, row-major 32 x 32): lane c solves R x = e_c by back substitution; the rows
// of dead pivots are zero, so the matching columns of the orthonormalised block are zero.
__device__ __forceinline__ void svd_rinv_warp(const double (&r)[kSvdRank], uint32_t dead, int lane,
                                              float *__restrict__ Rinv)
{
    double x[kSvdRank];
#pragma unroll
    for (int i = kSvdRank - 1; i >= 0; --i) {
        double v = (i == lane) ? 1.0 : 0.0;
#pragma unroll
        for (int k = i + 1; k < kSvdRank; ++k)
            v = fma(-__shfl_sync(kFull, r[i], k), x[k], v);   // R[i][k] is lane k's r[i]
        const double rii = __shfl_sync(kFull, r[i], i);
        x[i] = ((dead >> i) & 1u) ? 0.0 : v / rii;
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
            double a = 0.0, b = 0.0, g = 0.0;
#pragma unroll
            for (int i = 0; i < kSvdRank; ++i) {
                const double p = __shfl_sync(kFull, r[i], partner);
                a = fma(r[i], r[i], a);
                b = fma(p, p, b);
                g = fma(r[i], p, g);
            }
            const double app = lower ? a : b, aqq = lower ? b : a;
            const double nrm = sqrt(app) * sqrt(aqq);
            double c = 1.0, s = 0.0;
            if (fabs(g) > kJacobiSkip * nrm) {
                off = fmax(off, fabs(g) / nrm);
                const double z = (aqq - app) / (2.0 * g);
                const double t = (z >= 0.0 ? 1.0 : -1.0) / (fabs(z) + sqrt(fma(z, z, 1.0)));
                c = 1.0 / sqrt(fma(t, t, 1.0));
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
        if (off <= kJacobiTol)
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
template <bool EIG>
__global__ void __launch_bounds__(32) svd_small_kernel(const double *__restrict__ Gp, int C, float *__restrict__ Rinv,
                                                       double *__restrict__ Xo, double *__restrict__ So)
{
    const int lane = threadIdx.x;
    double g[kSvdRank], r[kSvdRank];
    svd_load_gram(Gp, C, lane, g);
    const uint32_t dead = svd_chol_warp(g, r, lane, EIG ? 0.0 : 1.0);
    if (EIG)
        svd_jacobi_warp(r, lane, Xo, So);
    else
        svd_rinv_warp(r, dead, lane, Rinv);
}

// A[row, :] <- A[row, :] Rinv (Rinv upper triangular, fp32), one row per thread
__global__ void __launch_bounds__(256) svd_apply_kernel(float *__restrict__ A, int64_t rows,
                                                        const float *__restrict__ Rinv)
{
    __shared__ float Rs[kSvdRank][kSvdRank];
    for (int e = threadIdx.x; e < kSvdRank * kSvdRank; e += blockDim.x)
        Rs[e >> 5][e & 31] = Rinv[e];
    __syncthreads();
    const int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (row >= rows)
        return;
    float *a_row = A + row * kSvdRank;
    float a[kSvdRank];
#pragma unroll
    for (int i = 0; i < kSvdRank; ++i)
        a[i] = a_row[i];
#pragma unroll
    for (int j = 0; j < kSvdRank; ++j) {
        float s = 0.0f;
#pragma unroll
        for (int i = 0; i <= j; ++i)
            s = fmaf(a[i], Rs[i][j], s);
        a_row[j] = s;                                  // a[] keeps the old row
    }
}

// up[n, :] = bf16(U[n, :] X S^(1/4)) for rows n < N, then down[k, :] = bf16(B[k, :] X S^(-1/4))
// for the next K rows (S = eigenvalues of B^T B = sigma^2, so S^(1/4) = sigma^(1/2)); a zero
// sigma gives a zero column of down.  One row per thread.
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
    uint16_t *dst = is_up ? up + row * kSvdRank : down + (row - N) * kSvdRank;
    const float *sc = is_up ? sc_up : sc_down;
    float a[kSvdRank];
#pragma unroll
    for (int i = 0; i < kSvdRank; ++i)
        a[i] = src[i];
#pragma unroll
    for (int j = 0; j < kSvdRank; ++j) {
        float s = 0.0f;
#pragma unroll
        for (int i = 0; i < kSvdRank; ++i)
            s = fmaf(a[i], X[i][j], s);
        dst[j] = (uint16_t)f32_to_bf16_bits(s * sc[j]);
    }
}

// ---------------------------------------------------------------------------
// R[n, k] = RN(W[n, k] - L[n, k]), L = fmaf chain over r = 0..31 of up[n, r] down[k, r] from 0
// (the reconstruct's chain).  Tiles of 64 rows x 256 columns, grid-stride; thread t owns column
// 256 kb + t of the tile's 64 rows, lora_down of that column in registers, lora_up rows read as
// shared-memory broadcasts.  R may alias W (each element is read before it is written, by the
// same thread).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) svd_residual_kernel(const float *W, int64_t N, int64_t K,
                                                           const uint16_t *__restrict__ up,
                                                           const uint16_t *__restrict__ down, float *R)
{
    __shared__ float us[64][kSvdRank];
    const int tid = threadIdx.x;
    const int64_t NT = N / 64, T = NT * (K / 256);
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        const int64_t kb = t / NT, n0 = (t % NT) * 64;
        const int64_t k = kb * 256 + tid;
        __syncthreads();                               // the previous tile's reads of us are done
        for (int e = tid; e < 64 * kSvdRank; e += 256)
            us[e >> 5][e & 31] = bf16_bits_to_f32(up[(n0 + (e >> 5)) * kSvdRank + (e & 31)]);
        float d[kSvdRank];
#pragma unroll
        for (int r = 0; r < kSvdRank; ++r)
            d[r] = bf16_bits_to_f32(down[k * kSvdRank + r]);
        __syncthreads();
#pragma unroll 2
        for (int n = 0; n < 64; ++n) {
            float L = 0.0f;
#pragma unroll
            for (int r = 0; r < kSvdRank; ++r)
                L = fmaf(us[n][r], d[r], L);
            const int64_t idx = (n0 + n) * K + k;
            R[idx] = __fsub_rn(W[idx], L);
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

size_t svd_workspace_bytes(int64_t N, int64_t K)
{
    const int64_t rows = max64(N, K);
    return up256((size_t)N * kSvdRank * 4) + up256((size_t)K * kSvdRank * 4) +
           up256((size_t)8 * rows * kSvdRank * 4) + up256((size_t)(rows / kGramRows) * kSvdRank * kSvdRank * 8) +
           up256(kSvdRank * kSvdRank * 4) + up256(kSvdRank * kSvdRank * 8) + up256(kSvdRank * 8);
}

// splits s in {1, 2, 4, 8} of the reduction dimension `depth` (each part a multiple of 32 deep)
// until the grid of `tiles` x s CTAs reaches the target
static int svd_splits(int64_t tiles, int64_t depth)
{
    int s = 1;
    while (s < 8 && tiles * s < kSvdTargetCtas && depth % (kSvdChunk * 2 * s) == 0)
        s *= 2;
    return s;
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

static cudaError_t svd_orth(float *A, int64_t rows, const SvdWs &w, cudaStream_t s, const char **stage)
{
    const int C = (int)(rows / kGramRows);
    for (int pass = 0; pass < 2; ++pass) {             // CholeskyQR, twice
        svd_gram_kernel<<<(unsigned)C, 256, 0, s>>>(A, w.Gp);
        SVD_STEP("svd gram");
        svd_small_kernel<false><<<1, 32, 0, s>>>(w.Gp, C, w.Rinv, nullptr, nullptr);
        SVD_STEP("svd cholesky");
        svd_apply_kernel<<<(unsigned)((rows + 255) / 256), 256, 0, s>>>(A, rows, w.Rinv);
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

cudaError_t launch_svd_init(const float *W, int64_t N, int64_t K, const float *omega, int iters, uint16_t *up,
                            uint16_t *down, float *R, void *ws, int sms, cudaStream_t s, const char **stage)
{
    const int64_t rows = max64(N, K);
    uint8_t *p = reinterpret_cast<uint8_t *>(ws);
    SvdWs w;
    w.Y = reinterpret_cast<float *>(p);
    p += up256((size_t)N * kSvdRank * 4);
    w.V = reinterpret_cast<float *>(p);
    p += up256((size_t)K * kSvdRank * 4);
    w.P = reinterpret_cast<float *>(p);
    p += up256((size_t)8 * rows * kSvdRank * 4);
    w.Gp = reinterpret_cast<double *>(p);
    p += up256((size_t)(rows / kGramRows) * kSvdRank * kSvdRank * 8);
    w.Rinv = reinterpret_cast<float *>(p);
    p += up256(kSvdRank * kSvdRank * 4);
    w.X = reinterpret_cast<double *>(p);
    p += up256(kSvdRank * kSvdRank * 8);
    w.S = reinterpret_cast<double *>(p);

    *stage = "svd start block copy";
    cudaError_t e = cudaMemcpyAsync(w.V, omega, (size_t)K * kSvdRank * 4, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess)
        return e;
    if ((e = svd_orth(w.V, K, w, s, stage)) != cudaSuccess)
        return e;
    const int sv = svd_splits(N / kSvdTile, K), sz = svd_splits(K / kSvdTile, N);
    for (int it = 0; it < iters; ++it) {
        svd_wv_kernel<<<dim3((unsigned)(N / kSvdTile), (unsigned)sv), kSvdTile, 0, s>>>(W, N, K, K / sv, w.V, w.P);
        SVD_STEP("svd W V");
        if ((e = svd_sum(w.P, sv, N, w.Y, sms, s, stage)) != cudaSuccess)
            return e;
        if ((e = svd_orth(w.Y, N, w, s, stage)) != cudaSuccess)
            return e;
        svd_wtu_kernel<<<dim3((unsigned)(K / kSvdTile), (unsigned)sz), kSvdTile, 0, s>>>(W, K, N / sz, w.Y, w.P);
        SVD_STEP("svd W^T U");
        if ((e = svd_sum(w.P, sz, K, w.V, sms, s, stage)) != cudaSuccess)
            return e;
        if (it + 1 < iters && (e = svd_orth(w.V, K, w, s, stage)) != cudaSuccess)
            return e;
    }
    // B = W^T U is in w.V; the eigen-decomposition of its Gram gives the rotation and sigma^2
    const int CK = (int)(K / kGramRows);
    svd_gram_kernel<<<(unsigned)CK, 256, 0, s>>>(w.V, w.Gp);
    SVD_STEP("svd gram");
    svd_small_kernel<true><<<1, 32, 0, s>>>(w.Gp, CK, nullptr, w.X, w.S);
    SVD_STEP("svd jacobi");
    svd_factors_kernel<<<(unsigned)((N + K + 255) / 256), 256, 0, s>>>(w.Y, w.V, N, K, w.X, w.S, up, down);
    SVD_STEP("svd factors");
    const int64_t tiles = (N / 64) * (K / 256);
    const int64_t grid = tiles < (int64_t)sms * 4 ? tiles : (int64_t)sms * 4;
    svd_residual_kernel<<<(unsigned)grid, 256, 0, s>>>(W, N, K, up, down, R);
    SVD_STEP("svd residual");
    return cudaSuccess;
}

}  // namespace sq
