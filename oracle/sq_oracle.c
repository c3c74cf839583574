/*
 * sq_oracle.c -- plain, slow, scalar CPU oracle for the SquareQ W4 linear
 * layer.  TEST INFRASTRUCTURE ONLY: the parity tests, the smoke check and the
 * bench's CPU-baseline leg call it; the product (libsq, the CUDA path) never
 * links, imports or executes anything here, and this file shares no code,
 * header, table or constant with it.
 *
 * What it computes (SquareQ README, section "SquareQ v3 -- W4 (Hadamard-256 +
 * low-rank + int4 / NVFP4)"):
 *
 *     W = lora_up . lora_down^T + inverse_H256( dequant( residual ) )
 *
 * with a block-diagonal normalised Hadamard-256 over the input dim
 * ("Rotation" paragraph), an int4 group-32/64 codec with MSE-swept scale
 * fractions or an NVFP4 codec (e2m1 codes; one ue4m3 scale per 16 values,
 * stored in cuBLASLt's tiled order; one fp32 scale for the tensor) ("Residual codecs"
 * paragraph), and a rank-32 bf16 low-rank branch ("Low-rank branch"); plus
 * the v3.1 int8 mode (int8 per-row MSE-swept codes of the rotated residual,
 * rank-16 low-rank branch; section "v3.1 -- int8-residual mode").
 *
 * Arithmetic rules (the pages fix none of them; these are the readings that
 * make bit-exact parity well defined):
 *   - fp32 values are IEEE binary32, one round-to-nearest-even per operation,
 *     and no contraction into FMA (build with -ffp-contract=off, no
 *     -ffast-math) except where fmaf() is written;
 *   - every narrowing conversion (bf16, fp16, ue4m3, e2m1) is round to nearest,
 *     ties to even, through one routine, round_to_grid(), written from the
 *     formats' definitions;
 *   - forward outputs are evaluated in fp64 on the exact decoded operands.
 *
 * OpenMP only spreads independent rows / groups over threads; each output is
 * still computed by one thread in the order written here.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int or_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* Rounding to a small floating-point grid                                   */
/* ------------------------------------------------------------------------ */

/*
 * Round a non-negative finite value a to the nearest value of a binary
 * floating-point grid with `mant_bits` fraction bits whose smallest normal
 * exponent is `emin` (below 2^emin the spacing is fixed at 2^(emin-mant_bits),
 * i.e. gradual underflow).  Ties go to the even multiple of the spacing, which
 * is the value whose last fraction bit is 0.  No upper limit is applied here.
 * The input is a float widened to double, so a / spacing is exact.
 */
static double round_to_grid(double a, int mant_bits, int emin)
{
    int E;
    if (a == 0.0)
        return 0.0;
    if (a < ldexp(1.0, emin)) {
        E = emin;
    } else {
        int ex;
        (void)frexp(a, &ex);     /* a = m * 2^ex, m in [0.5, 1) */
        E = ex - 1;              /* 2^E <= a < 2^(E+1) */
    }
    double spacing = ldexp(1.0, E - mant_bits);
    return nearbyint(a / spacing) * spacing;   /* default mode: ties to even */
}

/* exponent E with 2^E <= v < 2^(E+1), for v > 0 */
static int floor_log2(double v)
{
    int ex;
    (void)frexp(v, &ex);
    return ex - 1;
}

/* bf16: 7 fraction bits, fp32's exponent range (emin = -126). */
uint16_t or_f32_to_bf16(float v)
{
    uint32_t bits;
    memcpy(&bits, &v, 4);
    uint16_t sign = (uint16_t)((bits >> 16) & 0x8000u);
    if (isnan(v))
        return (uint16_t)(sign | 0x7FC0u);
    if (isinf(v))
        return (uint16_t)(sign | 0x7F80u);
    double r = round_to_grid(fabs((double)v), 7, -126);
    if (r >= ldexp(1.0, 128))
        return (uint16_t)(sign | 0x7F80u);            /* overflow -> inf */
    float rf = (float)r;                               /* exact: r is on the bf16 grid */
    uint32_t rb;
    memcpy(&rb, &rf, 4);
    return (uint16_t)(sign | (rb >> 16));
}

float or_bf16_to_f32(uint16_t h)
{
    uint32_t bits = (uint32_t)h << 16;
    float v;
    memcpy(&v, &bits, 4);
    return v;
}

/* bf16 of n values (the routine above, element by element) */
void or_f32_to_bf16_n(const float *v, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = or_f32_to_bf16(v[i]);
}

/* IEEE binary16: 10 fraction bits, emin = -14, largest finite 65504. */
uint16_t or_f32_to_f16(float v)
{
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    if (isnan(v))
        return (uint16_t)(sign | 0x7E00u);
    if (isinf(v))
        return (uint16_t)(sign | 0x7C00u);
    double r = round_to_grid(fabs((double)v), 10, -14);
    if (r > 65504.0)
        return (uint16_t)(sign | 0x7C00u);            /* overflow -> inf */
    if (r == 0.0)
        return sign;
    if (r < ldexp(1.0, -14))                           /* subnormal: r = m * 2^-24 */
        return (uint16_t)(sign | (uint16_t)(r / ldexp(1.0, -24)));
    int E = floor_log2(r);
    uint32_t mant = (uint32_t)(r / ldexp(1.0, E - 10)) - 1024u;
    return (uint16_t)(sign | ((uint32_t)(E + 15) << 10) | mant);
}

float or_f16_to_f32(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 31;
    int m = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp(1024.0 + m, e - 15 - 10);
    return (float)(sign ? -v : v);
}

/*
 * Unsigned e4m3 ("ue4m3") block scale: 4 exponent bits (bias 7), 3 fraction
 * bits, smallest normal 2^-6, spacing 2^-9 below it, largest finite 448
 * (code 0x7E; 0x7F is NaN).  Conversion is round-to-nearest-even with
 * saturation to 448 ("satfinite").  The input must be >= 0 or NaN.
 */
uint8_t or_f32_to_ue4m3(float v)
{
    if (isnan(v))
        return 0x7Fu;
    if (!(v > 0.0f))
        return 0x00u;
    double r = isinf(v) ? 448.0 : round_to_grid((double)v, 3, -6);
    if (r > 448.0)
        r = 448.0;
    if (r == 0.0)
        return 0x00u;
    if (r < ldexp(1.0, -6))
        return (uint8_t)(r / ldexp(1.0, -9));        /* codes 1..7 */
    int E = floor_log2(r);
    uint32_t mant = (uint32_t)(r / ldexp(1.0, E - 3)) - 8u;
    return (uint8_t)(((uint32_t)(E + 7) << 3) | mant);
}

float or_ue4m3_to_f32(uint8_t c)
{
    int e = (c >> 3) & 15;
    int m = c & 7;
    if (c == 0x7F || c == 0xFF)
        return NAN;
    if (e == 0)
        return (float)ldexp((double)m, -9);
    return (float)ldexp(8.0 + m, e - 7 - 3);
}

/*
 * e2m1 (FP4): sign bit, 2 exponent bits (bias 1), 1 fraction bit.
 * Magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6} for codes 0..7.  Conversion is
 * round-to-nearest-even with saturation to 6; the sign bit is kept, so a
 * negative value that rounds to zero gives code 0x8.
 */
uint8_t or_f32_to_e2m1(float v)
{
    static const double grid[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    uint8_t sign = signbit(v) ? 0x8u : 0x0u;
    double a = fabs((double)v);
    double r = isinf(v) ? 6.0 : round_to_grid(a, 1, 0);
    if (r > 6.0)
        r = 6.0;
    for (uint8_t c = 0; c < 8; c++)
        if (grid[c] == r)
            return (uint8_t)(sign | c);
    return (uint8_t)(sign | 0x7u);   /* unreachable for finite inputs */
}

float or_e2m1_to_f32(uint8_t c)
{
    static const float mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
    float v = mag[c & 7];
    return (c & 8) ? -v : v;
}

/* ------------------------------------------------------------------------ */
/* O1, O2: block-diagonal normalised Hadamard-256 over the input dim         */
/* ------------------------------------------------------------------------ */

/*
 * In-place normalised Hadamard transform of 256 values (SquareQ README,
 * "Rotation" paragraph: block-diagonal normalised Hadamard-256).  Reading:
 * Sylvester ordering, H[i][j] = (-1)^popcount(i & j) / 16, evaluated as
 * radix-2 butterflies with strides 1, 2, 4, ..., 128 (each butterfly writes
 * a+b to the lower and a-b to the upper index), then a scale by 1/16, which
 * is exact in binary.  H is symmetric and orthogonal, so it is its own
 * inverse: the same routine serves as inverse_H256.
 */
void or_fwht256(float *v)
{
    for (int h = 1; h < 256; h <<= 1) {
        for (int j = 0; j < 256; j++) {
            if ((j & h) == 0) {
                float a = v[j];
                float b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
        }
    }
    for (int j = 0; j < 256; j++)
        v[j] = v[j] * 0.0625f;
}

/* Rotate every 256-wide block of every row of a [rows, K] fp32 matrix. */
void or_rotate_rows_f32(const float *in, int64_t rows, int64_t K, float *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t b = 0; b < K; b += 256) {
            float v[256];
            for (int i = 0; i < 256; i++)
                v[i] = in[r * K + b + i];
            or_fwht256(v);
            for (int i = 0; i < 256; i++)
                out[r * K + b + i] = v[i];
        }
    }
}

/* Same for a bf16 matrix (bit patterns); bf16 widens to fp32 exactly. */
void or_rotate_rows_bf16(const uint16_t *in, int64_t rows, int64_t K, float *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t b = 0; b < K; b += 256) {
            float v[256];
            for (int i = 0; i < 256; i++)
                v[i] = or_bf16_to_f32(in[r * K + b + i]);
            or_fwht256(v);
            for (int i = 0; i < 256; i++)
                out[r * K + b + i] = v[i];
        }
    }
}

/* ------------------------------------------------------------------------ */
/* O3: int4 group-32 codec with an MSE-swept scale fraction                  */
/* ------------------------------------------------------------------------ */

/*
 * Fraction j of the sweep: f_j = (50 + 2 j) / 100, j = 0..25, correctly
 * rounded to fp32 (IEEE division of two exact values).
 */
float or_int4_fraction(int j)
{
    return (float)(50 + 2 * j) / 100.0f;
}

/*
 * One group of 32 rotated residual values (SquareQ README, "Residual codecs":
 * int4 group-32 scales with MSE-swept fractions).  For each fraction f_j the
 * scale is s = fp16(RN(RN(f_j * a) / 7)), a = max|r_i|, and the codes are
 * q_i = clamp(rint_even(RN(r_i * RN(1/s))), -7, 7); the group's squared error
 * sum_i RN((r_i - q_i s)^2) is accumulated by an xor butterfly over the 32
 * lanes (strides 16, 8, 4, 2, 1; lane 0's value is the result).  A scale that
 * rounds to 0 gives q = 0 and error r_i.  The smallest error wins; on a tie the
 * smaller fraction wins.  Outputs: 32 codes in [-7, 7], the fp16 scale bits,
 * the winning j.
 */
void or_int4_group32(const float *r, int8_t *q_out, uint16_t *s_out, uint8_t *j_out)
{
    float a = 0.0f;
    for (int i = 0; i < 32; i++) {
        float m = fabsf(r[i]);
        if (m > a)
            a = m;
    }
    float best = INFINITY;
    int best_j = -1;
    for (int j = 0; j < 26; j++) {
        float f = or_int4_fraction(j);
        float fa = f * a;
        float s7 = fa / 7.0f;
        uint16_t sh = or_f32_to_f16(s7);
        float s = or_f16_to_f32(sh);
        int8_t q[32];
        float p[32];
        if (s == 0.0f) {
            for (int i = 0; i < 32; i++) {
                q[i] = 0;
                p[i] = r[i] * r[i];
            }
        } else {
            float inv = 1.0f / s;
            for (int i = 0; i < 32; i++) {
                float v = r[i] * inv;
                float rq = nearbyintf(v);
                if (rq > 7.0f)
                    rq = 7.0f;
                if (rq < -7.0f)
                    rq = -7.0f;
                q[i] = (int8_t)rq;
                float qs = rq * s;              /* exact: <= 14 significant bits */
                float e = r[i] - qs;
                p[i] = e * e;
            }
        }
        for (int d = 16; d >= 1; d >>= 1) {
            float nxt[32];
            for (int i = 0; i < 32; i++)
                nxt[i] = p[i] + p[i ^ d];
            memcpy(p, nxt, sizeof(p));
        }
        float mse = p[0];
        if (best_j < 0 || mse < best) {
            best = mse;
            best_j = j;
            memcpy(q_out, q, 32);
            *s_out = sh;
        }
    }
    *j_out = (uint8_t)best_j;
}

/*
 * One group of 64 rotated residual values: the group-64 variant the same
 * paragraph allows beside group 32.  The same sweep
 * over the 64 values (a = max|r_i| over all 64); the pages give no order for
 * the squared-error sum, and the reading taken here is the group-32 rule per
 * half: each 32-value half is summed by the xor butterfly above (strides 16, 8,
 * 4, 2, 1), then the two half sums are added (first half + second half).
 */
void or_int4_group64(const float *r, int8_t *q_out, uint16_t *s_out, uint8_t *j_out)
{
    float a = 0.0f;
    for (int i = 0; i < 64; i++) {
        float m = fabsf(r[i]);
        if (m > a)
            a = m;
    }
    float best = INFINITY;
    int best_j = -1;
    for (int j = 0; j < 26; j++) {
        float f = or_int4_fraction(j);
        float fa = f * a;
        float s7 = fa / 7.0f;
        uint16_t sh = or_f32_to_f16(s7);
        float s = or_f16_to_f32(sh);
        int8_t q[64];
        float p[64];
        if (s == 0.0f) {
            for (int i = 0; i < 64; i++) {
                q[i] = 0;
                p[i] = r[i] * r[i];
            }
        } else {
            float inv = 1.0f / s;
            for (int i = 0; i < 64; i++) {
                float v = r[i] * inv;
                float rq = nearbyintf(v);
                if (rq > 7.0f)
                    rq = 7.0f;
                if (rq < -7.0f)
                    rq = -7.0f;
                q[i] = (int8_t)rq;
                float qs = rq * s;              /* exact: <= 14 significant bits */
                float e = r[i] - qs;
                p[i] = e * e;
            }
        }
        float half[2];
        for (int h = 0; h < 2; h++) {
            float *ph = p + 32 * h;
            for (int d = 16; d >= 1; d >>= 1) {
                float nxt[32];
                for (int i = 0; i < 32; i++)
                    nxt[i] = ph[i] + ph[i ^ d];
                memcpy(ph, nxt, sizeof(nxt));
            }
            half[h] = ph[0];
        }
        float mse = half[0] + half[1];
        if (best_j < 0 || mse < best) {
            best = mse;
            best_j = j;
            memcpy(q_out, q, 64);
            *s_out = sh;
        }
    }
    *j_out = (uint8_t)best_j;
}

/*
 * int4 builder: rotate R [N, K] fp32 row-blockwise, then run the group codec
 * on every 32 consecutive rotated values of a row.  codes [N, K/2]: element
 * 2k in the low nibble, 4-bit two's complement; scales [N, K/32] fp16 bits;
 * frac [N, K/32] winning j (may be NULL).
 */
void or_build_int4(const float *R, int64_t N, int64_t K,
                   uint8_t *codes, uint16_t *scales, uint8_t *frac)
{
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++) {
        for (int64_t b = 0; b < K; b += 256) {
            float v[256];
            for (int i = 0; i < 256; i++)
                v[i] = R[n * K + b + i];
            or_fwht256(v);
            for (int g = 0; g < 8; g++) {
                int8_t q[32];
                uint16_t s;
                uint8_t j;
                or_int4_group32(v + 32 * g, q, &s, &j);
                int64_t gi = n * (K / 32) + (b / 32) + g;
                scales[gi] = s;
                if (frac)
                    frac[gi] = j;
                for (int i = 0; i < 32; i += 2) {
                    uint8_t lo = (uint8_t)q[i] & 0xFu;
                    uint8_t hi = (uint8_t)q[i + 1] & 0xFu;
                    codes[n * (K / 2) + (b + 32 * g + i) / 2] = (uint8_t)(lo | (hi << 4));
                }
            }
        }
    }
}

/*
 * The same builder for a group size of 32 or 64: scales and frac are
 * [N, K/group].  group 32 is or_build_int4.
 */
void or_build_int4_g(const float *R, int64_t N, int64_t K, int group,
                     uint8_t *codes, uint16_t *scales, uint8_t *frac)
{
    if (group == 32) {
        or_build_int4(R, N, K, codes, scales, frac);
        return;
    }
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++) {
        for (int64_t b = 0; b < K; b += 256) {
            float v[256];
            for (int i = 0; i < 256; i++)
                v[i] = R[n * K + b + i];
            or_fwht256(v);
            for (int g = 0; g < 4; g++) {
                int8_t q[64];
                uint16_t s;
                uint8_t j;
                or_int4_group64(v + 64 * g, q, &s, &j);
                int64_t gi = n * (K / 64) + (b / 64) + g;
                scales[gi] = s;
                if (frac)
                    frac[gi] = j;
                for (int i = 0; i < 64; i += 2) {
                    uint8_t lo = (uint8_t)q[i] & 0xFu;
                    uint8_t hi = (uint8_t)q[i + 1] & 0xFu;
                    codes[n * (K / 2) + (b + 64 * g + i) / 2] = (uint8_t)(lo | (hi << 4));
                }
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* O4, O5: NVFP4 codec and the tiled scale-factor layout                     */
/* ------------------------------------------------------------------------ */

/*
 * Byte offset of scale (row r, scale column c) in the tiled layout, C = K/16
 * scale columns per row (a multiple of 4).  The pages name cuBLASLt's tiled scale
 * layout without printing it; this is the publicly documented 1D
 * block-scaling layout: 128-row x 4-column tiles of 512 bytes, tiles ordered
 * along the scale columns first, and inside a tile row r%32 picks a 16-byte
 * line, (r%128)/32 a 4-byte word in it and c%4 the byte.
 */
int64_t or_sf_offset(int64_t r, int64_t c, int64_t C)
{
    return ((r / 128) * (C / 4) + c / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4);
}

/* bytes of a tiled scale buffer for `rows` rows of K elements */
int64_t or_sf_bytes(int64_t rows, int64_t K)
{
    return ((rows + 127) / 128) * 128 * (K / 16);
}

/* Global scale g = RN(A / (6 * 448)) from the rotated tensor's absmax A. */
float or_nvfp4_global_scale(float A)
{
    return A / 2688.0f;
}

/*
 * One block of 16 rotated values with global scale g (SquareQ README,
 * "Residual codecs": e2m1 codes, a ue4m3 scale per 16 values and one fp32
 * scale for the tensor).
 * b = max|r|, sf = ue4m3(RN(b / RN(6 g))); with den = RN(value(sf) * g) the
 * codes are e2m1(RN(r_i * RN(1/den))).  sf == 0 or g == 0 gives all-zero
 * codes.  codes8 gets 8 bytes, element 2k in the low nibble.
 */
void or_nvfp4_block16(const float *r, float g, uint8_t *codes8, uint8_t *sf_out)
{
    float b = 0.0f;
    for (int i = 0; i < 16; i++) {
        float m = fabsf(r[i]);
        if (m > b)
            b = m;
    }
    uint8_t sf = 0;
    uint8_t c[16];
    memset(c, 0, sizeof(c));
    if (g != 0.0f) {
        float sixg = 6.0f * g;
        float ratio = b / sixg;
        sf = or_f32_to_ue4m3(ratio);
        if (sf != 0) {
            float dec = or_ue4m3_to_f32(sf);
            float den = dec * g;
            float inv = 1.0f / den;
            for (int i = 0; i < 16; i++)
                c[i] = or_f32_to_e2m1(r[i] * inv);
        }
    }
    for (int i = 0; i < 8; i++)
        codes8[i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));
    *sf_out = sf;
}

/*
 * Quantise an already rotated [rows, K] fp32 matrix with global scale g.
 * codes [rows, K/2]; sf_tiled gets or_sf_bytes(rows, K) bytes in the tiled
 * layout, padding rows zero.
 */
void or_nvfp4_quant_rotated(const float *rot, int64_t rows, int64_t K, float g,
                            uint8_t *codes, uint8_t *sf_tiled)
{
    int64_t C = K / 16;
    memset(sf_tiled, 0, (size_t)or_sf_bytes(rows, K));
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t c = 0; c < C; c++) {
            uint8_t sf;
            or_nvfp4_block16(rot + r * K + 16 * c, g, codes + r * (K / 2) + 8 * c, &sf);
            sf_tiled[or_sf_offset(r, c, C)] = sf;
        }
    }
}

static float absmax_f32(const float *v, int64_t n)
{
    float a = 0.0f;
    for (int64_t i = 0; i < n; i++) {
        float m = fabsf(v[i]);
        if (m > a)
            a = m;
    }
    return a;
}

/*
 * NVFP4 builder: rotate R, A = max|rotated R|, g_w = RN(A / 2688), then the
 * block codec.  `rot_scratch` holds N*K floats (caller-owned).
 */
void or_build_nvfp4(const float *R, int64_t N, int64_t K, float *rot_scratch,
                    uint8_t *codes, uint8_t *sf_tiled, float *g_out)
{
    or_rotate_rows_f32(R, N, K, rot_scratch);
    float A = absmax_f32(rot_scratch, N * K);
    float g = or_nvfp4_global_scale(A);
    or_nvfp4_quant_rotated(rot_scratch, N, K, g, codes, sf_tiled);
    *g_out = g;
}

/*
 * O6 activation quantisation: rotate x [M, K] bf16, g_x = RN(max|xr| / 2688)
 * unless `static_g` is set (then *g_inout is used as given), block codec, and
 * the low-rank input t[m, r] = sum_k x[m, k] * lora_down[k, r] in fp64
 * (lora_down [K, 32] bf16; t may be NULL).  `rot_scratch` holds M*K floats.
 */
void or_act_quant_nvfp4(const uint16_t *x, int64_t M, int64_t K, int static_g,
                        float *g_inout, float *rot_scratch,
                        uint8_t *codes, uint8_t *sf_tiled,
                        const uint16_t *lora_down, double *t)
{
    or_rotate_rows_bf16(x, M, K, rot_scratch);
    float g = *g_inout;
    if (!static_g)
        g = or_nvfp4_global_scale(absmax_f32(rot_scratch, M * K));
    or_nvfp4_quant_rotated(rot_scratch, M, K, g, codes, sf_tiled);
    *g_inout = g;
    if (t) {
#pragma omp parallel for schedule(static)
        for (int64_t m = 0; m < M; m++) {
            for (int rr = 0; rr < 32; rr++) {
                double acc = 0.0;
                for (int64_t k = 0; k < K; k++)
                    acc += (double)or_bf16_to_f32(x[m * K + k]) *
                           (double)or_bf16_to_f32(lora_down[k * 32 + rr]);
                t[m * 32 + rr] = acc;
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* O7, O8: forward y = x . W^T                                              */
/* ------------------------------------------------------------------------ */

/*
 * Since W = U D^T + H(deq(Q)) and H is symmetric, y = x W^T =
 * H(x) deq(Q)^T + (x D) U^T: the rotation moves onto the activation
 * (SquareQ README, the op-level parity paragraph of the FP4 forward: rotation,
 * block quantisation and tiled scales of x, then the GEMM and its epilogue).
 *
 * NVFP4 forward, fp64 on the exact decoded operands:
 *   y[m,n] = g_x g_w sum_k e2m1(xc[m,k]) sf_x(m,k/16) e2m1(wc[n,k]) sf_w(n,k/16)
 *            + sum_r t[m,r] U[n,r]
 * Only the rows listed in `rows` (n_rows of them) are evaluated; y is
 * [n_rows, N].  t is [M, 32] fp64 (or NULL for no low-rank term), U [N, 32]
 * bf16 bits.
 */
void or_linear_fwd_nvfp4(const uint8_t *xc, const uint8_t *xsf, float g_x,
                         const uint8_t *wc, const uint8_t *wsf, float g_w,
                         const double *t, const uint16_t *U,
                         int64_t M, int64_t N, int64_t K,
                         const int64_t *rows, int64_t n_rows, double *y)
{
    int64_t C = K / 16;
    (void)M;
    /* decoded activation rows, e2m1 * sf (exact in fp64) */
    double *xd = (double *)malloc((size_t)(n_rows * K) * sizeof(double));
    for (int64_t i = 0; i < n_rows; i++) {
        int64_t m = rows[i];
        for (int64_t k = 0; k < K; k++) {
            uint8_t byte = xc[m * (K / 2) + k / 2];
            uint8_t code = (k & 1) ? (byte >> 4) : (byte & 0xF);
            xd[i * K + k] = (double)or_e2m1_to_f32(code) *
                            (double)or_ue4m3_to_f32(xsf[or_sf_offset(m, k / 16, C)]);
        }
    }
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++) {
        double *wd = (double *)malloc((size_t)K * sizeof(double));
        for (int64_t k = 0; k < K; k++) {
            uint8_t byte = wc[n * (K / 2) + k / 2];
            uint8_t code = (k & 1) ? (byte >> 4) : (byte & 0xF);
            wd[k] = (double)or_e2m1_to_f32(code) *
                    (double)or_ue4m3_to_f32(wsf[or_sf_offset(n, k / 16, C)]);
        }
        for (int64_t i = 0; i < n_rows; i++) {
            int64_t m = rows[i];
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++)
                acc += xd[i * K + k] * wd[k];
            double out = (double)g_x * (double)g_w * acc;
            if (t)
                for (int r = 0; r < 32; r++)
                    out += t[m * 32 + r] * (double)or_bf16_to_f32(U[n * 32 + r]);
            y[i * N + n] = out;
        }
        free(wd);
    }
    free(xd);
}

/*
 * int4 forward ("dequant-first"), fp64 on the exact operands:
 *   xb = bf16(H(x)),  wb[n,k] = bf16(q[n,k] * s[n,k/32]),
 *   y[m,n] = sum_k xb wb + sum_r t[m,r] U[n,r].
 * xrot is the fp32 rotated x [M, K]; codes/scales as or_build_int4 writes.
 */
void or_linear_fwd_int4_g(const float *xrot, const uint8_t *codes, const uint16_t *scales, int group,
                          const double *t, const uint16_t *U,
                          int64_t M, int64_t N, int64_t K,
                          const int64_t *rows, int64_t n_rows, double *y)
{
    (void)M;
    double *xb = (double *)malloc((size_t)(n_rows * K) * sizeof(double));
    for (int64_t i = 0; i < n_rows; i++)
        for (int64_t k = 0; k < K; k++)
            xb[i * K + k] = (double)or_bf16_to_f32(or_f32_to_bf16(xrot[rows[i] * K + k]));
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++) {
        double *wb = (double *)malloc((size_t)K * sizeof(double));
        for (int64_t k = 0; k < K; k++) {
            uint8_t byte = codes[n * (K / 2) + k / 2];
            int nib = (k & 1) ? (byte >> 4) : (byte & 0xF);
            int q = nib >= 8 ? nib - 16 : nib;
            float s = or_f16_to_f32(scales[n * (K / group) + k / group]);
            float d = (float)q * s;                     /* exact */
            wb[k] = (double)or_bf16_to_f32(or_f32_to_bf16(d));
        }
        for (int64_t i = 0; i < n_rows; i++) {
            int64_t m = rows[i];
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++)
                acc += xb[i * K + k] * wb[k];
            if (t)
                for (int r = 0; r < 32; r++)
                    acc += t[m * 32 + r] * (double)or_bf16_to_f32(U[n * 32 + r]);
            y[i * N + n] = acc;
        }
        free(wb);
    }
    free(xb);
}

/* group 32 (scales [N, K/32]) */
void or_linear_fwd_int4(const float *xrot, const uint8_t *codes, const uint16_t *scales,
                        const double *t, const uint16_t *U,
                        int64_t M, int64_t N, int64_t K,
                        const int64_t *rows, int64_t n_rows, double *y)
{
    or_linear_fwd_int4_g(xrot, codes, scales, 32, t, U, M, N, K, rows, n_rows, y);
}

/* ------------------------------------------------------------------------ */
/* v3.1 int8 per-row codec (rank-16 low-rank branch)                         */
/* ------------------------------------------------------------------------ */

/*
 * The squared-error sum of one row of K values p[0..K-1] (K % 256 == 0), in
 * the order fixed for the int8 codec: inside each 256-block, every 32-value
 * group is summed by the xor butterfly of the int4 codec (strides 16, 8, 4, 2,
 * 1; element 0), the block's 8 group sums by an xor butterfly over the group
 * index (strides 4, 2, 1; group 0), and the blocks are added in order from
 * block 0: E = ((B_0 + B_1) + B_2) + ...  The pages print no order; this is
 * the reading (one level more than the int4 group rule, then a plain running
 * sum over the row).
 */
static float int8_row_error(const float *p_in, int64_t K)
{
    float E = 0.0f;
    for (int64_t b = 0; b < K; b += 256) {
        float g[8];
        for (int k = 0; k < 8; k++) {
            float p[32];
            memcpy(p, p_in + b + 32 * k, sizeof(p));
            for (int d = 16; d >= 1; d >>= 1) {
                float nxt[32];
                for (int i = 0; i < 32; i++)
                    nxt[i] = p[i] + p[i ^ d];
                memcpy(p, nxt, sizeof(p));
            }
            g[k] = p[0];
        }
        for (int d = 4; d >= 1; d >>= 1) {
            float nxt[8];
            for (int k = 0; k < 8; k++)
                nxt[k] = g[k] + g[k ^ d];
            memcpy(g, nxt, sizeof(g));
        }
        E = (b == 0) ? g[0] : E + g[0];
    }
    return E;
}

/*
 * One row of K rotated residual values (SquareQ README, "v3.1 -- int8-residual
 * mode": the rotated residual of a rank-16 branch in int8, one MSE-chosen
 * scale per row).
 * a = max|r_k| over the row; for each fraction f_j of the int4 sweep
 * (j = 0..25) the fp32 scale is s = RN(RN(f_j a) / 127) and the codes
 * q_k = clamp(rint_even(RN(r_k RN(1/s))), -127, 127); the error of value k is
 * e_k = fmaf(-q_k, s, r_k) (r - q s with one rounding: q s is not exact in
 * fp32 any more) and p_k = RN(e_k^2), summed by int8_row_error.  A scale of 0
 * gives q = 0 and p_k = RN(r_k^2).  The smallest error wins, the smaller j on a
 * tie.  Readings: the scale is kept in fp32 (one per row, so its bytes do not
 * matter), the code range is symmetric (-128 is never used), the fraction grid
 * is the int4 codec's.
 */
void or_int8_row(const float *r, int64_t K, int8_t *q_out, float *s_out, uint8_t *j_out)
{
    float a = 0.0f;
    for (int64_t k = 0; k < K; k++) {
        float m = fabsf(r[k]);
        if (m > a)
            a = m;
    }
    float *p = (float *)malloc((size_t)K * sizeof(float));
    int8_t *q = (int8_t *)malloc((size_t)K);
    float best = INFINITY;
    int best_j = -1;
    for (int j = 0; j < 26; j++) {
        float f = or_int4_fraction(j);
        float fa = f * a;
        float s = fa / 127.0f;
        if (s == 0.0f) {
            for (int64_t k = 0; k < K; k++) {
                q[k] = 0;
                p[k] = r[k] * r[k];
            }
        } else {
            float inv = 1.0f / s;
            for (int64_t k = 0; k < K; k++) {
                float v = r[k] * inv;
                float rq = nearbyintf(v);
                if (rq > 127.0f)
                    rq = 127.0f;
                if (rq < -127.0f)
                    rq = -127.0f;
                q[k] = (int8_t)rq;
                float e = fmaf(-rq, s, r[k]);
                p[k] = e * e;
            }
        }
        float E = int8_row_error(p, K);
        if (best_j < 0 || E < best) {
            best = E;
            best_j = j;
            memcpy(q_out, q, (size_t)K);
            *s_out = s;
        }
    }
    *j_out = (uint8_t)best_j;
    free(p);
    free(q);
}

/*
 * int8 builder: rotate each row of R [N, K] block-wise with H256, then the row
 * codec.  codes [N, K] int8, scales [N] fp32, frac [N] (may be NULL).
 */
void or_build_int8(const float *R, int64_t N, int64_t K, int8_t *codes, float *scales, uint8_t *frac)
{
#pragma omp parallel for schedule(dynamic)
    for (int64_t n = 0; n < N; n++) {
        float *row = (float *)malloc((size_t)K * sizeof(float));
        for (int64_t b = 0; b < K; b += 256) {
            memcpy(row + b, R + n * K + b, 256 * sizeof(float));
            or_fwht256(row + b);
        }
        uint8_t j;
        or_int8_row(row, K, codes + n * K, scales + n, &j);
        if (frac)
            frac[n] = j;
        free(row);
    }
}

/*
 * int8 forward ("dequant-first", as the int4 codec), fp64 on the exact operands:
 *   xb = bf16(H(x)),  wb[n,k] = bf16(RN(q[n,k] * s[n])),
 *   y[m,n] = sum_k xb wb + sum_{r<16} t[m,r] U[n,r]
 * with the rank-16 branch: t [M, 16] fp64 = x lora_down, U [N, 16] bf16.
 */
void or_linear_fwd_int8(const float *xrot, const int8_t *codes, const float *scales,
                        const double *t, const uint16_t *U,
                        int64_t M, int64_t N, int64_t K,
                        const int64_t *rows, int64_t n_rows, double *y)
{
    (void)M;
    double *xb = (double *)malloc((size_t)(n_rows * K) * sizeof(double));
    for (int64_t i = 0; i < n_rows; i++)
        for (int64_t k = 0; k < K; k++)
            xb[i * K + k] = (double)or_bf16_to_f32(or_f32_to_bf16(xrot[rows[i] * K + k]));
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++) {
        double *wb = (double *)malloc((size_t)K * sizeof(double));
        for (int64_t k = 0; k < K; k++) {
            float d = (float)codes[n * K + k] * scales[n];
            wb[k] = (double)or_bf16_to_f32(or_f32_to_bf16(d));
        }
        for (int64_t i = 0; i < n_rows; i++) {
            int64_t m = rows[i];
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++)
                acc += xb[i * K + k] * wb[k];
            if (t)
                for (int r = 0; r < 16; r++)
                    acc += t[m * 16 + r] * (double)or_bf16_to_f32(U[n * 16 + r]);
            y[i * N + n] = acc;
        }
        free(wb);
    }
    free(xb);
}

/* low-rank input t[m, r] = sum_k x[m, k] lora_down[k, r] in fp64, rank columns */
void or_lowrank_input(const uint16_t *x, int64_t M, int64_t K, const uint16_t *lora_down, int rank, double *t)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; m++) {
        for (int rr = 0; rr < rank; rr++) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++)
                acc += (double)or_bf16_to_f32(x[m * K + k]) * (double)or_bf16_to_f32(lora_down[k * rank + rr]);
            t[m * rank + rr] = acc;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* O9: bf16 reconstruct of W from the payload                                */
/* ------------------------------------------------------------------------ */

/*
 * W[n,k] = bf16( RN( L[n,k] + h[n,k] ) ) (SquareQ README, the op-level parity
 * paragraph: the backward's bf16 reconstruct from the forward's payload), where
 *   d = q * s (int4, exact) or RN(RN(e2m1 * value(sf)) * g_w) (NVFP4),
 *   h = inverse_H256 of d over each 256-block of the row (= the same FWHT),
 *   L = fmaf chain over r = 0..31 of U[n,r] * D[k,r], starting from 0.
 * residual_only drops L: W = bf16(h).
 * fmt: 1 = int4 g32 (scales fp16 [N, K/32]), 2 = NVFP4 (sf tiled, g_w),
 * 3 = int4 g64 (scales fp16 [N, K/64]), 4 = int8 per row (codes int8 [N, K],
 * scales fp32 [N], d = RN(q * s), low-rank rank 16: U [N, 16], D [K, 16], the
 * fmaf chain over r = 0..15).
 */
void or_reconstruct_bf16(int fmt, const uint8_t *codes, const void *scales, float g_w,
                         const uint16_t *U, const uint16_t *D,
                         int64_t N, int64_t K, int residual_only, uint16_t *W)
{
    int64_t C = K / 16;
    const int rank = fmt == 4 ? 16 : 32;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++) {
        for (int64_t b = 0; b < K; b += 256) {
            float v[256];
            for (int i = 0; i < 256; i++) {
                int64_t k = b + i;
                if (fmt == 4) {
                    v[i] = (float)((const int8_t *)codes)[n * K + k] * ((const float *)scales)[n];
                    continue;
                }
                uint8_t byte = codes[n * (K / 2) + k / 2];
                uint8_t nib = (k & 1) ? (byte >> 4) : (byte & 0xF);
                if (fmt == 1 || fmt == 3) {
                    const int64_t G = fmt == 3 ? 64 : 32;
                    int q = nib >= 8 ? (int)nib - 16 : (int)nib;
                    float s = or_f16_to_f32(((const uint16_t *)scales)[n * (K / G) + k / G]);
                    v[i] = (float)q * s;
                } else {
                    float dec = or_ue4m3_to_f32(((const uint8_t *)scales)[or_sf_offset(n, k / 16, C)]);
                    float e = or_e2m1_to_f32(nib);
                    float ed = e * dec;
                    v[i] = ed * g_w;
                }
            }
            or_fwht256(v);
            for (int i = 0; i < 256; i++) {
                int64_t k = b + i;
                float out = v[i];
                if (!residual_only) {
                    float L = 0.0f;
                    for (int r = 0; r < rank; r++)
                        L = fmaf(or_bf16_to_f32(U[n * rank + r]), or_bf16_to_f32(D[k * rank + r]), L);
                    out = L + v[i];
                }
                W[n * K + k] = or_f32_to_bf16(out);
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Backward of the input: dx = dy W on the bf16 reconstruct                  */
/* ------------------------------------------------------------------------ */

/*
 * dx[m, k] = sum_n dy[m, n] W[n, k] in fp64 on the exact bf16 operands
 * (SquareQ README, "End-to-end": the backward rebuilds bf16 W from the payload
 * and runs the normal bf16 GEMM).  dy [M, N] and W [N, K] are bf16 bits (W as
 * or_reconstruct_bf16 writes it); only the rows listed in `rows` are
 * evaluated; dx is [n_rows, K].
 */
void or_linear_bwd_dx(const uint16_t *dy, const uint16_t *W, int64_t M, int64_t N, int64_t K,
                      const int64_t *rows, int64_t n_rows, double *dx)
{
    (void)M;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n_rows; i++) {
        double *acc = (double *)calloc((size_t)K, sizeof(double));
        for (int64_t n = 0; n < N; n++) {
            double a = (double)or_bf16_to_f32(dy[rows[i] * N + n]);
            if (a == 0.0)
                continue;
            for (int64_t k = 0; k < K; k++)
                acc[k] += a * (double)or_bf16_to_f32(W[n * K + k]);
        }
        memcpy(dx + i * K, acc, (size_t)K * sizeof(double));
        free(acc);
    }
}

/* ------------------------------------------------------------------------ */
/* SVD init: residual of the low-rank branch                                */
/* ------------------------------------------------------------------------ */

/*
 * R[n, k] = RN(W[n, k] - L[n, k]) with L the fmaf chain over r = 0..rank-1 of
 * up[n, r] * down[k, r] from 0 -- the same L the bf16 reconstruct adds back
 * (SquareQ README, "Low-rank branch" paragraph: the branch comes from the
 * weight's SVD, and the residual is what is left of the weight; "v3.1 -- int8-residual mode": rank
 * 16).  W, R fp32 [N, K]; up [N, rank], down [K, rank] bf16 bits; rank 32 or 16.
 */
void or_svd_residual(const float *W, const uint16_t *up, const uint16_t *down, int64_t N, int64_t K, int rank,
                     float *R)
{
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++) {
        for (int64_t k = 0; k < K; k++) {
            float L = 0.0f;
            for (int r = 0; r < rank; r++)
                L = fmaf(or_bf16_to_f32(up[n * rank + r]), or_bf16_to_f32(down[k * rank + r]), L);
            R[n * K + k] = W[n * K + k] - L;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* SVD init: the rank-32 (or rank-16) truncated SVD of the weight            */
/* ------------------------------------------------------------------------ */

/*
 * bf16 of an fp64 value, rounded once (round to nearest, ties to even) on the
 * bf16 grid: 7 fraction bits, fp32's exponent range, overflow to infinity.
 * Going through fp32 first would round twice, which differs whenever the fp32
 * value lands on a bf16 midpoint that the fp64 value is not on.
 */
uint16_t or_f64_to_bf16(double v)
{
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    if (isnan(v))
        return (uint16_t)(sign | 0x7FC0u);
    if (isinf(v))
        return (uint16_t)(sign | 0x7F80u);
    double r = round_to_grid(fabs(v), 7, -126);      /* a / spacing is exact for any double */
    if (r >= ldexp(1.0, 128))
        return (uint16_t)(sign | 0x7F80u);
    float rf = (float)r;                               /* exact: r is on the bf16 grid */
    uint32_t rb;
    memcpy(&rb, &rf, 4);
    return (uint16_t)(sign | (rb >> 16));
}

/* start block of the subspace iteration: a 64-bit linear congruential
 * sequence (Knuth's MMIX multiplier and increment), top 53 bits as a uniform
 * value in [-1, 1) */
static double lcg_uniform(uint64_t *s)
{
    *s = *s * 6364136223846793005ull + 1442695040888963407ull;
    return (double)(*s >> 11) * ldexp(1.0, -52) - 1.0;
}

static double dot_f64(const double *a, const double *b, int64_t n)
{
    double s = 0.0;
    for (int64_t i = 0; i < n; i++)
        s += a[i] * b[i];
    return s;
}

/*
 * Orthonormalise the p vectors (each `len` long, stored one after another) by
 * modified Gram-Schmidt, applied twice.  A vector that has (next to) nothing
 * left after the projections is replaced by a fresh start vector and
 * projected again, so the result always has p orthonormal columns.
 */
static void orthonormalise(double *A, int64_t len, int p, uint64_t *seed)
{
    for (int j = 0; j < p; j++) {
        double *a = A + (int64_t)j * len;
        for (int attempt = 0; attempt < 4; attempt++) {
            double before = sqrt(dot_f64(a, a, len));
            for (int pass = 0; pass < 2; pass++)
                for (int i = 0; i < j; i++) {
                    const double *q = A + (int64_t)i * len;
                    double c = dot_f64(q, a, len);
                    for (int64_t t = 0; t < len; t++)
                        a[t] -= c * q[t];
                }
            double nrm = sqrt(dot_f64(a, a, len));
            if (nrm > 0.0 && nrm > 1e-10 * before) {
                for (int64_t t = 0; t < len; t++)
                    a[t] /= nrm;
                break;
            }
            for (int64_t t = 0; t < len; t++)
                a[t] = lcg_uniform(seed);
        }
    }
}

/*
 * One-sided Jacobi (Hestenes): rotate pairs of the p columns of B (each `len`
 * long, stored one after another) until every pair is orthogonal to within
 * tol, applying the same rotations to the columns of J (p x p, starts as I).
 * A pair (i, j) with a_ii = |b_i|^2, a_jj = |b_j|^2, a_ij = b_i . b_j is
 * rotated by the angle that zeroes a_ij: zeta = (a_jj - a_ii) / (2 a_ij),
 * t = sign(zeta) / (|zeta| + sqrt(1 + zeta^2)), c = 1 / sqrt(1 + t^2), s = c t,
 * b_i <- c b_i - s b_j, b_j <- s b_i + c b_j.  Pairs are visited row by row.
 */
static void jacobi_onesided(double *B, int64_t len, int p, double *J, double tol)
{
    for (int sweep = 0; sweep < 100; sweep++) {
        int rotated = 0;
        for (int i = 0; i < p - 1; i++)
            for (int j = i + 1; j < p; j++) {
                double *bi = B + (int64_t)i * len, *bj = B + (int64_t)j * len;
                double aii = dot_f64(bi, bi, len), ajj = dot_f64(bj, bj, len), aij = dot_f64(bi, bj, len);
                if (aii == 0.0 || ajj == 0.0 || fabs(aij) <= tol * sqrt(aii * ajj))
                    continue;
                double zeta = (ajj - aii) / (2.0 * aij);
                double t = copysign(1.0, zeta) / (fabs(zeta) + sqrt(1.0 + zeta * zeta));
                double c = 1.0 / sqrt(1.0 + t * t), s = c * t;
                for (int64_t e = 0; e < len; e++) {
                    double x = bi[e], y = bj[e];
                    bi[e] = c * x - s * y;
                    bj[e] = s * x + c * y;
                }
                double *ji = J + (int64_t)i * p, *jj = J + (int64_t)j * p;
                for (int e = 0; e < p; e++) {
                    double x = ji[e], y = jj[e];
                    ji[e] = c * x - s * y;
                    jj[e] = s * x + c * y;
                }
                rotated++;
            }
        if (!rotated)
            return;
    }
}

/* Z[j][n] = sum_k W[n][k] V[j][k]  (vectors V[j] of length K, Z[j] of length N) */
static void mul_w(const float *W, int64_t N, int64_t K, const double *V, int p, double *Z)
{
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++)
        for (int j = 0; j < p; j++) {
            const float *w = W + n * K;
            const double *v = V + (int64_t)j * K;
            double s = 0.0;
            for (int64_t k = 0; k < K; k++)
                s += (double)w[k] * v[k];
            Z[(int64_t)j * N + n] = s;
        }
}

/* Y[j][k] = sum_n W[n][k] U[j][n], each sum taken over n in order */
static void mul_wt(const float *W, int64_t N, int64_t K, const double *U, int p, double *Y)
{
    const int64_t kblk = 256;
#pragma omp parallel for schedule(static)
    for (int64_t k0 = 0; k0 < K; k0 += kblk) {
        int64_t k1 = k0 + kblk < K ? k0 + kblk : K;
        for (int j = 0; j < p; j++)
            for (int64_t k = k0; k < k1; k++)
                Y[(int64_t)j * K + k] = 0.0;
        for (int64_t n = 0; n < N; n++) {
            const float *w = W + n * K;
            for (int j = 0; j < p; j++) {
                double u = U[(int64_t)j * N + n];
                double *y = Y + (int64_t)j * K;
                for (int64_t k = k0; k < k1; k++)
                    y[k] += (double)w[k] * u;
            }
        }
    }
}

/*
 * Leading singular triplets of W [N, K] fp32 (SquareQ README, "Low-rank
 * branch" paragraph: the branch is taken from the weight's SVD).  Block
 * subspace iteration in fp64 with p = min(64, N, K) vectors:
 *     V <- orthonormal start block [K, p]
 *     repeat:  B = W V;  one-sided Jacobi on B's columns (B J = U S, the
 *              Rayleigh-Ritz step: the SVD of W restricted to span V);
 *              U = B J / S, V <- V J, sorted by S descending;
 *              Y = W^T U;  stop when |y_i - s_i v_i| <= 1e-13 s_0 for every
 *              i < rank (the triplets are singular triplets of W to that
 *              residual);  else V <- orthonormalised Y.
 * With p = min(N, K) one step spans W's whole row space, so the result is
 * the full SVD's leading part.  Outputs: sigma[rank] descending, u [N, rank]
 * and v [K, rank] (row-major), each pair's sign fixed so that its largest |v|
 * entry (first one on a tie) is positive.  Returns the number of iterations.
 */
int or_svd_top(const float *W, int64_t N, int64_t K, int rank, int max_iter, double *sigma, double *u_out,
               double *v_out)
{
    int p = 64;
    if (p > N)
        p = (int)N;
    if (p > K)
        p = (int)K;
    const int stride = rank;                /* row stride of u_out, v_out */
    if (rank > p)
        rank = p;                           /* triplets beyond min(N, K) are zero */
    double *V = (double *)malloc(sizeof(double) * (size_t)(K * p));
    double *B = (double *)malloc(sizeof(double) * (size_t)(N * p));
    double *Y = (double *)malloc(sizeof(double) * (size_t)(K * p));
    double *J = (double *)malloc(sizeof(double) * (size_t)(p * p));
    double *VJ = (double *)malloc(sizeof(double) * (size_t)(K * p));
    double *S = (double *)malloc(sizeof(double) * (size_t)p);
    int *ord = (int *)malloc(sizeof(int) * (size_t)p);
    uint64_t seed = 0x5EEDull;
    for (int64_t i = 0; i < K * p; i++)
        V[i] = lcg_uniform(&seed);
    orthonormalise(V, K, p, &seed);
    const double jtol = 1e-15 * sqrt((double)N);
    int it;
    for (it = 1;; it++) {
        mul_w(W, N, K, V, p, B);
        for (int i = 0; i < p * p; i++)
            J[i] = (i / p == i % p) ? 1.0 : 0.0;
        jacobi_onesided(B, N, p, J, jtol);
        /* V J, column norms of B J, U = B J / S (stored back into B) */
        for (int j = 0; j < p; j++) {
            double *vj = VJ + (int64_t)j * K;
            for (int64_t k = 0; k < K; k++) {
                double s = 0.0;
                for (int i = 0; i < p; i++)
                    s += V[(int64_t)i * K + k] * J[(int64_t)j * p + i];
                vj[k] = s;
            }
            double *b = B + (int64_t)j * N;
            S[j] = sqrt(dot_f64(b, b, N));
            for (int64_t n = 0; n < N; n++)
                b[n] = S[j] > 0.0 ? b[n] / S[j] : 0.0;
        }
        /* order by S descending (stable) */
        for (int j = 0; j < p; j++)
            ord[j] = j;
        for (int a = 1; a < p; a++)
            for (int b2 = a; b2 > 0 && S[ord[b2]] > S[ord[b2 - 1]]; b2--) {
                int t = ord[b2];
                ord[b2] = ord[b2 - 1];
                ord[b2 - 1] = t;
            }
        mul_wt(W, N, K, B, p, Y);
        double s0 = S[ord[0]], worst = 0.0;
        for (int i = 0; i < rank; i++) {
            const double *y = Y + (int64_t)ord[i] * K, *vj = VJ + (int64_t)ord[i] * K;
            double r2 = 0.0;
            for (int64_t k = 0; k < K; k++) {
                double d = y[k] - S[ord[i]] * vj[k];
                r2 += d * d;
            }
            if (sqrt(r2) > worst)
                worst = sqrt(r2);
        }
        if (s0 == 0.0 || worst <= 1e-13 * s0 || it >= max_iter)
            break;
        memcpy(V, Y, sizeof(double) * (size_t)(K * p));
        orthonormalise(V, K, p, &seed);
    }
    for (int i = 0; i < rank; i++) {
        const double *ui = B + (int64_t)ord[i] * N, *vi = VJ + (int64_t)ord[i] * K;
        int64_t big = 0;
        for (int64_t k = 1; k < K; k++)
            if (fabs(vi[k]) > fabs(vi[big]))
                big = k;
        double sg = vi[big] < 0.0 ? -1.0 : 1.0;
        sigma[i] = S[ord[i]];
        for (int64_t n = 0; n < N; n++)
            u_out[n * stride + i] = sg * ui[n];
        for (int64_t k = 0; k < K; k++)
            v_out[k * stride + i] = sg * vi[k];
    }
    for (int i = rank; i < stride; i++) {
        sigma[i] = 0.0;
        for (int64_t n = 0; n < N; n++)
            u_out[n * stride + i] = 0.0;
        for (int64_t k = 0; k < K; k++)
            v_out[k * stride + i] = 0.0;
    }
    free(V);
    free(B);
    free(Y);
    free(J);
    free(VJ);
    free(S);
    free(ord);
    return it;
}

/*
 * SVD init of the low-rank branch: the leading 32 singular triplets
 * (or_svd_top), of which the first `rank` (32, or 16 for the int8 mode's
 * branch: its 16 leading pairs) make the factors, the singular values split
 * evenly between them,
 *     up[n, i] = bf16(u[n, i] sqrt(sigma_i)),  down[k, i] = bf16(v[k, i] sqrt(sigma_i)),
 * each rounded from fp64 to bf16 once, and R = RN(W - L) with L the
 * reconstruct's fmaf chain over the rank (or_svd_residual).  Returns the
 * iteration count.
 */
int or_svd_init(const float *W, int64_t N, int64_t K, int rank, int max_iter, uint16_t *up, uint16_t *down,
                float *R, double *sigma)
{
    double *u = (double *)malloc(sizeof(double) * (size_t)(N * 32));
    double *v = (double *)malloc(sizeof(double) * (size_t)(K * 32));
    double s32[32];
    int it = or_svd_top(W, N, K, 32, max_iter, s32, u, v);
    for (int i = 0; i < rank; i++) {
        sigma[i] = s32[i];
        double rs = sqrt(sigma[i]);
        for (int64_t n = 0; n < N; n++)
            up[n * rank + i] = or_f64_to_bf16(u[n * 32 + i] * rs);
        for (int64_t k = 0; k < K; k++)
            down[k * rank + i] = or_f64_to_bf16(v[k * 32 + i] * rs);
    }
    free(u);
    free(v);
    or_svd_residual(W, up, down, N, K, rank, R);
    return it;
}
