// sq_device.cuh -- device helpers shared by the libsq kernels (sm_100a).
//
// Rounding discipline: every fp32 operation that feeds an integer or packed
// output uses the explicit round-to-nearest intrinsics (__fadd_rn, __fmul_rn,
// __fdiv_rn, __frcp_rn, ...), so the compiler cannot contract or reorder it,
// and the result is the IEEE result of the operation sequence stated in sq.h.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace sq {

constexpr int kRank = 32;          // low-rank branch rank
constexpr int kHad = 256;          // Hadamard block size over K
constexpr int kSfBlock = 16;       // NVFP4 values per ue4m3 scale
constexpr int kGroup = 32;         // int4 values per fp16 scale
constexpr int kFracCount = 26;     // int4 scale fractions 0.50, 0.52, ..., 1.00

// device status word bits (first word of every workspace)
constexpr uint32_t kStatusTimeout = 1u;      // a bounded wait gave up
constexpr uint32_t kStatusNonfinite = 2u;    // the SQ_CHECK_FINITE scan met a NaN or an infinity
constexpr uint32_t kStatusIndex = 4u;        // a device-side index check failed (the access was skipped)

// Device-side index check: true if ok; otherwise sets kStatusIndex in *status
// (when non-NULL) and returns false so the caller skips the access.  Kernels
// call it through SQ_DCHECK, which is the check itself in a build with
// SQ_DEBUG_CHECKS and the constant true otherwise.
__device__ __forceinline__ bool dcheck(bool ok, uint32_t *status)
{
    if (!ok && status)
        atomicOr(status, kStatusIndex);
    return ok;
}

#ifdef SQ_DEBUG_CHECKS
#define SQ_DCHECK(cond, status) (::sq::dcheck((cond), (status)))
#else
#define SQ_DCHECK(cond, status) (true)
#endif

// ---------------------------------------------------------------------------
// Hadamard-256 over one warp.
//
// Layout: lane l holds v[0..3] = elements 4l..4l+3 and v[4..7] = elements
// 128+4l..128+4l+3 of the 256-block, so a warp's loads are contiguous.
// Butterfly stride h pairs element j with j+h when (j & h) == 0; the lower
// element becomes a+b and the upper a-b (a = lower, b = upper), strides in the
// order 1, 2, 4, ..., 128, then a scale by 1/16 (exact).  Strides 1 and 2 and
// 128 pair values inside a lane; strides 4..64 pair lane l with lane l^(h/4).
// Every butterfly has the same two operands whichever lane computes it, so
// the result equals the sequential radix-2 transform bit for bit.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void fwht256_warp(float (&v)[8], int lane)
{
#pragma unroll
    for (int half = 0; half < 8; half += 4) {
        float a0 = v[half + 0], a1 = v[half + 1], a2 = v[half + 2], a3 = v[half + 3];
        // h = 1
        float b0 = __fadd_rn(a0, a1), b1 = __fsub_rn(a0, a1);
        float b2 = __fadd_rn(a2, a3), b3 = __fsub_rn(a2, a3);
        // h = 2
        v[half + 0] = __fadd_rn(b0, b2);
        v[half + 2] = __fsub_rn(b0, b2);
        v[half + 1] = __fadd_rn(b1, b3);
        v[half + 3] = __fsub_rn(b1, b3);
    }
#pragma unroll
    for (int x = 1; x <= 16; x <<= 1) {          // h = 4x
        const float sg = (lane & x) == 0 ? 1.0f : -1.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float p = __shfl_xor_sync(0xffffffffu, v[i], x);
            v[i] = __fmaf_rn(sg, v[i], p);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {                // h = 128
        float a = v[i], b = v[i + 4];
        v[i] = __fadd_rn(a, b);
        v[i + 4] = __fsub_rn(a, b);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
        v[i] = __fmul_rn(v[i], 0.0625f);
}

// ---------------------------------------------------------------------------
// Two fp32 lanes in one 64-bit register (sm_100 packed arithmetic).  Each lane
// of add / sub / mul / fma .rn.f32x2 is rounded once, exactly like the scalar
// instruction, so packed and scalar code give identical bits.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void f2_unpack(uint64_t v, float &lo, float &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b)
{
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b)
{
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b)
{
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

// ---------------------------------------------------------------------------
// Hadamard-256 over 8 lanes.
//
// Layout: lane q = lane % 8 of an aligned group of 8 lanes holds v[0..31] =
// elements 32q..32q+31 of one 256-block (a warp holds 4 blocks).  Strides
// 1..16 pair values inside a lane, strides 32, 64, 128 pair lane q with lane
// q ^ 1, q ^ 2, q ^ 4.  Same butterflies, same operands, same order of
// strides as the sequential transform, so the result is identical bit for bit.
// Strides >= 2 run on packed pairs (v[2j], v[2j+1]).  With SCALE = false the
// final multiply by 1/16 is left to the caller (exact: a power of two).
// ---------------------------------------------------------------------------
template <bool SCALE = true>
__device__ __forceinline__ void fwht256_l32(float (&v)[32], int lane)
{
#pragma unroll
    for (int j = 0; j < 16; ++j) {               // stride 1, inside each pair
        const float a = v[2 * j], b = v[2 * j + 1];
        v[2 * j] = __fadd_rn(a, b);
        v[2 * j + 1] = __fsub_rn(a, b);
    }
    uint64_t p[16];
#pragma unroll
    for (int j = 0; j < 16; ++j)
        p[j] = f2_pack(v[2 * j], v[2 * j + 1]);
#pragma unroll
    for (int hp = 1; hp < 16; hp <<= 1)          // strides 2, 4, 8, 16 = pair strides 1..8
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if ((j & hp) == 0) {
                const uint64_t a = p[j], b = p[j + hp];
                p[j] = f2_add(a, b);
                p[j + hp] = f2_sub(a, b);
            }
#pragma unroll
    for (int x = 1; x <= 4; x <<= 1) {          // strides 32x, across lanes
        // lower lane: p + v, upper lane: p - v, as one fma with +-1 (same single rounding)
        const float sg = (lane & x) == 0 ? 1.0f : -1.0f;
        const uint64_t sg2 = f2_pack(sg, sg);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            float lo, hi;
            f2_unpack(p[j], lo, hi);
            const uint64_t o = f2_pack(__shfl_xor_sync(0xffffffffu, lo, x), __shfl_xor_sync(0xffffffffu, hi, x));
            p[j] = f2_fma(sg2, p[j], o);
        }
    }
    if (SCALE) {
        const uint64_t sc = f2_pack(0.0625f, 0.0625f);
#pragma unroll
        for (int j = 0; j < 16; ++j)
            p[j] = f2_mul(p[j], sc);
    }
#pragma unroll
    for (int j = 0; j < 16; ++j)
        f2_unpack(p[j], v[2 * j], v[2 * j + 1]);
}

// ---------------------------------------------------------------------------
// Hadamard-256 over 8 lanes, strided layout, without the final 1/16.
//
// Lane q = lane % 8 of an aligned group of 8 lanes holds v[8b + j] = element
// 64b + 8q + j of one 256-block (b = 0..3, j = 0..7): every 16-byte piece of a
// row it reads is a different bank slot for the 8 lanes.  Strides 1, 2, 4 pair
// values inside a lane, strides 8, 16, 32 pair lane q with q ^ 1, q ^ 2, q ^ 4,
// strides 64, 128 pair values inside a lane again: the sequential order of
// strides with the same operands, so every element is identical bit for bit to
// the sequential transform (before its 1/16).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void fwht256_l32s_unscaled(float (&v)[32], int lane)
{
#pragma unroll
    for (int j = 0; j < 16; ++j) {               // stride 1, inside each pair
        const float a = v[2 * j], b = v[2 * j + 1];
        v[2 * j] = __fadd_rn(a, b);
        v[2 * j + 1] = __fsub_rn(a, b);
    }
    uint64_t p[16];                              // p[4b + j/2] = (v[8b + j], v[8b + j + 1]), j even
#pragma unroll
    for (int j = 0; j < 16; ++j)
        p[j] = f2_pack(v[2 * j], v[2 * j + 1]);
#pragma unroll
    for (int hp = 1; hp <= 2; hp <<= 1)          // strides 2, 4
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if ((j & hp) == 0) {
                const uint64_t a = p[j], b = p[j + hp];
                p[j] = f2_add(a, b);
                p[j + hp] = f2_sub(a, b);
            }
#pragma unroll
    for (int x = 1; x <= 4; x <<= 1) {           // strides 8, 16, 32, across lanes
        const float sg = (lane & x) == 0 ? 1.0f : -1.0f;
        const uint64_t sg2 = f2_pack(sg, sg);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            float lo, hi;
            f2_unpack(p[j], lo, hi);
            const uint64_t o = f2_pack(__shfl_xor_sync(0xffffffffu, lo, x), __shfl_xor_sync(0xffffffffu, hi, x));
            p[j] = f2_fma(sg2, p[j], o);
        }
    }
#pragma unroll
    for (int hp = 4; hp <= 8; hp <<= 1)          // strides 64, 128
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if ((j & hp) == 0) {
                const uint64_t a = p[j], b = p[j + hp];
                p[j] = f2_add(a, b);
                p[j + hp] = f2_sub(a, b);
            }
#pragma unroll
    for (int j = 0; j < 16; ++j)
        f2_unpack(p[j], v[2 * j], v[2 * j + 1]);
}

// ---------------------------------------------------------------------------
// Hadamard-256 over 4 lanes, without the final 1/16 (fwht256_q4_from_s2: the
// strides from 2 on, for pairs whose stride-1 butterfly is done).
//
// Layout: the four quarters q = 0..3 of a 256-block sit in lanes 8q + r of a
// warp (r = 0..7 picks one of eight blocks), and quarter q holds elements
// 64q .. 64q+63 as pairs p[j] = (v[2j], v[2j+1]).  Stride 1 pairs the two
// values of a pair, strides 2 .. 32 pair whole pairs inside the lane (packed
// f32x2 arithmetic), strides 64 and 128 pair lane q with lane q ^ 1 (lane ^ 8)
// and q ^ 2 (lane ^ 16).  The same butterflies with the same operands in the
// same order of strides as the sequential transform, so every element equals
// the sequential result (before its 1/16) bit for bit.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void fwht256_q4_from_s2(uint64_t (&p)[32], int lane)
{
#pragma unroll
    for (int hp = 1; hp <= 16; hp <<= 1)          // strides 2 .. 32
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if ((j & hp) == 0) {
                const uint64_t a = p[j], b = p[j + hp];
                p[j] = f2_add(a, b);
                p[j + hp] = f2_sub(a, b);
            }
#pragma unroll
    for (int x = 8; x <= 16; x <<= 1) {           // strides 64, 128, across lanes
        // lower lane: own + partner, upper lane: partner - own, one fma with +-1 each
        const float sg = (lane & x) == 0 ? 1.0f : -1.0f;
        const uint64_t sg2 = f2_pack(sg, sg);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            float lo, hi;
            f2_unpack(p[j], lo, hi);
            const uint64_t o = f2_pack(__shfl_xor_sync(0xffffffffu, lo, x), __shfl_xor_sync(0xffffffffu, hi, x));
            p[j] = f2_fma(sg2, p[j], o);
        }
    }
}

__device__ __forceinline__ void fwht256_q4_unscaled(uint64_t (&p)[32], int lane)
{
#pragma unroll
    for (int j = 0; j < 32; ++j) {               // stride 1, inside each pair
        float a, b;
        f2_unpack(p[j], a, b);
        p[j] = f2_pack(__fadd_rn(a, b), __fsub_rn(a, b));
    }
    fwht256_q4_from_s2(p, lane);
}

// 64 bf16 values (one 128-byte row R of a box of 64 columns stored with the
// 128-byte swizzle: 16-byte piece i of the row at i ^ (R % 8)) as fp32 pairs.
// Eight lanes reading the same piece of eight consecutive rows hit eight
// different bank groups.
__device__ __forceinline__ void load_row64_bf16_sw128(const uint8_t *box, int R, uint64_t (&p)[32])
{
    const uint8_t *row = box + R * 128;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint4 a = *reinterpret_cast<const uint4 *>(row + 16 * (i ^ (R & 7)));
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
            p[4 * i + j] = f2_pack(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xFFFF0000u));
    }
}

// The same row with the stride-1 butterfly folded into the widening (mixed
// bf16 / fp32 arithmetic, one rounding each, like the fp32 butterfly on the
// exactly widened values): pair j becomes (RN(v[2j] + v[2j+1]),
// RN(v[2j] - v[2j+1])), the difference as fma(v[2j+1], -1, v[2j]) -- the same
// bits as the fp32 subtraction, zero signs included.
__device__ __forceinline__ void load_row64_bf16_sw128_s1(const uint8_t *box, int R, uint64_t (&p)[32])
{
    const uint8_t *row = box + R * 128;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint4 a = *reinterpret_cast<const uint4 *>(row + 16 * (i ^ (R & 7)));
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float lo = __uint_as_float(w[j] << 16);
            float sum, diff;
            asm("{\n\t.reg .b16 h0, h1, m1;\n\tmov.b32 {h0, h1}, %2;\n\tmov.b16 m1, 0xBF80;\n\t"
                "add.rn.f32.bf16 %0, h1, %3;\n\t"
                "fma.rn.f32.bf16 %1, h1, m1, %3;\n\t}"
                : "=f"(sum), "=f"(diff) : "r"(w[j]), "f"(lo));
            p[4 * i + j] = f2_pack(sum, diff);
        }
    }
}

// max(a, b, c) in one instruction (sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// 32 consecutive values into registers (fp32 source or bf16 bit patterns)
__device__ __forceinline__ void load32(const float *p, float (&v)[32])
{
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(p) + i);
        v[4 * i] = a.x; v[4 * i + 1] = a.y; v[4 * i + 2] = a.z; v[4 * i + 3] = a.w;
    }
}

__device__ __forceinline__ void load32(const uint16_t *p, float (&v)[32])
{
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 a = __ldg(reinterpret_cast<const uint4 *>(p) + i);
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
            v[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
    }
}

// ---------------------------------------------------------------------------
// Narrowing conversions (PTX cvt, round-to-nearest-even, satfinite).
// ---------------------------------------------------------------------------

// ue4m3 code of a non-negative value (e4m3 with sign 0; saturates at 448).
__device__ __forceinline__ uint32_t to_ue4m3(float v)
{
    uint16_t packed;   // upper byte <- first source, lower byte <- second source
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(packed) : "f"(0.0f), "f"(v));
    return (uint32_t)packed & 0xFFu;
}

// value of a ue4m3 code (exact through fp16)
__device__ __forceinline__ float ue4m3_value(uint32_t code)
{
    uint32_t h2;
    uint16_t in = (uint16_t)(code & 0xFFu);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// e2m1 magnitude codes of two non-negative values, packed lo | hi << 4.
__device__ __forceinline__ uint32_t to_e2m1x2_mag(float lo, float hi)
{
    uint32_t out;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
        "cvt.u32.u8 %0, t;\n\t}"
        : "=r"(out) : "f"(hi), "f"(lo));
    return out;
}

// e2m1 codes of two values with their sign bits kept (negative -> bit 3 set,
// including values that round to zero), packed lo | hi << 4.  The signed
// conversion keeps the sign of a negative value that rounds to zero (checked
// against the magnitude conversion plus explicit sign bits).
__device__ __forceinline__ uint32_t to_e2m1x2(float lo, float hi)
{
    return to_e2m1x2_mag(lo, hi);
}

// e2m1 codes of four values, packed a | b << 4 | c << 8 | d << 12
__device__ __forceinline__ uint32_t to_e2m1x4(float a, float b, float c, float d)
{
    uint16_t out;
    asm("{\n\t.reg .b8 t0, t1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t1, %4, %3;\n\t"
        "mov.b16 %0, {t0, t1};\n\t}"
        : "=h"(out) : "f"(a), "f"(b), "f"(c), "f"(d));
    return out;
}

// values of two e2m1 codes held in one byte (low nibble first), exact
__device__ __forceinline__ float2 e2m1x2_value(uint32_t byte)
{
    uint32_t h2;
    uint16_t in = (uint16_t)(byte & 0xFFu);
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.u8.u16 t, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
        : "=r"(h2) : "h"(in));
    __half2 h = *reinterpret_cast<__half2 *>(&h2);
    return __half22float2(h);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t bits16)
{
    return __uint_as_float(bits16 << 16);
}

__device__ __forceinline__ uint32_t f32_to_bf16_bits(float v)
{
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// bf16(lo) | bf16(hi) << 16, both round to nearest even, in one conversion
// instruction (cvt.rn.bf16x2.f32 puts its first source in the upper half)
__device__ __forceinline__ uint32_t f32x2_to_bf16x2_bits(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Integer codes to exact floats without the int-to-float conversion unit:
// 2^23 + u (0 <= u < 2^23) is the float whose bit pattern is 0x4B000000 | u,
// so a small integer is recovered by one exact subtraction.
//   int4 (4-bit two's complement nibble n):  q = (n ^ 8) - 8
//   int8 (byte b, two's complement):         q = (b ^ 0x80) - 128
// v[i] = q of nibble i of w (nibble 0 = low bits)
__device__ __forceinline__ void int4x8_to_f32(uint32_t w, float (&v)[8])
{
    const uint32_t x = w ^ 0x88888888u;
#pragma unroll
    for (int i = 0; i < 8; ++i)
        v[i] = __fsub_rn(__uint_as_float(0x4B000000u | ((x >> (4 * i)) & 0xFu)), 8388616.0f);
}

// v[i] = q of byte i of w (byte 0 = low bits)
__device__ __forceinline__ void int8x4_to_f32(uint32_t w, float (&v)[4])
{
    const uint32_t x = w ^ 0x80808080u;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        v[i] = __fsub_rn(__uint_as_float(__byte_perm(x, 0x4B000000u, 0x7650u + i)), 8388736.0f);
}

// tiled scale-factor byte offset, C = K/16 scale columns
__device__ __forceinline__ int64_t sf_offset(int64_t r, int64_t c, int64_t C)
{
    return ((r >> 7) * (C >> 2) + (c >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (c & 3);
}

// non-negative float max through its bit pattern (for atomicMax on u32)
__device__ __forceinline__ void atomic_max_nonneg(uint32_t *addr, float v)
{
    atomicMax(addr, __float_as_uint(v));
}

}  // namespace sq
