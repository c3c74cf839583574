"""The int4 dequantisation of the GEMM's W ring, checked on the CPU for every case.

The stand-alone definition is wb = bf16(q s): q in [-8, 7] times the fp16 group scale s, exact
in fp32, rounded once to bf16 (round to nearest even).  The GEMM forms it in bf16x2 arithmetic
(sq_gemm.cu, dq_int4x8).  A byte permute and a mask put the offset code q + 8 under the exponent
of 128, giving the bf16 value 128 + q + 8.  One bf16 subtract of 136 gives q exactly.  With s_hi
= bf16(s) and s_lo = s - s_hi, one bf16 multiply gives c = q s_lo exactly, and one bf16 fma gives
bf16(q s_hi + c).  That last step is the only rounding.  This test emulates each step, every
rounding included, for all 16 codes and every finite non-negative fp16 scale (31744 of them),
and compares with the definition bit for bit, signs of zero included.
"""
import numpy as np


def rn_bf16(x):
    """Round float64 values to bf16 (round to nearest even), returned as float64; exact for the
    magnitudes here (no overflow, no bf16 subnormals)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                         # x = m 2^e, 0.5 <= |m| < 1 (m = 0 for x = 0)
    return np.ldexp(np.round(m * 256.0) / 256.0, e)   # np.round: half to even; keeps -0


def byte_perm(a, b, s):
    """The selector's low three bits of each nibble pick a byte of {b:a}."""
    src = [(a >> (8 * i)) & 0xFF for i in range(4)] + [(b >> (8 * i)) & 0xFF for i in range(4)]
    return sum(src[(s >> (4 * n)) & 7] << (8 * n) for n in range(4))


def bf16_bits_to_f64(h):
    return np.array([h << 16], dtype=np.uint32).view(np.float32).astype(np.float64)[0]


def code_values_as_bf16(w):
    """The device's eight bf16 values 128 + (q + 8) of the code word w, in element order."""
    x = w ^ 0x88888888
    lo, hi = x & 0x0F0F0F0F, (x >> 4) & 0x0F0F0F0F
    out = []
    for j in range(4):
        v = (byte_perm(lo, hi, ((4 + j) << 8) | j) & 0x00FF00FF) | 0x43004300
        out += [bf16_bits_to_f64(v & 0xFFFF), bf16_bits_to_f64(v >> 16)]
    return out


def test_code_extraction_gives_every_offset_code_in_order():
    rng = np.random.default_rng(5)
    for w in list(rng.integers(0, 2**32, size=200, dtype=np.uint64)) + [0, 0xFFFFFFFF, 0x76543210, 0x89ABCDEF]:
        w = int(w)
        got = code_values_as_bf16(w)
        nib = [(w >> (4 * i)) & 0xF for i in range(8)]
        q = [n - 16 if n >= 8 else n for n in nib]
        assert got == [128.0 + qi + 8 for qi in q], hex(w)


def test_split_scale_fma_equals_bf16_of_the_product_for_every_scale():
    s16 = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16)     # +0 .. 65504, subnormals too
    s = s16.astype(np.float64)
    s_hi = rn_bf16(s)
    s_lo = s - s_hi
    assert np.array_equal(rn_bf16(s_lo), s_lo)                        # s_lo is a bf16 value
    for q in range(-8, 8):
        v = 128.0 + q + 8                                            # the extracted code, exact
        qq = rn_bf16(v - 136.0)                                      # bf16 subtract
        assert qq == q
        c = rn_bf16(qq * s_lo)                                       # bf16 multiply
        assert np.array_equal(c, qq * s_lo)                           # exact
        got = rn_bf16(qq * s_hi + c)                                  # bf16 fma: one rounding
        want = rn_bf16(np.float32(q) * s16.astype(np.float32))         # bf16(q s), q s exact in fp32
        assert np.array_equal(got, want), f"q = {q}"
        assert np.array_equal(np.signbit(got), np.signbit(want)), f"q = {q}: sign of zero"
