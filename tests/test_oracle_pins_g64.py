"""Pins of the oracle's int4 group-64 codec (SquareQ README, "Residual codecs"
paragraph: int4 scales per group of 32 or 64 values, the fraction chosen by MSE).

Reading pinned here: the same 26-fraction sweep as group 32 over 64 values
(a = max over all 64), with the squared-error sum taken as the group-32 xor
butterfly of each 32-value half, then first half + second half.
"""
import numpy as np

import synth_inputs as si


def _fp16(v):
    return float(np.float16(v))


def test_g64_bruteforce_fraction_is_minimal(oracle_mod):
    """Exhaustive: all 26 candidate errors in fp64, the pick is minimal up to rounding."""
    rng = np.random.default_rng(64)
    for trial in range(200):
        r = rng.standard_normal(64)
        if trial % 3 == 1:
            r[rng.integers(0, 64)] *= 8.0
        if trial % 3 == 2:
            r = rng.standard_t(4, 64)
        r = (r * rng.lognormal(-3, 1)).astype(np.float32)
        q, s_bits, j = oracle_mod.int4_group64(r)
        assert q.min() >= -7 and q.max() <= 7
        a = float(np.abs(r).max())
        errs = []
        for jj in range(26):
            f = np.float32((50 + 2 * jj) / 100)
            s = _fp16(np.float32(np.float32(f * np.float32(a)) / np.float32(7)))
            qq = np.clip(np.round(r.astype(np.float64) / s), -7, 7) if s else np.zeros(64)
            errs.append(float(((r.astype(np.float64) - qq * s) ** 2).sum()))
        errs = np.array(errs)
        assert errs[j] <= errs.min() * (1 + 1e-5) + 1e-30
        s_expect = np.float32(np.float32(np.float32(oracle_mod.int4_fraction(j)) * np.float32(a)) / np.float32(7))
        assert s_bits == np.float32(s_expect).astype(np.float16).view(np.uint16)


def test_g64_exact_roundtrip_on_grid(oracle_mod):
    rng = np.random.default_rng(65)
    for _ in range(50):
        s = _fp16(rng.lognormal(-6, 1))
        q = rng.integers(-7, 8, 64)
        q[rng.integers(0, 64)] = 7 * rng.choice([-1, 1])
        r = (q * s).astype(np.float32)
        qo, sb, j = oracle_mod.int4_group64(r)
        assert np.array_equal(qo, q)
        assert float(np.uint16(sb).view(np.float16)) == s
        assert j == 25


def test_g64_ties_go_to_smaller_fraction(oracle_mod):
    # all-zero group: every fraction has zero error -> j = 0, s = 0
    q, s, j = oracle_mod.int4_group64(np.zeros(64, np.float32))
    assert j == 0 and s == 0 and not q.any()
    # a = 7 * 2^-24: j = 0 (f = 0.5) rounds the scale to fp16 0 (error = sum r^2); every j >= 1
    # gives s = 2^-24 (fp16 bits 0x0001) and zero error, a 25-way tie -> the smallest, j = 1
    r = np.full(64, 7 * 2.0 ** -24, np.float32)
    q, s, j = oracle_mod.int4_group64(r)
    assert j == 1 and s == 1 and np.all(q == 7)


def test_g64_of_two_equal_halves_is_g32(oracle_mod):
    """Two copies of a group-32 input: same max, every candidate error exactly doubles
    (the two half sums are equal, and x + x is exact), so the same scale, fraction and
    codes must come out -- pins the half-sum reading against the group-32 codec."""
    rng = np.random.default_rng(66)
    for _ in range(100):
        h = (rng.standard_normal(32) * rng.lognormal(-3, 1)).astype(np.float32)
        q32, s32, j32 = oracle_mod.int4_group32(h)
        q64, s64, j64 = oracle_mod.int4_group64(np.concatenate([h, h]))
        assert (s64, j64) == (s32, j32)
        assert np.array_equal(q64, np.concatenate([q32, q32]))


def test_g64_builder_layout_and_forward(oracle_mod):
    M, K, N = 16, 512, 128
    d = si.make_inputs(M, K, N, 67)
    codes, scales, frac = oracle_mod.build_int4(d["R"], group=64)
    assert codes.shape == (N, K // 2) and scales.shape == (N, K // 64) and frac.shape == (N, K // 64)
    # the builder runs the group codec on consecutive 64-value groups of the rotated rows
    rot = np.concatenate([oracle_mod.fwht256(d["R"][3, b:b + 256]) for b in range(0, K, 256)])
    for g in range(K // 64):
        q, s, j = oracle_mod.int4_group64(rot[64 * g:64 * g + 64])
        nib = (q & 0xF).astype(np.uint8)
        assert np.array_equal(codes[3, 32 * g:32 * g + 32], nib[0::2] | (nib[1::2] << 4))
        assert scales[3, g] == s and frac[3, g] == j
    # the forward decodes group-64 scales
    xr = oracle_mod.rotate_rows_bf16(d["x"])
    y = oracle_mod.linear_fwd_int4(xr, codes, scales, None, None, M, N, K, group=64)
    nib = np.stack([codes & 0xF, codes >> 4], -1).reshape(N, K).astype(np.int64)
    qd = np.where(nib >= 8, nib - 16, nib)
    s = np.repeat(scales.view(np.float16).astype(np.float64), 64, axis=1)
    wb = si.bf16_bits_to_f32(si.to_bf16_bits((qd * s).astype(np.float32))).astype(np.float64)
    xb = si.bf16_bits_to_f32(si.to_bf16_bits(xr)).astype(np.float64)
    assert np.allclose(y, xb @ wb.T, rtol=1e-12, atol=1e-12 * np.abs(y).max())


def test_g64_reconstruct_decodes_group64_scales(oracle_mod):
    N, K = 2, 512
    rng = np.random.default_rng(68)
    q = rng.integers(-7, 8, (N, K))
    sv = np.array([2.0 ** -5, 2.0 ** -7, 2.0 ** -4, 2.0 ** -6] * 2)      # one per 64-group
    nib = (q & 0xF).astype(np.uint8)
    codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    scales = np.tile(np.float16(sv).view(np.uint16), (N, 1))
    zU = np.zeros((N, 32), np.uint16)
    zD = np.zeros((K, 32), np.uint16)
    W = oracle_mod.reconstruct_bf16(oracle_mod.FMT_INT4_G64, codes, scales, 0.0, zU, zD, N, K,
                                    residual_only=True)
    d = (q * np.repeat(sv, 64)[None, :]).astype(np.float32)
    want = np.stack([np.concatenate([oracle_mod.fwht256(d[n, b:b + 256]) for b in range(0, K, 256)])
                     for n in range(N)])
    assert np.array_equal(W, si.to_bf16_bits(want.astype(np.float32)))
