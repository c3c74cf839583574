"""Pins of the oracle's SVD init of the low-rank branch (SquareQ README, "Low-rank
branch" paragraph: a rank-32 bf16 branch taken from the weight's SVD).

Readings pinned here: the rank-32 truncated SVD, singular values split evenly between
the factors (up = U sqrt(sigma), down = V sqrt(sigma), each rounded from fp64 to bf16
once), and the residual R = RN(W - L) with L the reconstruct's rank-32 fmaf chain, so that
the layer's own reconstruct of an exact residual gives back W.  The oracle computes the
SVD itself in scalar C (subspace iteration with a one-sided Jacobi step); numpy's LAPACK
SVD appears here only as the independent reference it is checked against.
"""
import math
from fractions import Fraction

import numpy as np

import synth_inputs as si


def lowrank_weight(N, K, seed, scale=4.0):
    """A weight with a clear rank-32 part: scale * U D^T (config factors) + R."""
    d = si.make_inputs(4, K, N, seed)
    U = si.bf16_bits_to_f32(d["U"]).astype(np.float64)
    D = si.bf16_bits_to_f32(d["D"]).astype(np.float64)
    return (scale * U @ D.T + d["R"]).astype(np.float32)


def test_svd_init_decomposition_is_exact(oracle_mod):
    """W - R equals the fmaf chain of the bf16 factors, value by value (the subtraction is
    the only rounding), and R + L reproduces W within one rounding of R."""
    W = lowrank_weight(256, 512, 90)
    up, down, R, S = oracle_mod.svd_init(W)
    U = si.bf16_bits_to_f32(up).astype(np.float64)
    D = si.bf16_bits_to_f32(down).astype(np.float64)
    L = U @ D.T
    back = R.astype(np.float64) + L
    assert np.abs(back - W).max() <= 2.0 ** -23 * np.abs(W).max() * 4
    # residual of the fmaf chain vs the fp64 dot: within the chain's rounding
    bound = 32 * 2.0 ** -24 * (np.abs(U) @ np.abs(D).T) + 2.0 ** -24 * np.abs(W)
    assert np.all(np.abs((W.astype(np.float64) - R) - L) <= bound + 1e-30)


def test_svd_init_is_eckart_young(oracle_mod):
    """||R||_F equals the tail energy sqrt(sum_{i>32} sigma_i^2) up to the bf16 rounding of the
    factors, and the split is even: ||up[:, i]|| = ||down[:, i]|| = sqrt(sigma_i)."""
    W = lowrank_weight(192, 768, 91)
    up, down, R, S = oracle_mod.svd_init(W)
    sig = np.linalg.svd(W.astype(np.float64), compute_uv=False)
    tail = np.sqrt((sig[32:] ** 2).sum())
    assert np.allclose(S, sig[:32], rtol=1e-12)
    rn = np.linalg.norm(R.astype(np.float64))
    L = si.bf16_bits_to_f32(up).astype(np.float64) @ si.bf16_bits_to_f32(down).astype(np.float64).T
    assert rn >= tail * (1 - 1e-9)
    assert rn <= np.sqrt(tail ** 2 + (2 * 2.0 ** -8 * np.linalg.norm(L)) ** 2)
    cu = np.linalg.norm(si.bf16_bits_to_f32(up).astype(np.float64), axis=0)
    cd = np.linalg.norm(si.bf16_bits_to_f32(down).astype(np.float64), axis=0)
    assert np.allclose(cu, np.sqrt(S), rtol=4e-3) and np.allclose(cd, np.sqrt(S), rtol=4e-3)


def test_svd_init_exact_rank_32(oracle_mod):
    """A weight of rank <= 32 leaves only the factors' bf16 rounding in R."""
    rng = np.random.default_rng(92)
    A = rng.standard_normal((128, 32))
    B = rng.standard_normal((512, 32))
    W = (A @ B.T / 10).astype(np.float32)
    up, down, R, S = oracle_mod.svd_init(W)
    assert np.linalg.norm(R) <= 2 * 2.0 ** -8 * np.linalg.norm(W)
    assert np.linalg.norm(R) >= 1e-6 * np.linalg.norm(W)      # the bf16 rounding is there


def test_svd_init_rank16_is_the_int8_modes_branch(oracle_mod):
    """Rank 16 (the int8 mode's branch): the factors are the first 16 columns of the rank-32
    factors (the same singular pairs), the residual's tail energy is that beyond sigma_16, and
    W - R is the rank-16 fmaf chain that the int8 reconstruct adds back."""
    W = lowrank_weight(192, 512, 94)
    up32, down32, _, S32 = oracle_mod.svd_init(W)
    up, down, R, S = oracle_mod.svd_init(W, rank=16)
    assert up.shape == (192, 16) and down.shape == (512, 16)
    assert np.array_equal(up, up32[:, :16]) and np.array_equal(down, down32[:, :16])
    assert np.array_equal(S, S32[:16])
    sig = np.linalg.svd(W.astype(np.float64), compute_uv=False)
    tail = np.sqrt((sig[16:] ** 2).sum())
    U = si.bf16_bits_to_f32(up).astype(np.float64)
    D = si.bf16_bits_to_f32(down).astype(np.float64)
    L = U @ D.T
    rn = np.linalg.norm(R.astype(np.float64))
    assert rn >= tail * (1 - 1e-9)
    assert rn <= np.sqrt(tail ** 2 + (2 * 2.0 ** -8 * np.linalg.norm(L)) ** 2)
    bound = 16 * 2.0 ** -24 * (np.abs(U) @ np.abs(D).T) + 2.0 ** -24 * np.abs(W)
    assert np.all(np.abs((W.astype(np.float64) - R) - L) <= bound + 1e-30)
    # the chain is the int8 reconstruct's: the residual of a zero weight is -L exactly, and zero
    # codes reconstruct to bf16(L), bit for bit
    R0 = oracle_mod.svd_residual(np.zeros((192, 512), np.float32), up, down)
    Wz = oracle_mod.reconstruct_bf16(oracle_mod.FMT_INT8_ROW, np.zeros((192, 512), np.int8),
                                     np.zeros(192, np.float32), 0.0, up, down, 192, 512)
    assert np.array_equal(Wz, si.to_bf16_bits(-R0))


def bf16_of_f64_exact(v):
    """bf16 bits of a float64 by exact rational arithmetic: the nearest value of the bf16 grid
    (7 fraction bits, smallest normal 2^-126, spacing 2^-133 below it), ties to the even
    multiple of the spacing, infinity from 2^128 on."""
    if v != v:
        return 0x7FC0 | (0x8000 if math.copysign(1.0, v) < 0 else 0)
    sign = 0x8000 if math.copysign(1.0, v) < 0 else 0
    a = Fraction(abs(v))
    if a == 0:
        return sign
    _, e = math.frexp(abs(v))
    E = max(e - 1, -126)
    q = Fraction(2) ** (E - 7)
    n = a / q
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    val = fl * q
    if val >= Fraction(2) ** 128:
        return sign | 0x7F80
    return sign | int(np.array([float(val)], np.float32).view(np.uint32)[0] >> 16)


def test_f64_to_bf16_rounds_once(oracle_mod):
    """The fp64 -> bf16 conversion of the factors is one rounding: a value just above (below) a
    bf16 midpoint goes up (down) even when its fp32 rounding lands on the midpoint itself, where
    a detour through fp32 would round to even instead.  Checked against exact rational rounding
    on those cases, exact midpoints, subnormals, overflow and random doubles."""
    mid = 1.0 + 2.0 ** -8                       # between bf16 1.0 and 1.0078125
    cases = [mid + 2.0 ** -40, mid - 2.0 ** -40, mid, 1.0 + 3 * 2.0 ** -8 - 2.0 ** -41,
             -(mid + 2.0 ** -40), 2.0 ** -130 * (1 + 2.0 ** -30), 2.0 ** -134, 3 * 2.0 ** -134,
             (2 - 2.0 ** -8) * 2.0 ** 127, (2 - 2.0 ** -8) * 2.0 ** 127 * (1 - 2.0 ** -50), 1e300, 0.0, -0.0]
    for v in cases:
        assert oracle_mod.f64_to_bf16(v) == bf16_of_f64_exact(v), v
    assert oracle_mod.f64_to_bf16(mid + 2.0 ** -40) == 0x3F81
    assert oracle_mod.f64_to_bf16(mid - 2.0 ** -40) == 0x3F80
    rng = np.random.default_rng(95)
    for v in rng.standard_normal(3000) * np.exp(rng.uniform(-60, 60, 3000)):
        assert oracle_mod.f64_to_bf16(float(v)) == bf16_of_f64_exact(float(v)), v


def test_svd_init_rounds_factors_once(oracle_mod):
    """A weight whose singular vectors are unit vectors (a scaled partial permutation), so the
    factor entries are sqrt(sigma) exactly.  sigma = 1 + 2^-7 + 2^-16 + 2^-23 has
    sqrt(sigma) = 1 + 2^-8 + 0.996 * 2^-24: above the bf16 midpoint 1 + 2^-8, but its fp32
    rounding is that midpoint.  Rounded once the entry is bf16 1 + 2^-7 (0x3F81); through fp32
    it would be 1.0 (0x3F80)."""
    N, K = 128, 256
    special = 1.0 + 2.0 ** -7 + 2.0 ** -16 + 2.0 ** -23
    assert float(np.float32(special)) == special
    sig = np.concatenate([np.linspace(8.0, 2.0, 31), [special], np.linspace(0.5, 0.1, 8)])
    rows = np.random.default_rng(96).permutation(N)[:40]
    cols = np.random.default_rng(97).permutation(K)[:40]
    sign = np.where(np.arange(40) % 3 == 0, -1.0, 1.0)
    W = np.zeros((N, K), np.float32)
    W[rows, cols] = (sig * sign).astype(np.float32)
    up, down, R, S = oracle_mod.svd_init(W)
    i = 31                                       # the special value is the 32nd largest
    assert abs(S[i] / special - 1) <= 1e-14
    assert up[rows[i], i] == 0x3F81 and down[cols[i], i] == 0x3F81
    exact = np.array([bf16_of_f64_exact(math.sqrt(s)) for s in sig[:32]])
    assert np.array_equal(up[rows[:32], np.arange(32)] & 0x7FFF, exact)
    assert np.array_equal(down[cols[:32], np.arange(32)] & 0x7FFF, exact)
