"""Pins of the oracle's SVD init of the low-rank branch (SquareQ README, "Low-rank
branch" paragraph: a rank-32 bf16 branch taken from the weight's SVD).

Readings pinned here: the rank-32 truncated SVD, singular values split evenly between
the factors (up = U sqrt(sigma), down = V sqrt(sigma), each rounded to bf16 once), and
the residual R = RN(W - L) with L the reconstruct's rank-32 fmaf chain, so that the
layer's own reconstruct of an exact residual gives back W.
"""
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
