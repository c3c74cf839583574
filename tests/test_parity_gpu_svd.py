"""SVD init of the rank-32 low-rank branch (SquareQ README, "Low-rank branch"
paragraph) through the C ABI against the CPU oracle.

The oracle takes the truncated SVD in scalar C (fp64 subspace iteration run to a 1e-13
residual, one-sided Jacobi Rayleigh-Ritz steps); the GPU runs 8 rounds of subspace
iteration from a seeded start block.  The test weights have a spectral gap at 32
(sigma_32 / sigma_33 >= 3, checked), so the rank-32 product L = up down^T is unique
and the iteration error, (sigma_33 / sigma_32)^(2 iters) <= 3^-16, is negligible.
Compared:
- L against the oracle's within ||dL||_F / ||L||_F <= 2 * 2^-9: each factor is rounded
  to bf16 once (relative error <= 2^-9 per entry), which bounds the difference of two
  correctly rounded factorisations of the same L to first order;
- the residual bit for bit against the oracle's R = RN(W - L) on the GPU's own factors;
- the residual's norm against the optimal one (Eckart-Young).
"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from sqcase import bits16, first_mismatch, host, to_dev

pytestmark = pytest.mark.gpu

L_TOL = 2 * 2.0 ** -9


@pytest.fixture(scope="module")
def sq():
    import bit_quantized_frozen_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    m.lib()
    return m


def gap_weight(N, K, seed):
    """A rank-32 part with singular values 8 .. 2 (geometric) plus the synthetic residual of the
    layer shape scaled to spectral norm 0.5: a gap of about 4 at index 32."""
    rng = np.random.default_rng(seed)
    A = rng.standard_normal((N, 32)) / np.sqrt(N)
    B = rng.standard_normal((K, 32)) / np.sqrt(K)
    s = np.geomspace(8.0, 2.0, 32)
    noise = si.make_inputs(4, K, N, seed)["R"].astype(np.float64)
    noise *= 0.5 / np.linalg.norm(noise, 2)
    W = ((A * s) @ B.T + noise).astype(np.float32)
    S = np.linalg.svd(W.astype(np.float64), compute_uv=False)
    assert S[31] >= 3 * S[32], "test weight without a spectral gap"
    return W


def omega(K, seed):
    return np.random.default_rng(seed).standard_normal((K, 32)).astype(np.float32)


def run_gpu(sq, W, om, iters=8):
    up, down, R = sq.svd_init(to_dev(W), to_dev(om), iters)
    torch.cuda.synchronize()
    return bits16(up), bits16(down), host(R)


def lowrank_product(up, down):
    return si.bf16_bits_to_f32(up).astype(np.float64) @ si.bf16_bits_to_f32(down).astype(np.float64).T


def check_against_oracle(W, up, down, R, rows=None):
    oup, odown, oR, S = oracle.svd_init(W)
    L, Lo = lowrank_product(up, down), lowrank_product(oup, odown)
    err = np.linalg.norm(L - Lo) / np.linalg.norm(Lo)
    assert err <= L_TOL, f"low-rank product differs by {err:.3e}"
    sel = slice(None) if rows is None else rows
    Rw = oracle.svd_residual(W[sel], up[sel], down)
    assert np.array_equal(R[sel].view(np.uint32), Rw.view(np.uint32)), first_mismatch(R[sel], Rw)
    assert np.linalg.norm(R) <= np.linalg.norm(oR) * (1 + 1e-2)


@pytest.mark.parametrize("shape", [(256, 512), (384, 768), (1024, 256)])
def test_svd_init_matches_truncated_svd(sq, shape):
    N, K = shape
    W = gap_weight(N, K, 100 + N)
    up, down, R = run_gpu(sq, W, omega(K, 7))
    check_against_oracle(W, up, down, R)


def test_svd_init_singular_values_split_evenly(sq):
    """up and down carry sigma^(1/2) each: column norms of the factors against the oracle's."""
    W = gap_weight(256, 512, 110)
    up, down, _ = run_gpu(sq, W, omega(512, 11))
    oup, odown, _, S = oracle.svd_init(W)
    for f, o in ((up, oup), (down, odown)):
        n = np.linalg.norm(si.bf16_bits_to_f32(f).astype(np.float64), axis=0)
        no = np.linalg.norm(si.bf16_bits_to_f32(o).astype(np.float64), axis=0)
        assert np.allclose(n, no, rtol=4e-3)
        assert np.allclose(n, np.sqrt(S), rtol=4e-3)


def test_svd_init_is_deterministic_and_exact_rank(sq):
    rng = np.random.default_rng(101)
    W = (rng.standard_normal((256, 32)) @ rng.standard_normal((512, 32)).T / 8).astype(np.float32)
    a = run_gpu(sq, W, omega(512, 8))
    b = run_gpu(sq, W, omega(512, 8))
    for x, y in zip(a, b):
        assert np.array_equal(x.view(np.uint8), y.view(np.uint8))
    up, down, R = a
    assert np.linalg.norm(R) <= 2 * 2.0 ** -8 * np.linalg.norm(W)
    Rw = oracle.svd_residual(W, up, down)
    assert np.array_equal(R.view(np.uint32), Rw.view(np.uint32))


def test_svd_init_ill_conditioned(sq):
    """Singular values 1e4 .. 1 above the gap (the blocks between the products are orthonormalised
    once, the final U twice): the product still matches the truncated SVD."""
    rng = np.random.default_rng(104)
    N, K = 512, 1024
    A = np.linalg.qr(rng.standard_normal((N, 40)))[0]
    B = np.linalg.qr(rng.standard_normal((K, 40)))[0]
    s = np.concatenate([np.geomspace(1e4, 1.0, 32), np.geomspace(0.2, 0.1, 8)])
    W = ((A * s) @ B.T).astype(np.float32)
    up, down, R = run_gpu(sq, W, omega(K, 14))
    oup, odown, _, _ = oracle.svd_init(W)
    L, Lo = lowrank_product(up, down), lowrank_product(oup, odown)
    assert np.linalg.norm(L - Lo) / np.linalg.norm(Lo) <= L_TOL
    Rw = oracle.svd_residual(W, up, down)
    assert np.array_equal(R.view(np.uint32), Rw.view(np.uint32))


def test_svd_init_ragged_gram_partials(sq):
    """N = 640 and K = 1280 are not multiples of the 512-row Gram partials (the last partial of
    each has 128 or 256 rows), and split the products 8 and 4 ways."""
    W = gap_weight(640, 1280, 105)
    up, down, R = run_gpu(sq, W, omega(1280, 15))
    check_against_oracle(W, up, down, R)


def test_svd_init_rounds_converge(sq):
    """iters = 1, 2, 3 from the same start block: the residual is RN(W - L) of the factors bit for
    bit every time, and the distance of L to the truncated SVD shrinks by at least 4x per round
    (subspace iteration contracts by (sigma_33 / sigma_32)^2 <= 1/9 per round on this weight)."""
    W = gap_weight(256, 512, 106)
    oup, odown, _, _ = oracle.svd_init(W)
    Lo = lowrank_product(oup, odown)
    errs = []
    for iters in (1, 2, 3):
        up, down, R = run_gpu(sq, W, omega(512, 16), iters=iters)
        Rw = oracle.svd_residual(W, up, down)
        assert np.array_equal(R.view(np.uint32), Rw.view(np.uint32))
        errs.append(np.linalg.norm(lowrank_product(up, down) - Lo) / np.linalg.norm(Lo))
    assert errs[1] < errs[0] / 4 and errs[2] < errs[1] / 4, errs


def test_svd_init_zero_weight(sq):
    W = np.zeros((128, 256), np.float32)
    up, down, R = run_gpu(sq, W, omega(256, 9), iters=2)
    assert not up.any() and not down.any() and not R.view(np.uint32).any()


def test_svd_init_residual_in_place(sq):
    """R may be the weight's own buffer."""
    W = gap_weight(256, 512, 112)
    Wd = to_dev(W)
    up = torch.empty((256, 32), dtype=torch.bfloat16, device="cuda")
    down = torch.empty((512, 32), dtype=torch.bfloat16, device="cuda")
    ws = sq.workspace(sq.SQ_OP_SVD_INIT, 0, 256, 512)
    sq.sq_svd_init(Wd, to_dev(omega(512, 12)), 8, up, down, Wd, ws)
    torch.cuda.synchronize()
    Rw = oracle.svd_residual(W, bits16(up), bits16(down))
    assert np.array_equal(host(Wd).view(np.uint32), Rw.view(np.uint32))


def test_svd_init_projection_shape(sq):
    W = gap_weight(1536, 3072, 102)
    up, down, R = run_gpu(sq, W, omega(3072, 10))
    check_against_oracle(W, up, down, R, rows=np.array([0, 7, 777, 1535]))


@pytest.mark.slow
def test_svd_init_large(sq):
    W = gap_weight(4096, 2048, 103)
    up, down, R = run_gpu(sq, W, omega(2048, 13))
    check_against_oracle(W, up, down, R, rows=np.array([0, 1, 2048, 4095]))


@pytest.mark.slow
def test_svd_init_bench_shape_properties(sq):
    """The bench workload's full weight W = U D^T + R (16384 x 6144, no spectral gap, 8 rounds):
    properties that hold at any size.  R is RN(W - L) bit for bit on sampled rows; the factors'
    columns are orthogonal with up^T up = down^T down = diag(sigma) in descending order (the even
    split), up to the bf16 rounding of the factors."""
    d = si.make_config("large_4480x16384x6144")
    U = torch.from_numpy(d["U"].view(np.int16)).cuda().view(torch.bfloat16)
    D = torch.from_numpy(d["D"].view(np.int16)).cuda().view(torch.bfloat16)
    W = torch.from_numpy(d["R"]).cuda() + U.float() @ D.float().T
    up, down, R = sq.svd_init(W, to_dev(omega(W.shape[1], 17)), 8)
    torch.cuda.synchronize()
    up_b, down_b = bits16(up), bits16(down)
    rows = np.array([0, 1, 8191, 16383])
    Wr = W[rows].cpu().numpy()
    Rr = R[rows].cpu().numpy()
    Rw = oracle.svd_residual(Wr, up_b[rows], down_b)
    assert np.array_equal(Rr.view(np.uint32), Rw.view(np.uint32)), first_mismatch(Rr, Rw)
    for f in (up_b, down_b):
        F = si.bf16_bits_to_f32(f).astype(np.float64)
        G = F.T @ F
        dg = np.sqrt(np.diag(G))
        assert np.all(np.diff(np.diag(G)) <= 1e-2 * np.diag(G)[:-1])          # descending
        off = np.abs(G / np.outer(dg, dg) - np.eye(32)).max()
        assert off <= 1e-2, off
    su = np.diag(si.bf16_bits_to_f32(up_b).astype(np.float64).T @ si.bf16_bits_to_f32(up_b).astype(np.float64))
    sd = np.diag(si.bf16_bits_to_f32(down_b).astype(np.float64).T @ si.bf16_bits_to_f32(down_b).astype(np.float64))
    assert np.allclose(su, sd, rtol=1e-2)


def gap16_weight(N, K, seed):
    """A rank-32 part with singular values 8 .. 4 then 1 .. 0.5 (a gap of 4 at index 16) plus the
    synthetic residual scaled to spectral norm 0.1."""
    rng = np.random.default_rng(seed)
    A = rng.standard_normal((N, 32)) / np.sqrt(N)
    B = rng.standard_normal((K, 32)) / np.sqrt(K)
    s = np.concatenate([np.geomspace(8.0, 4.0, 16), np.geomspace(1.0, 0.5, 16)])
    noise = si.make_inputs(4, K, N, seed)["R"].astype(np.float64)
    noise *= 0.1 / np.linalg.norm(noise, 2)
    W = ((A * s) @ B.T + noise).astype(np.float32)
    S = np.linalg.svd(W.astype(np.float64), compute_uv=False)
    assert S[15] >= 3 * S[16], "test weight without a spectral gap at 16"
    return W


@pytest.mark.parametrize("shape", [(256, 512), (1024, 768)])
def test_svd_init_rank16(sq, shape):
    """Rank 16 (the int8 mode's branch): factors [N, 16] / [K, 16], the rank-16 product against the
    oracle's truncated SVD, the residual of the rank-16 chain bit for bit."""
    N, K = shape
    W = gap16_weight(N, K, 120 + N)
    up, down, R = sq.svd_init(to_dev(W), to_dev(omega(K, 18)), 8, rank=16)
    torch.cuda.synchronize()
    assert tuple(up.shape) == (N, 16) and tuple(down.shape) == (K, 16)
    up_b, down_b, Rh = bits16(up), bits16(down), host(R)
    oup, odown, oR, _ = oracle.svd_init(W, rank=16)
    L, Lo = lowrank_product(up_b, down_b), lowrank_product(oup, odown)
    err = np.linalg.norm(L - Lo) / np.linalg.norm(Lo)
    assert err <= L_TOL, f"rank-16 product differs by {err:.3e}"
    Rw = oracle.svd_residual(W, up_b, down_b)
    assert np.array_equal(Rh.view(np.uint32), Rw.view(np.uint32)), first_mismatch(Rh, Rw)
    assert np.linalg.norm(Rh) <= np.linalg.norm(oR) * (1 + 1e-2)


def test_svd_init_then_int8_mode(sq):
    """The int8 mode end to end from a weight: SVD init at rank 16, the int8 builder on its
    residual, the reconstruct of W -- every step on the GPU, compared with the oracle run on the
    GPU's SVD outputs (codes, scales and the bf16 reconstruct bit for bit)."""
    W = gap16_weight(384, 768, 130)
    up, down, R = sq.svd_init(to_dev(W), to_dev(omega(768, 19)), 8, rank=16)
    w = sq.build_int8(R, up, down)
    Wb = sq.reconstruct_bf16(w)
    torch.cuda.synchronize()
    Rh, up_b, down_b = host(R), bits16(up), bits16(down)
    c, s, _ = oracle.build_int8(Rh)
    assert np.array_equal(host(w.codes), c) and np.array_equal(host(w.scales).view(np.uint32), s.view(np.uint32))
    Wo = oracle.reconstruct_bf16(oracle.FMT_INT8_ROW, c, s, 0.0, up_b, down_b, 384, 768)
    assert np.array_equal(bits16(Wb), Wo), first_mismatch(bits16(Wb), Wo)
    # the rebuilt weight is close to the original (int8 residual error plus bf16 output rounding)
    Wf = si.bf16_bits_to_f32(Wo).astype(np.float64)
    assert np.linalg.norm(Wf - W) <= 4e-3 * np.linalg.norm(W)
