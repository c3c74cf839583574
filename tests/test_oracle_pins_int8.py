"""Pins of the oracle's int8 per-row codec (SquareQ README, "v3.1 -- int8-residual
mode": the rotated residual of a rank-16 branch in int8, one MSE-chosen scale per row).

Readings pinned here: the int4 fraction grid f_j = (50 + 2j)/100, an fp32 row scale
s = RN(RN(f_j a) / 127), codes clamp(rint(RN(r RN(1/s))), -127, 127), the error
fmaf(-q, s, r) squared, the row sum taken block by block (see the oracle), the
smallest error winning with ties to the smaller fraction; dequantisation RN(q s);
the low-rank branch of rank 16.
"""
import numpy as np
import torch

import synth_inputs as si


def _scale(oracle_mod, j, a):
    f = np.float32(oracle_mod.int4_fraction(j))
    return np.float32(np.float32(f * np.float32(a)) / np.float32(127))


def test_int8_row_bruteforce_fraction_is_minimal(oracle_mod):
    """All 26 candidate errors in fp64 on the fp32 scales; the pick is minimal up to rounding,
    and the stored scale is the winner's."""
    rng = np.random.default_rng(80)
    for trial in range(60):
        K = 256 * (1 + trial % 3)
        r = rng.standard_normal(K)
        if trial % 3 == 1:
            r[rng.integers(0, K, 3)] *= 10.0
        if trial % 3 == 2:
            r = rng.standard_t(4, K)
        r = (r * rng.lognormal(-4, 1)).astype(np.float32)
        q, s, j = oracle_mod.int8_row(r)
        assert q.min() >= -127 and q.max() <= 127
        a = float(np.abs(r).max())
        errs = []
        for jj in range(26):
            sj = float(_scale(oracle_mod, jj, a))
            qq = np.clip(np.round(r.astype(np.float64) / sj), -127, 127)
            errs.append(float(((r.astype(np.float64) - qq * sj) ** 2).sum()))
        errs = np.array(errs)
        assert errs[j] <= errs.min() * (1 + 1e-4) + 1e-30
        assert s == _scale(oracle_mod, j, a)
        # the codes are the nearest multiples of the chosen scale (clamped)
        want = np.clip(np.round(r.astype(np.float64) / float(s)), -127, 127)
        assert np.abs(q - want).max() <= 1
        assert np.mean(q == want) > 0.999


def test_int8_row_exact_roundtrip_on_grid(oracle_mod):
    rng = np.random.default_rng(81)
    for _ in range(40):
        K = 512
        # a scale with <= 17 significant bits, so 127 s and every q s are exact in fp32
        s = np.float32(np.ldexp(float(rng.integers(1 << 16, 1 << 17)), int(rng.integers(-40, -20))))
        q = rng.integers(-127, 128, K)
        q[rng.integers(0, K)] = 127 * rng.choice([-1, 1])
        r = (q * np.float64(s)).astype(np.float32)
        assert np.array_equal(r.astype(np.float64), q * np.float64(s))
        qo, so, j = oracle_mod.int8_row(r)
        assert np.array_equal(qo, q)
        assert so == s
        assert j == 25


def test_int8_zero_row_and_tiny_row(oracle_mod):
    q, s, j = oracle_mod.int8_row(np.zeros(256, np.float32))
    assert not q.any() and s == 0.0 and j == 0
    # a row whose scale underflows to 0 for every fraction: codes 0, error sum r^2 for all j -> j = 0
    r = np.zeros(256, np.float32)
    r[7] = np.float32(1e-45)
    q, s, j = oracle_mod.int8_row(r)
    assert not q.any() and s == 0.0 and j == 0


def test_int8_build_rotates_rows(oracle_mod):
    N, K = 6, 768
    d = si.make_inputs(4, K, N, 82)
    codes, scales, frac = oracle_mod.build_int8(d["R"])
    rot = oracle_mod.rotate_rows_f32(d["R"])
    for n in range(N):
        q, s, j = oracle_mod.int8_row(rot[n])
        assert np.array_equal(codes[n], q) and scales[n] == s and frac[n] == j
    # unclamped values decode within half a step; clamped ones lie beyond the last step
    deq = codes.astype(np.float64) * scales[:, None].astype(np.float64)
    sc = scales[:, None].astype(np.float64)
    inner = np.abs(codes.astype(np.int64)) < 127
    assert np.all((np.abs(deq - rot) <= 0.5 * sc * (1 + 1e-6))[inner])
    assert np.all((np.abs(rot) >= 126.5 * sc * (1 - 1e-6))[~inner])


def test_int8_forward_equals_decoded_gemm(oracle_mod):
    M, K, N = 20, 512, 136
    d = si.make_inputs(M, K, N, 83)
    U16, D16 = np.ascontiguousarray(d["U"][:, :16]), np.ascontiguousarray(d["D"][:, :16])
    codes, scales, _ = oracle_mod.build_int8(d["R"])
    xr = oracle_mod.rotate_rows_bf16(d["x"])
    t = oracle_mod.lowrank_input(d["x"], D16)
    y = oracle_mod.linear_fwd_int8(xr, codes, scales, t, U16, M, N, K)
    wf = (torch.from_numpy(codes.astype(np.float32)) * torch.from_numpy(scales)[:, None]).to(torch.bfloat16)
    wb = wf.to(torch.float64).numpy()
    xb = torch.from_numpy(xr).to(torch.bfloat16).to(torch.float64).numpy()
    U = si.bf16_bits_to_f32(U16).astype(np.float64)
    x = si.bf16_bits_to_f32(d["x"]).astype(np.float64)
    D = si.bf16_bits_to_f32(D16).astype(np.float64)
    assert np.allclose(t, x @ D, rtol=1e-12, atol=1e-12 * np.abs(x @ D).max())
    want = xb @ wb.T + t @ U.T
    assert np.allclose(y, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    rows = np.array([5, 0, 19])                      # a row subset evaluates exactly those rows
    ys = oracle_mod.linear_fwd_int8(xr, codes, scales, t, U16, M, N, K, rows)
    assert np.array_equal(ys, y[rows])
    Wtrue = U @ D.T + d["R"].astype(np.float64)
    ref = x @ Wtrue.T
    cos = (y * ref).sum() / np.linalg.norm(y) / np.linalg.norm(ref)
    assert cos > 0.999


def test_int8_reconstruct_on_grid_is_explicit_hadamard(oracle_mod):
    N, K = 3, 512
    rng = np.random.default_rng(84)
    q = rng.integers(-127, 128, (N, K)).astype(np.int8)
    s = np.full(N, 2.0 ** -9, np.float32)
    zU, zD = np.zeros((N, 16), np.uint16), np.zeros((K, 16), np.uint16)
    W = oracle_mod.reconstruct_bf16(oracle_mod.FMT_INT8_ROW, q, s, 0.0, zU, zD, N, K)
    i = np.arange(256)
    pop = np.vectorize(lambda v: bin(v).count("1"))(i[:, None] & i[None, :])
    H = np.where(pop % 2 == 0, 1.0, -1.0) / 16.0
    d = q.astype(np.float64) * 2.0 ** -9
    h = np.concatenate([d[:, b:b + 256] @ H.T for b in (0, 256)], 1)
    assert np.array_equal(W, si.to_bf16_bits(h.astype(np.float32)))


def test_int8_reconstruct_rank16_chain(oracle_mod):
    N, K = 40, 512
    d = si.make_inputs(8, K, N, 85)
    U16, D16 = np.ascontiguousarray(d["U"][:, :16]), np.ascontiguousarray(d["D"][:, :16])
    U = si.bf16_bits_to_f32(U16).astype(np.float64)
    D = si.bf16_bits_to_f32(D16).astype(np.float64)
    codes = np.zeros((N, K), np.int8)
    W = oracle_mod.reconstruct_bf16(oracle_mod.FMT_INT8_ROW, codes, np.zeros(N, np.float32), 0.0, U16, D16, N, K)
    L = U @ D.T
    Wf = si.bf16_bits_to_f32(W).astype(np.float64)
    bound = 16 * 2.0 ** -24 * (np.abs(U) @ np.abs(D).T) + 2.0 ** -8 * np.abs(L)
    assert np.all(np.abs(Wf - L) <= bound + 1e-30)
    c, s, _ = oracle_mod.build_int8(d["R"])
    Wr = si.bf16_bits_to_f32(oracle_mod.reconstruct_bf16(oracle_mod.FMT_INT8_ROW, c, s, 0.0, U16, D16, N, K))
    ref = L + d["R"]
    cos = (Wr * ref).sum() / np.linalg.norm(Wr) / np.linalg.norm(ref)
    assert cos > 0.9999
