"""Pins of the CPU oracle against facts it does not compute itself.

Each test ties one oracle routine to something outside it: a closed form, an
explicit matrix, a library conversion (numpy float16, torch bf16 / fp8), a
brute-force search, or a hand-worked golden table under tests/golden/.  The
routines follow the SquareQ README, section "SquareQ v3 -- W4"; the tests say
which part of it each one pins.
"""
import os

import numpy as np
import pytest
import torch

import synth_inputs as si

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                rows.append(line.split())
    return rows


def sylvester(n=256):
    i = np.arange(n)
    pop = np.vectorize(lambda v: bin(v).count("1"))(i[:, None] & i[None, :])
    return np.where(pop % 2 == 0, 1.0, -1.0) / np.sqrt(n)


# --------------------------------------------------------------------------
# O1/O2 rotation ("Rotation": block-diagonal normalised Hadamard-256)
# --------------------------------------------------------------------------

def test_fwht_basis_equals_sylvester_and_is_involution(oracle_mod):
    H = sylvester()
    for i in range(256):
        e = np.zeros(256, np.float32)
        e[i] = 1.0
        col = oracle_mod.fwht256(e)
        assert np.array_equal(col.astype(np.float64), H[:, i])      # exact: dyadic values
        back = oracle_mod.fwht256(col)
        assert np.array_equal(back, e)                               # H H = I, exactly


def test_fwht_matches_explicit_matrix_within_error_bound(oracle_mod):
    H = sylvester()
    rng = np.random.default_rng(11)
    for _ in range(20):
        v = (rng.standard_normal(256) * rng.lognormal(0, 2)).astype(np.float32)
        got = oracle_mod.fwht256(v).astype(np.float64)
        want = H @ v.astype(np.float64)
        bound = 8 * 2.0 ** -24 * np.abs(v.astype(np.float64)).sum() / 16 * 1.01
        assert np.max(np.abs(got - want)) <= bound
        # orthogonality: the norm is kept
        assert abs(np.linalg.norm(got) - np.linalg.norm(v)) <= 256 * bound
        twice = oracle_mod.fwht256(oracle_mod.fwht256(v)).astype(np.float64)
        assert np.max(np.abs(twice - v)) <= 2 * bound + 1e-30


def test_rotation_is_block_diagonal_over_k(oracle_mod):
    rng = np.random.default_rng(3)
    R = rng.standard_normal((3, 768)).astype(np.float32)
    out = oracle_mod.rotate_rows_f32(R)
    H = sylvester()
    for b in range(3):
        blk = R[:, 256 * b:256 * (b + 1)].astype(np.float64) @ H.T
        assert np.allclose(out[:, 256 * b:256 * (b + 1)], blk, atol=1e-5)
    xb = si.to_bf16_bits(R)
    outx = oracle_mod.rotate_rows_bf16(xb)
    assert np.array_equal(outx, oracle_mod.rotate_rows_f32(si.bf16_bits_to_f32(xb)))


# --------------------------------------------------------------------------
# conversions (bf16 / fp16 / ue4m3 / e2m1), pinned to libraries and tables
# --------------------------------------------------------------------------

def _probe_floats(n, seed):
    rng = np.random.default_rng(seed)
    bits = rng.integers(0, 2 ** 32, n, dtype=np.uint64).astype(np.uint32)
    vals = bits.view(np.float32)
    return vals[np.isfinite(vals)]


def test_bf16_matches_torch(oracle_mod):
    vals = _probe_floats(20000, 1)
    # add exact halfway points between neighbouring bf16 values
    hb = (np.arange(0x3F80, 0x3FA0, dtype=np.uint32) << 16) | 0x8000
    vals = np.concatenate([vals, hb.view(np.float32), -hb.view(np.float32),
                           np.array([0.0, -0.0, 3.4e38, 1e-45], np.float32)])
    want = si.to_bf16_bits(vals)
    got = np.array([oracle_mod.f32_to_bf16(v) for v in vals], np.uint16)
    assert np.array_equal(got, want)


def test_f16_matches_numpy(oracle_mod):
    rng = np.random.default_rng(2)
    vals = np.concatenate([
        (rng.standard_normal(20000) * np.exp(rng.uniform(-20, 12, 20000))).astype(np.float32),
        # halfway points of fp16 (normal and subnormal), and overflow edges
        ((np.arange(1, 2048, 7) + 0.5) * 2.0 ** -24).astype(np.float32),
        ((np.arange(1024, 2048, 5) + 0.5) * 2.0 ** -3).astype(np.float32),
        np.array([65504, 65519, 65520, 65536, 1e-8, 2.0 ** -25, 3 * 2.0 ** -26], np.float32),
    ])
    with np.errstate(over="ignore"):                 # 65520 and above overflow to inf on purpose
        want = vals.astype(np.float16).view(np.uint16)
    got = np.array([oracle_mod.f32_to_f16(v) for v in vals], np.uint16)
    assert np.array_equal(got, want)
    for h in list(range(0, 0x7C00, 97)) + [0x7BFF, 0x0001, 0x03FF, 0x0400]:
        assert oracle_mod.f16_to_f32(h) == float(np.uint16(h).view(np.float16))


def _ue4m3_table():
    return np.array([oracle_mod_free_ue4m3(c) for c in range(0x7F)])


def oracle_mod_free_ue4m3(c):
    e, m = c >> 3, c & 7
    return m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)


def _nearest_even(v, table):
    """Nearest table value; ties to the even code (fraction LSB 0)."""
    d = np.abs(table - v)
    best = np.flatnonzero(d == d.min())
    if len(best) == 1:
        return int(best[0])
    even = [b for b in best if b % 2 == 0]
    return int(even[0])


def test_ue4m3_golden_and_bruteforce(oracle_mod):
    for code, val in _golden("ue4m3_values.txt"):
        assert oracle_mod.ue4m3_to_f32(int(code, 16)) == float(val)
    table = _ue4m3_table()
    for c in range(0x7F):
        assert oracle_mod.ue4m3_to_f32(c) == table[c]
    rng = np.random.default_rng(5)
    mids = (table[1:] + table[:-1]) / 2
    vals = np.concatenate([mids, mids * (1 + 2.0 ** -20), mids * (1 - 2.0 ** -20),
                           rng.uniform(0, 460, 3000), np.exp(rng.uniform(-9, 6, 3000)),
                           [448.0, 455.9, 463.9, 464.0, 500.0, 1e30, 2.0 ** -11]]).astype(np.float32)
    for v in vals:
        want = _nearest_even(min(float(v), 448.0), table)
        assert oracle_mod.f32_to_ue4m3(v) == want, v
    # torch's e4m3 conversion agrees wherever no saturation is involved
    sub = vals[vals <= 448]
    tb = torch.from_numpy(sub).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle_mod.f32_to_ue4m3(v) for v in sub], np.uint8)
    assert np.array_equal(got, tb)


def test_e2m1_golden_ties_and_grid(oracle_mod):
    for v, code, dec in _golden("e2m1_ties.txt"):
        c = oracle_mod.f32_to_e2m1(float(v))
        assert c == int(code, 16), v
        assert oracle_mod.e2m1_to_f32(c) == float(dec)
    grid = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0}
    decoded = {oracle_mod.e2m1_to_f32(c) for c in range(16)}
    assert decoded == grid | {-g for g in grid}
    table = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    rng = np.random.default_rng(9)
    for v in rng.uniform(-8, 8, 4000).astype(np.float32):
        c = oracle_mod.f32_to_e2m1(v)
        assert (c & 7) == _nearest_even(min(abs(float(v)), 6.0), table)
        assert (c >> 3) == (1 if v < 0 else 0)


# --------------------------------------------------------------------------
# O3 int4 group-32 codec with MSE-swept fractions
# --------------------------------------------------------------------------

def _fp16(v):
    return float(np.float32(v).astype(np.float16))


def test_int4_fraction_grid(oracle_mod):
    for j in range(26):
        assert oracle_mod.int4_fraction(j) == np.float32((50 + 2 * j) / 100)
    assert oracle_mod.int4_fraction(0) == np.float32(0.5)
    assert oracle_mod.int4_fraction(25) == np.float32(1.0)


def test_int4_bruteforce_fraction_is_minimal(oracle_mod):
    """Exhaustive: recompute all 26 candidate errors in fp64 and check the pick."""
    rng = np.random.default_rng(21)
    for trial in range(300):
        kind = trial % 3
        r = rng.standard_normal(32)
        if kind == 1:
            r[rng.integers(0, 32)] *= 8.0            # an outlier
        if kind == 2:
            r = rng.standard_t(4, 32)
        r = (r * rng.lognormal(-3, 1)).astype(np.float32)
        q, s_bits, j = oracle_mod.int4_group32(r)
        assert q.min() >= -7 and q.max() <= 7
        a = float(np.abs(r).max())
        errs = []
        for jj in range(26):
            f = np.float32((50 + 2 * jj) / 100)
            s = _fp16(np.float32(np.float32(f * np.float32(a)) / np.float32(7)))
            qq = np.clip(np.round(r.astype(np.float64) / s), -7, 7) if s else np.zeros(32)
            errs.append(float(((r.astype(np.float64) - qq * s) ** 2).sum()))
        errs = np.array(errs)
        assert errs[j] <= errs.min() * (1 + 1e-5) + 1e-30
        s_expect = np.float32(np.float32(np.float32(oracle_mod.int4_fraction(j)) * np.float32(a)) / np.float32(7))
        assert s_bits == np.float32(s_expect).astype(np.float16).view(np.uint16)
        s = float(np.uint16(s_bits).view(np.float16))
        ideal = r.astype(np.float64) / s
        want = np.clip(np.round(ideal), -7, 7)
        # codes differ from exact rounding only at a knife-edge half
        diff = q != want
        assert np.all(np.abs(np.abs(ideal[diff] - np.trunc(ideal[diff])) - 0.5) < 1e-5)


def test_int4_exact_roundtrip_on_grid(oracle_mod):
    rng = np.random.default_rng(4)
    for _ in range(50):
        s = _fp16(rng.lognormal(-6, 1))
        q = rng.integers(-7, 8, 32)
        q[rng.integers(0, 32)] = 7 * rng.choice([-1, 1])
        r = (q * s).astype(np.float32)
        qo, sb, j = oracle_mod.int4_group32(r)
        assert np.array_equal(qo, q)
        assert float(np.uint16(sb).view(np.float16)) == s
        assert j == 25


def test_int4_ties_go_to_smaller_fraction(oracle_mod):
    # all-zero group: every fraction has zero error -> j = 0, s = 0
    q, s, j = oracle_mod.int4_group32(np.zeros(32, np.float32))
    assert j == 0 and s == 0 and not q.any()
    # a = 7 * 2^-24: f * a / 7 lands in the fp16 subnormal range; j = 0 (f = 0.5)
    # ties to s = 0, every j >= 1 gives s = 2^-24 and zero error -> j = 1
    r = np.full(32, 7 * 2.0 ** -24, np.float32)
    q, s, j = oracle_mod.int4_group32(r)
    assert j == 1 and s == 1 and np.all(q == 7)


def test_int4_build_packing_and_rotation(oracle_mod):
    # one row whose rotated values are on the grid: pick the rotated row first
    s = 2.0 ** -6
    q = np.tile(np.array([7, -7, 1, -1, 0, 3, -3, 2] * 4), 8)
    rot = (q * s).astype(np.float32)
    R = oracle_mod.fwht256(rot[:256])[None, :]        # H is its own inverse
    R = np.concatenate([R, oracle_mod.fwht256(rot[256:512] if rot.size >= 512 else rot[:256])[None, :]], 1)
    codes, scales, frac = oracle_mod.build_int4(R.astype(np.float32))
    assert codes.shape == (1, 256) and scales.shape == (1, 16)
    assert codes[0, 0] == 0x97           # q0 = 7 (low nibble), q1 = -7 -> 0x9 (high)
    assert codes[0, 1] == 0xF1           # 1, -1
    assert codes[0, 2] == 0x30           # 0, 3
    assert codes[0, 3] == 0x2D           # -3, 2
    assert np.all(scales == np.float16(s).view(np.uint16))
    assert np.all(frac == 25)


# --------------------------------------------------------------------------
# O4/O5 NVFP4 codec and tiled layout
# --------------------------------------------------------------------------

def test_sf_layout_golden_and_bijection(oracle_mod):
    for r, c, C, off in _golden("sf_tiled_offsets.txt"):
        assert oracle_mod.sf_offset(int(r), int(c), int(C)) == int(off)
    for rows, C in [(128, 16), (256, 32), (384, 48)]:
        offs = np.array([oracle_mod.sf_offset(r, c, C) for r in range(rows) for c in range(C)])
        assert np.array_equal(np.sort(offs), np.arange(rows * C))
    assert oracle_mod.sf_bytes(1, 256) == 128 * 16
    assert oracle_mod.sf_bytes(129, 512) == 256 * 32


def test_nvfp4_exact_roundtrip_on_grid(oracle_mod):
    rng = np.random.default_rng(8)
    g = 2.0 ** -12
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    table = _ue4m3_table()
    rows, K = 8, 256
    e = rng.choice(grid, (rows, K)) * rng.choice([-1, 1], (rows, K))
    S = rng.choice(table[9:0x7E], (rows, K // 16))
    e.reshape(rows, K // 16, 16)[:, :, 0] = 6.0      # every block reaches 6 * S
    S[0, 0] = 448.0                                   # tensor absmax = 2688 g
    vals = (e.reshape(rows, K // 16, 16) * S[:, :, None] * g).reshape(rows, K).astype(np.float32)
    A = float(np.abs(vals).max())
    assert A == 2688 * g
    gg = oracle_mod.nvfp4_global_scale(A)
    assert gg == g
    codes, sf = oracle_mod.nvfp4_quant_rotated(vals, g)
    for r in range(rows):
        for c in range(K // 16):
            assert oracle_mod.ue4m3_to_f32(sf[oracle_mod.sf_offset(r, c, K // 16)]) == S[r, c]
            for i in range(16):
                k = 16 * c + i
                byte = codes[r, k // 2]
                code = (byte >> 4) if (k & 1) else (byte & 0xF)
                assert oracle_mod.e2m1_to_f32(code) == e[r, k] or (e[r, k] == 0 and oracle_mod.e2m1_to_f32(code) == 0)
    assert sf[oracle_mod.sf_offset(0, 0, K // 16)] == 0x7E


def test_nvfp4_block_bruteforce(oracle_mod):
    rng = np.random.default_rng(12)
    table = _ue4m3_table()
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    for _ in range(200):
        r = (rng.standard_t(4, 16) * rng.lognormal(-4, 1)).astype(np.float32)
        A = float(np.abs(r).max()) * float(rng.uniform(1, 30))
        g = np.float32(np.float32(A) / np.float32(2688))
        codes, sf = oracle_mod.nvfp4_block16(r, g)
        b = float(np.abs(r).max())
        ratio = b / (6 * float(g))
        # the chosen scale is the ue4m3 value nearest to b / (6 g)
        assert abs(table[sf] - ratio) <= np.abs(table - ratio).min() * (1 + 1e-6) + 1e-12
        if sf == 0:
            assert not codes.any()
            continue
        den = table[sf] * float(g)
        for i in range(16):
            code = (codes[i // 2] >> 4) if (i & 1) else (codes[i // 2] & 0xF)
            v = float(r[i]) / den
            dist = np.abs(grid - min(abs(v), 6.0))
            assert dist[code & 7] <= dist.min() + 1e-6
    # saturation: the block holding the tensor absmax never exceeds 0x7E
    r = np.linspace(-1, 1, 16).astype(np.float32)
    codes, sf = oracle_mod.nvfp4_block16(r, np.float32(1.0 / 2688))
    assert sf == 0x7E


def test_nvfp4_zero_tensor(oracle_mod):
    R = np.zeros((4, 256), np.float32)
    codes, sf, g = oracle_mod.build_nvfp4(R)
    assert g == 0 and not codes.any() and not sf.any()


# --------------------------------------------------------------------------
# O6-O9 activation quant, forwards, reconstruct
# --------------------------------------------------------------------------

E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6])


def _decode_nvfp4(codes, sf, rows, K):
    """numpy decode of a payload: e2m1 * ue4m3 (written here from the formats)."""
    table = _ue4m3_table()
    lo = codes & 0xF
    hi = codes >> 4
    nib = np.stack([lo, hi], -1).reshape(rows, K)
    r = np.arange(rows)[:, None]
    c = np.arange(K // 16)[None, :]
    C = K // 16
    off = ((r // 128) * (C // 4) + c // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (c % 4)
    s = table[sf[off]]
    return E2M1[nib] * np.repeat(s, 16, axis=1)


def test_build_nvfp4_global_scale_is_of_the_rotated_tensor(oracle_mod):
    """Rows of R are scaled Sylvester rows, so the rotated tensor is exactly one-hot: c at (0, 5)
    and c/4 at (1, 256 + 200), while R itself peaks at c/16.  The global scale must come from the
    rotated tensor, g_w = RN(c / 2688) = 2^-10, and both peaks decode back exactly (e2m1 6 times
    ue4m3 448, resp. 112, times g_w); every other value is 0."""
    N, K = 2, 512
    H16 = np.rint(sylvester() * 16)                         # the +-1 Sylvester matrix
    c = 2688.0 * 2.0 ** -10
    R = np.zeros((N, K), np.float32)
    R[0, :256] = (c / 16) * H16[5]
    R[1, 256:] = (c / 64) * H16[200]
    assert np.abs(R).max() == c / 16
    codes, sf, g = oracle_mod.build_nvfp4(R)
    assert g == np.float32(2.0 ** -10)
    want = np.zeros((N, K))
    want[0, 5] = c
    want[1, 256 + 200] = c / 4
    assert np.array_equal(_decode_nvfp4(codes, sf, N, K) * float(g), want)


def test_act_quant_lowrank_input_matches_matmul(oracle_mod):
    d = si.make_inputs(40, 512, 128, 7)
    codes, sf, g, t = oracle_mod.act_quant_nvfp4(d["x"], d["D"])
    want = si.bf16_bits_to_f32(d["x"]).astype(np.float64) @ si.bf16_bits_to_f32(d["D"]).astype(np.float64)
    assert np.allclose(t, want, rtol=1e-12, atol=1e-12)
    xr = oracle_mod.rotate_rows_bf16(d["x"])
    assert g == np.float32(np.float32(np.abs(xr).max()) / np.float32(2688))
    c2, s2, g2, _ = oracle_mod.act_quant_nvfp4(d["x"], None, static_g=g * 2)
    assert g2 == np.float32(g * 2)
    c3, s3 = oracle_mod.nvfp4_quant_rotated(xr, g * 2)
    assert np.array_equal(c2, c3) and np.array_equal(s2, s3)


def test_nvfp4_forward_equals_decoded_gemm(oracle_mod):
    M, K, N = 24, 512, 136
    d = si.make_inputs(M, K, N, 13)
    wc, wsf, gw = oracle_mod.build_nvfp4(d["R"])
    xc, xsf, gx, t = oracle_mod.act_quant_nvfp4(d["x"], d["D"])
    y = oracle_mod.linear_fwd_nvfp4(xc, xsf, gx, wc, wsf, gw, t, d["U"], M, N, K)
    X = _decode_nvfp4(xc, xsf, M, K)
    Wd = _decode_nvfp4(wc, wsf, N, K)
    U = si.bf16_bits_to_f32(d["U"]).astype(np.float64)
    want = float(gx) * float(gw) * (X @ Wd.T) + t @ U.T
    assert np.allclose(y, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    rows = np.array([5, 0, 23])
    ys = oracle_mod.linear_fwd_nvfp4(xc, xsf, gx, wc, wsf, gw, t, d["U"], M, N, K, rows)
    assert np.array_equal(ys, y[rows])
    # the whole chain approximates x W^T with W = U D^T + R (4-bit noise only)
    x = si.bf16_bits_to_f32(d["x"]).astype(np.float64)
    Wtrue = U @ si.bf16_bits_to_f32(d["D"]).astype(np.float64).T + d["R"].astype(np.float64)
    ref = x @ Wtrue.T
    cos = (y * ref).sum() / np.linalg.norm(y) / np.linalg.norm(ref)
    assert cos > 0.98


def test_int4_forward_equals_decoded_gemm(oracle_mod):
    M, K, N = 24, 512, 136
    d = si.make_inputs(M, K, N, 14)
    codes, scales, frac = oracle_mod.build_int4(d["R"])
    xr = oracle_mod.rotate_rows_bf16(d["x"])
    _, _, _, t = oracle_mod.act_quant_nvfp4(d["x"], d["D"])
    y = oracle_mod.linear_fwd_int4(xr, codes, scales, t, d["U"], M, N, K)
    nib = np.stack([codes & 0xF, codes >> 4], -1).reshape(N, K).astype(np.int64)
    q = np.where(nib >= 8, nib - 16, nib)
    s = np.repeat(scales.view(np.float16).astype(np.float64), 32, axis=1)
    wb = si.bf16_bits_to_f32(si.to_bf16_bits((q * s).astype(np.float32))).astype(np.float64)
    xb = si.bf16_bits_to_f32(si.to_bf16_bits(xr)).astype(np.float64)
    U = si.bf16_bits_to_f32(d["U"]).astype(np.float64)
    want = xb @ wb.T + t @ U.T
    assert np.allclose(y, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    rows = np.array([5, 0, 23])                      # a row subset evaluates exactly those rows
    ys = oracle_mod.linear_fwd_int4(xr, codes, scales, t, d["U"], M, N, K, rows)
    assert np.array_equal(ys, y[rows])
    x = si.bf16_bits_to_f32(d["x"]).astype(np.float64)
    Wtrue = U @ si.bf16_bits_to_f32(d["D"]).astype(np.float64).T + d["R"].astype(np.float64)
    ref = x @ Wtrue.T
    cos = (y * ref).sum() / np.linalg.norm(y) / np.linalg.norm(ref)
    assert cos > 0.99


def test_reconstruct_on_grid_is_explicit_hadamard(oracle_mod):
    N, K = 3, 512
    rng = np.random.default_rng(30)
    q = rng.integers(-7, 8, (N, K))
    s = 2.0 ** -5
    nib = (q & 0xF).astype(np.uint8)
    codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    scales = np.full((N, K // 32), np.float16(s).view(np.uint16), np.uint16)
    zeroU = np.zeros((N, 32), np.uint16)
    zeroD = np.zeros((K, 32), np.uint16)
    W = oracle_mod.reconstruct_bf16(oracle_mod.FMT_INT4, codes, scales, 0.0, zeroU, zeroD, N, K)
    H = sylvester()
    d = q * s
    h = np.concatenate([d[:, b:b + 256] @ H.T for b in (0, 256)], 1)
    assert np.array_equal(W, si.to_bf16_bits(h.astype(np.float32)))


def test_reconstruct_nvfp4_on_grid_is_explicit_hadamard(oracle_mod):
    """NVFP4 payload on a grid where every step is exact in fp32: e2m1 codes times ue4m3 scales in
    [1, 2) times g_w = 3 * 2^-8 are integer multiples of 3 * 2^-12 below 2^11 of them, so the fp32
    Hadamard sums are exact and W = bf16(H applied to the decoded values) is computable by the
    explicit matrix.  Pins the decode value(e2m1) * value(sf) * g_w, the tiled scale lookup and the
    inverse rotation; residual_only must give the same W whatever the low-rank factors hold."""
    N, K = 3, 512
    C = K // 16
    rng = np.random.default_rng(32)
    nib = rng.integers(0, 16, (N, K)).astype(np.uint8)
    codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    sfc = rng.integers(0x38, 0x40, (N, C)).astype(np.uint8)       # values 1 + m/8
    sf = np.zeros(128 * C, np.uint8)
    r = np.arange(N)[:, None]
    c = np.arange(C)[None, :]
    sf[((r // 128) * (C // 4) + c // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (c % 4)] = sfc
    g = np.float32(3 * 2.0 ** -8)
    d = E2M1[nib] * np.repeat(1 + (sfc & 7) / 8.0, 16, axis=1) * float(g)
    H = sylvester()
    h = np.concatenate([d[:, b:b + 256] @ H.T for b in (0, 256)], 1)
    want = si.to_bf16_bits(h.astype(np.float32))
    zeroU = np.zeros((N, 32), np.uint16)
    zeroD = np.zeros((K, 32), np.uint16)
    W = oracle_mod.reconstruct_bf16(oracle_mod.FMT_NVFP4, codes, sf, g, zeroU, zeroD, N, K)
    assert np.array_equal(W, want)
    U = si.to_bf16_bits(rng.standard_normal((N, 32)).astype(np.float32))
    D = si.to_bf16_bits(rng.standard_normal((K, 32)).astype(np.float32))
    Wr = oracle_mod.reconstruct_bf16(oracle_mod.FMT_NVFP4, codes, sf, g, U, D, N, K, residual_only=True)
    assert np.array_equal(Wr, want)


def test_reconstruct_lowrank_chain_and_fidelity(oracle_mod):
    N, K = 64, 512
    d = si.make_inputs(8, K, N, 31)
    U = si.bf16_bits_to_f32(d["U"]).astype(np.float64)
    D = si.bf16_bits_to_f32(d["D"]).astype(np.float64)
    codes, scales, _ = oracle_mod.build_int4(np.zeros((N, K), np.float32))
    W = oracle_mod.reconstruct_bf16(oracle_mod.FMT_INT4, codes, scales, 0.0, d["U"], d["D"], N, K)
    L = U @ D.T
    Wf = si.bf16_bits_to_f32(W).astype(np.float64)
    # fp32 fma chain within 32 u of the fp64 dot, then one bf16 rounding
    bound = 32 * 2.0 ** -24 * (np.abs(U) @ np.abs(D).T) + 2.0 ** -8 * np.abs(L)
    assert np.all(np.abs(Wf - L) <= bound + 1e-30)
    # full reconstruct approximates U D^T + R for both codecs
    for fmt in (oracle_mod.FMT_INT4, oracle_mod.FMT_NVFP4):
        if fmt == oracle_mod.FMT_INT4:
            c, s, _ = oracle_mod.build_int4(d["R"])
            g = 0.0
        else:
            c, s, g = oracle_mod.build_nvfp4(d["R"])
        W = si.bf16_bits_to_f32(oracle_mod.reconstruct_bf16(fmt, c, s, g, d["U"], d["D"], N, K)).astype(np.float64)
        ref = L + d["R"]
        cos = (W * ref).sum() / np.linalg.norm(W) / np.linalg.norm(ref)
        assert cos > (0.99 if fmt == oracle_mod.FMT_INT4 else 0.98)
        Wr = si.bf16_bits_to_f32(oracle_mod.reconstruct_bf16(fmt, c, s, g, d["U"], d["D"], N, K,
                                                             residual_only=True)).astype(np.float64)
        cos_r = (Wr * d["R"]).sum() / np.linalg.norm(Wr) / np.linalg.norm(d["R"])
        assert cos_r > 0.98


# --------------------------------------------------------------------------
# backward of the input ("End-to-end": bf16 reconstruct, then the bf16 GEMM)
# --------------------------------------------------------------------------

def test_bwd_dx_equals_decoded_gemm(oracle_mod):
    M, K, N = 12, 512, 136
    d = si.make_inputs(M, K, N, 33)
    c, s, _ = oracle_mod.build_int4(d["R"])
    W = oracle_mod.reconstruct_bf16(oracle_mod.FMT_INT4, c, s, 0.0, d["U"], d["D"], N, K)
    rng = np.random.default_rng(34)
    dy = si.to_bf16_bits(rng.standard_normal((M, N)).astype(np.float32))
    dy[3, :] = 0
    dx = oracle_mod.linear_bwd_dx(dy, W)
    want = si.bf16_bits_to_f32(dy).astype(np.float64) @ si.bf16_bits_to_f32(W).astype(np.float64)
    assert np.allclose(dx, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    rows = np.array([0, 5, 11], np.int64)
    assert np.array_equal(oracle_mod.linear_bwd_dx(dy, W, rows), dx[rows])
