"""Pins of the oracle's NVFP4 variant (SVDQuant review section 8: groups of
16 with FP8 scales; section 9.1 on the FP4 grid).  The E4M3 rounding is
checked against torch's float8_e4m3fn cast, the E2M1 rounding and the whole
row quantiser against an independent pipeline (numpy float32 arithmetic,
torch's E4M3 cast and exact rationals), and the product against a rational
brute force."""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth

GRID = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3),
        Fraction(4), Fraction(6)]


def _e4m3_torch(x):
    t = torch.tensor(np.asarray(x, dtype=np.float32)).to(torch.float8_e4m3fn)
    return t.to(torch.float32).numpy().astype(np.float64), t.view(torch.uint8).numpy()


def _decode_e4m3(bits):
    bits = int(bits)
    e, m = (bits >> 3) & 15, bits & 7
    return Fraction(m, 8) * Fraction(1, 64) if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)


def test_e4m3_matches_torch_cast_and_bit_decode():
    rng = np.random.default_rng(1)
    every = np.array([float(_decode_e4m3(b)) for b in range(127)])       # 0 .. 448, no NaN
    mids = (every[1:] + every[:-1]) / 2                                   # ties
    rand = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(447.0), 4000))
    x = np.concatenate([every, mids, rand]).astype(np.float32).astype(np.float64)
    mine = oracle.round_e4m3(x)
    ref, ref_bits = _e4m3_torch(x)
    assert np.array_equal(mine, ref)
    assert np.array_equal(oracle.e4m3_bits(mine), ref_bits)
    for b in range(127):
        assert oracle.e4m3_bits(np.array([every[b]]))[0] == b
    assert np.array_equal(oracle.round_e4m3([449.0, 463.0, 1e6]), [448.0] * 3)   # saturation


def _e2m1_exact(z, d):
    u = Fraction(z) / Fraction(d)
    a = abs(u)
    best = min(range(8), key=lambda i: (abs(a - GRID[i]), i % 2))          # nearest, then even
    return best | (8 if (u < 0 and best > 0) else 0)


def test_e2m1_codes_match_rational_rounding():
    rng = np.random.default_rng(2)
    d = np.float32(rng.uniform(0.01, 3.0))
    z = (rng.standard_normal(3000) * 3 * float(d)).astype(np.float32).astype(np.float64)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.5, 7.5]) * float(d)  # exact ties
    z = np.concatenate([z, mids, -mids, [0.0, -0.0]])
    codes = oracle.e2m1_codes(z, float(d))
    for zi, c in zip(z, codes):
        assert c == _e2m1_exact(zi, float(d)), (zi, c)


def _rows_independent(v):
    """The row quantiser through float32 numpy arithmetic, torch's E4M3 cast
    and exact rationals (no oracle code)."""
    v32 = v.astype(np.float32)
    rows, K = v32.shape
    s = np.max(np.abs(v32), axis=1) / np.float32(2688.0)
    d6 = np.float32(6.0) * s
    g = v32.reshape(rows, K // 16, 16)
    mg = np.max(np.abs(g), axis=2)
    t = np.where(d6[:, None] > 0, mg / np.where(d6 > 0, d6, 1)[:, None], 0).astype(np.float32)
    b, _ = _e4m3_torch(t)
    codes = np.zeros((rows, K), np.int64)
    for i in range(rows):
        for j in range(K):
            dd = Fraction(float(b[i, j // 16])) * Fraction(float(s[i]))
            codes[i, j] = 0 if dd == 0 else _e2m1_exact(float(v32[i, j]), dd)
    return codes, b, s.astype(np.float64)


def test_row_quantiser_matches_independent_pipeline():
    rng = np.random.default_rng(3)
    v = rng.standard_normal((6, 64)) * np.exp(rng.uniform(-8, 4, (6, 1)))
    v[:, 5] *= 40                                                        # an outlier channel
    v[2, 16:32] = 0                                                      # an all-zero group
    v[4] = 0                                                             # an all-zero row
    v = v.astype(np.float32).astype(np.float64)
    codes, b, s = oracle.quantize_nvfp4_rows(v)
    c2, b2, s2 = _rows_independent(v)
    assert np.array_equal(s, s2) and np.array_equal(b, b2) and np.array_equal(codes, c2)
    assert np.all(b[2, 1] == 0) and not codes[4].any() and s[4] == 0
    nz = s > 0
    assert np.all(np.max(b[nz], axis=1) == 448.0)       # the row's largest group maps to 448


def test_linear_nvfp4_is_the_rational_brute_force():
    rng = np.random.default_rng(4)
    M, K, N, r = 3, 32, 4, 2
    xc = rng.integers(0, 16, (M, K))
    wc = rng.integers(0, 16, (N, K))
    xb = oracle.round_e4m3(rng.uniform(0.01, 400, (M, K // 16)))
    wb = oracle.round_e4m3(rng.uniform(0.01, 400, (N, K // 16)))
    xs = rng.uniform(1e-4, 1e-2, M).astype(np.float32).astype(np.float64)
    ws = rng.uniform(1e-4, 1e-2, N).astype(np.float32).astype(np.float64)
    Z = oracle.round_bf16(rng.standard_normal((M, r)))
    L2 = oracle.round_bf16(rng.standard_normal((r, N)))
    bias = oracle.round_bf16(rng.standard_normal(N))
    Y, Yb = oracle.linear_nvfp4(xc, xb, xs, Z, wc, wb, ws, L2, bias)

    def val(c):
        v = GRID[int(c) & 7]
        return -v if int(c) & 8 else v
    for i in range(M):
        for n in range(N):
            acc = Fraction(0)
            for k in range(K):
                acc += (val(xc[i, k]) * Fraction(xb[i, k // 16]) * Fraction(xs[i]) *
                        val(wc[n, k]) * Fraction(wb[n, k // 16]) * Fraction(ws[n]))
            acc += sum(Fraction(Z[i, j]) * Fraction(L2[j, n]) for j in range(r)) + Fraction(bias[n])
            assert Y[i, n] == pytest.approx(float(acc), rel=1e-12, abs=1e-12)
    assert np.array_equal(Yb, oracle.round_bf16(Y))


def test_nvfp4_layer_on_the_outlier_workload():
    L = synth.make_layer(synth.WORKLOADS["tiny"])
    X = oracle.bf16_bits_to_f64(L.X)
    ref = X @ oracle.bf16_bits_to_f64(L.W).T
    a = oracle.calib_absmax(X)
    p = oracle.pack_weights_nvfp4(L.W, a, 16)
    q = oracle.pack_weights(L.W, a, 16)
    for k in ("inv_lambda", "L1b", "L2b", "R"):
        assert np.array_equal(p[k], q[k]), k
    xc, xb, xs, Z, _ = oracle.quantize_act_nvfp4(L.X, p["inv_lambda"], p["L1b"])
    Y, _ = oracle.linear_nvfp4(xc, xb, xs, Z, p["wcodes4"], p["wb4"], p["ws4"], p["L2b"], p["bias"])
    e = np.linalg.norm(Y - ref) / np.linalg.norm(ref)
    e4 = oracle.layer_output_error(L.X, q, L.W)
    assert e < 0.1 and e < 1.5 * e4
