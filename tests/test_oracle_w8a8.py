"""Pins of the oracle's W8A8 comparator (SVDQuant review section 8: the
eight-bit setting, rank 16 with dynamic per-token activation and
per-channel weight scales).  The quantiser is checked against exact rational
rounding with an independently computed fp32 scale, the product against a
Python-integer brute force, and the packed residual against its bound."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth


def _scale_f32(row):
    # fl32(max|v| / 127) by native fp32 division (IEEE: correctly rounded)
    m = np.float32(np.max(np.abs(np.asarray(row, dtype=np.float32))))
    return float(m / np.float32(127.0))


def test_int8_rows_match_exact_rational_rounding():
    rng = np.random.default_rng(7)
    v = (rng.standard_normal((40, 96)) * np.exp(rng.uniform(-6, 6, (40, 1)))).astype(np.float32)
    v = v.astype(np.float64)
    codes, s = oracle.quantize_rows_int8(v)
    for i in range(v.shape[0]):
        si = _scale_f32(v[i])
        assert s[i] == si
        for k in range(v.shape[1]):
            q = round(Fraction(v[i, k]) / Fraction(si))          # half to even
            assert codes[i, k] == max(-128, min(127, q)), (i, k)


def test_int8_ties_round_to_even():
    # max = 127/8 makes s = 1/8 exactly; (2j+1)/16 are exact ties
    j = np.arange(-60, 60)
    row = np.concatenate([[127 / 8], (2 * j + 1) / 16.0])
    codes, s = oracle.quantize_rows_int8(row[None, :])
    assert s[0] == 0.125
    expect = [round(Fraction(int(2 * x + 1), 2)) for x in j]     # Python rounds half to even
    assert codes[0, 0] == 127
    assert list(codes[0, 1:]) == expect
    assert all(c % 2 == 0 for c in codes[0, 1:])


def test_int8_bound_range_and_zero_rows():
    rng = np.random.default_rng(8)
    v = rng.standard_normal((16, 200)).astype(np.float32).astype(np.float64)
    v[3] = 0.0
    codes, s = oracle.quantize_rows_int8(v)
    assert s[3] == 0 and not codes[3].any()
    nz = s > 0
    err = np.abs(v[nz] - codes[nz] * s[nz][:, None])
    assert np.all(err <= s[nz][:, None] / 2)
    assert np.max(np.abs(codes)) == 127
    assert np.all(np.max(np.abs(codes[nz]), axis=1) == 127)    # the absmax element maps to +-127


def test_linear_w8a8_is_the_integer_brute_force():
    rng = np.random.default_rng(9)
    M, K, N, r = 5, 48, 7, 3
    xc = rng.integers(-127, 128, (M, K))
    wc = rng.integers(-127, 128, (N, K))
    s_x = rng.uniform(0.01, 2, M).astype(np.float32).astype(np.float64)
    s_w = rng.uniform(0.01, 2, N).astype(np.float32).astype(np.float64)
    Z = oracle.round_bf16(rng.standard_normal((M, r)))
    L2 = oracle.round_bf16(rng.standard_normal((r, N)))
    b = oracle.round_bf16(rng.standard_normal(N))
    Y, Yb = oracle.linear_w8a8(xc, s_x, Z, wc, s_w, L2, b)
    for i in range(M):
        for n in range(N):
            acc = 0
            for k in range(K):
                acc += int(xc[i, k]) * int(wc[n, k])
            exact = (Fraction(s_x[i]) * Fraction(s_w[n]) * acc
                     + sum(Fraction(Z[i, j]) * Fraction(L2[j, n]) for j in range(r)) + Fraction(b[n]))
            assert Y[i, n] == pytest.approx(float(exact), rel=1e-13, abs=1e-13)
    assert np.array_equal(Yb, oracle.round_bf16(Y))
    # a block of rows / columns is the same block of the full product
    Ys, _ = oracle.linear_w8a8(xc, s_x, Z, wc, s_w, L2, b, rows=[4, 1], cols=[6, 0, 2])
    assert np.array_equal(Ys, Y[np.ix_([4, 1], [6, 0, 2])])


@pytest.fixture(scope="module")
def tiny():
    return synth.make_layer(synth.WORKLOADS["tiny"])


def test_w8a8_pack_residual_and_bound(tiny):
    L = tiny
    a = oracle.calib_absmax(oracle.bf16_bits_to_f64(L.X))
    p = oracle.pack_weights_w8a8(L.W, a, 16, bias_bits=L.b)
    q = oracle.pack_weights(L.W, a, 16, bias_bits=L.b)
    for k in ("inv_lambda", "L1b", "L2b", "R", "bias"):
        assert np.array_equal(p[k], q[k]), k
    Rt = oracle.round_f32(p["R"].T)                                  # [N, K]
    assert p["wcodes8"].shape == Rt.shape and p["s_w8"].shape == (Rt.shape[0],)
    err = np.abs(Rt - p["wcodes8"] * p["s_w8"][:, None])
    assert np.all(err <= p["s_w8"][:, None] / 2)
    assert np.all(np.max(np.abs(p["wcodes8"]), axis=1) == 127)


def test_w8a8_layer_is_closer_than_w4a4(tiny):
    """Eight-bit operands with the same smoothing and factors land closer to
    X W than the four-bit group format on the outlier workload."""
    L = tiny
    X = oracle.bf16_bits_to_f64(L.X)
    ref = X @ oracle.bf16_bits_to_f64(L.W).T
    a = oracle.calib_absmax(X)
    p8 = oracle.pack_weights_w8a8(L.W, a, 16)
    xc, s_x, Z, _ = oracle.quantize_act_w8a8(L.X, p8["inv_lambda"], p8["L1b"])
    Y8, _ = oracle.linear_w8a8(xc, s_x, Z, p8["wcodes8"], p8["s_w8"], p8["L2b"], p8["bias"])
    e8 = np.linalg.norm(Y8 - ref) / np.linalg.norm(ref)
    e4 = oracle.layer_output_error(L.X, oracle.pack_weights(L.W, a, 16), L.W)
    assert e8 < e4 / 4
    assert e8 < 0.05


def test_w8a8_activation_side(tiny):
    L = tiny
    a = oracle.calib_absmax(oracle.bf16_bits_to_f64(L.X))
    p = oracle.pack_weights_w8a8(L.W, a, 16)
    xc, s_x, Z, xhat = oracle.quantize_act_w8a8(L.X, p["inv_lambda"], p["L1b"])
    # x~ and Z are the four-bit path's; only the quantiser differs
    _, _, Z4, xhat4 = oracle.quantize_act(L.X, p["inv_lambda"], p["L1b"])
    assert np.array_equal(xhat, xhat4) and np.array_equal(Z, Z4)
    for i in (0, 5, L.X.shape[0] - 1):
        assert s_x[i] == _scale_f32(xhat[i])
