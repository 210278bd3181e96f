"""Pins of the oracle's smoothing, SVD, residual, two-branch product and LoRA
steps against the identities of the SVDQuant technical review:
eq. 3 (section 3.1), eqs. 5-8 (section 4), eq. 10 + Eckart-Young (section 5),
eq. 13 (section 7), plus brute force on tiny inputs.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth


@pytest.fixture(scope="module")
def tiny():
    L = synth.make_layer(synth.WORKLOADS["tiny"])
    X = oracle.bf16_bits_to_f64(L.X)
    a = oracle.calib_absmax(X)
    p = oracle.pack_weights(L.W, a, 16, bias_bits=L.b)
    return L, X, a, p


def _rel(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


def test_calib_absmax_brute_force():
    X = np.array([[1.0, -3.0], [-2.0, 0.5], [0.25, 2.0]])
    assert list(oracle.calib_absmax(X)) == [2.0, 3.0]


def test_lambda_rule_values():
    lam = oracle.smoothing_lambda(np.array([4.0, 9.0, 0.0, 2.0]),
                                  np.array([1.0, 4.0, 3.0, 0.0]), 0.5)
    assert list(lam) == [2.0, 1.5, 1.0, 1.0]
    lam = oracle.smoothing_lambda(np.array([8.0]), np.array([4.0]), 0.25)
    assert abs(lam[0] - 8.0 ** 0.25 / 4.0 ** 0.75) < 1e-15


def test_smoothing_identity_eq3(tiny):
    L, X, a, p = tiny
    W = oracle.bf16_bits_to_f64(L.W).T
    lam = p["lam"]
    Xt = X / lam[None, :]
    assert _rel(Xt @ p["Wt"], X @ W) < 1e-12
    # a planted mistake (lambda applied along the output axis) breaks it
    bad_Wt = W * lam[:W.shape[1]][None, :] if W.shape[1] == W.shape[0] else None
    if bad_Wt is not None:
        assert _rel(Xt @ bad_Wt, X @ W) > 1e-3


def test_residual_identity_eq10(tiny):
    _, _, _, p = tiny
    # with the stored 16-bit factors (the deployed decomposition)
    assert np.max(np.abs(p["L1b"] @ p["L2b"] + p["R"] - p["Wt"])) <= 1e-12 * np.max(np.abs(p["Wt"]))
    # a residual with the wrong sign fails the same check
    bad_R = p["Wt"] + p["L1b"] @ p["L2b"]
    assert np.max(np.abs(p["L1b"] @ p["L2b"] + bad_R - p["Wt"])) > 1e-3


def test_spectral_norm_and_eckart_young(tiny):
    _, _, _, p = tiny
    r = 16
    R_exact = p["Wt"] - p["L1"] @ p["L2"]
    S = p["S"]
    assert abs(np.linalg.norm(R_exact, 2) - S[r]) <= 1e-10 * S[r]
    assert abs(np.linalg.norm(R_exact, "fro") ** 2 - np.sum(S[r:] ** 2)) <= 1e-10 * np.sum(S[r:] ** 2)
    assert np.isclose(p["sigma"][-1], S[r])
    # an independent routine: a power iteration on R^T R approaches the
    # spectral norm from below and never exceeds it
    rng = np.random.default_rng(0)
    v = rng.standard_normal(R_exact.shape[1])
    for _ in range(300):
        v = R_exact.T @ (R_exact @ v)
        v /= np.linalg.norm(v)
    est = np.linalg.norm(R_exact @ v)
    assert S[r] * (1 - 1e-4) <= est <= S[r] * (1 + 1e-12)


def test_rank0_without_quantisation_is_xw_plus_b(tiny):
    L, X, a, _ = tiny
    p0 = oracle.pack_weights(L.W, a, 0, bias_bits=L.b)
    W = oracle.bf16_bits_to_f64(L.W).T
    b = oracle.bf16_bits_to_f64(L.b)
    y = oracle.two_branch_unquantized(X, p0["lam"], p0["L1"], p0["L2"], p0["Wt"], b)
    assert _rel(y, X @ W + b) < 1e-12
    # and with the rank-16 split, still exact before quantisation
    p = oracle.pack_weights(L.W, a, 16, bias_bits=L.b)
    y = oracle.two_branch_unquantized(X, p["lam"], p["L1"], p["L2"],
                                      p["Wt"] - p["L1"] @ p["L2"], b)
    assert _rel(y, X @ W + b) < 1e-12


def test_partials_equal_dense_dequantised_product(tiny):
    L, X, a, p = tiny
    xc, s_x, Z, xhat = oracle.quantize_act(L.X, p["inv_lambda"], p["L1b"])
    Y, _ = oracle.linear(xc, s_x, np.zeros((X.shape[0], 0)), p["wcodes"], p["s_w"],
                         np.zeros((0, p["N"])), np.zeros(p["N"]))
    Qx = oracle.dequantize_groups(xc, s_x)
    Qw = oracle.dequantize_groups(p["wcodes"], p["s_w"])
    assert _rel(Y, Qx @ Qw.T) < 1e-12
    # brute force int64 partials on a corner
    P = oracle.group_partials(xc, p["wcodes"], rows=np.arange(5), cols=np.arange(7))
    for g in range(P.shape[0]):
        sl = slice(64 * g, 64 * g + 64)
        ref = xc[:5, sl].astype(np.int64) @ p["wcodes"][:7, sl].astype(np.int64).T
        assert np.array_equal(P[g], ref)


def test_activation_quantiser_tiny_brute_force():
    rng = np.random.default_rng(4)
    X = synth.f64_to_bf16_bits(rng.standard_normal((3, 128)) * 4)
    inv = oracle.round_f32(1.0 / np.exp(rng.normal(0, 1, 128)))
    L1b = oracle.round_bf16(rng.standard_normal((128, 2)))
    xc, s_x, Z, xhat = oracle.quantize_act(X, inv, L1b)
    Xf = oracle.bf16_bits_to_f64(X)
    for i in range(3):
        for k in range(128):
            # x~ = one fp32 rounding of the exact product
            assert xhat[i, k] == float(np.float32(float(Fraction(Xf[i, k]) * Fraction(inv[k]))))
        for j in range(2):
            acc = sum(Fraction(float(oracle.round_bf16(np.array([xhat[i, k]]))[0])) * Fraction(L1b[k, j])
                      for k in range(128))
            assert Z[i, j] == oracle.round_bf16(np.array([float(acc)]))[0]
        for g in range(2):
            m = max(abs(xhat[i, 64 * g:64 * g + 64]))
            assert s_x[g, i] == float(np.float32(m / 7.0))


def test_linear_tiny_brute_force():
    rng = np.random.default_rng(8)
    M, K, N, r = 2, 128, 3, 2
    xc = rng.integers(-7, 8, (M, K))
    wc = rng.integers(-7, 8, (N, K))
    s_x = oracle.round_f32(rng.uniform(0.1, 1, (2, M)))
    s_w = oracle.round_f32(rng.uniform(0.1, 1, (2, N)))
    Z = oracle.round_bf16(rng.standard_normal((M, r)))
    L2 = oracle.round_bf16(rng.standard_normal((r, N)))
    b = oracle.round_bf16(rng.standard_normal(N))
    Y, Yb = oracle.linear(xc, s_x, Z, wc, s_w, L2, b)
    for i in range(M):
        for n in range(N):
            acc = Fraction(b[n])
            for g in range(2):
                Pg = sum(int(xc[i, k]) * int(wc[n, k]) for k in range(64 * g, 64 * g + 64))
                acc += Fraction(s_x[g, i]) * Fraction(s_w[g, n]) * Pg
            acc += sum(Fraction(Z[i, j]) * Fraction(L2[j, n]) for j in range(r))
            assert abs(Y[i, n] - float(acc)) <= 1e-15 * abs(float(acc)) + 1e-300
    Yg, _ = oracle.linear(xc, s_x, Z, wc, s_w, L2, b, apply_gelu=True)
    assert np.allclose(Yg, 0.5 * Y * (1 + np.vectorize(math.erf)(Y / math.sqrt(2))), rtol=1e-15, atol=0)


def test_gelu_special_values():
    y = np.array([0.0, 10.0, -10.0, 1.0])
    g = oracle.gelu(y)
    assert g[0] == 0.0 and abs(g[1] - 10.0) < 1e-20 and abs(g[2]) < 1e-20
    assert abs(g[3] - 0.8413447460685429) < 1e-15
    x = np.linspace(-3, 3, 13)
    assert np.allclose(oracle.gelu(x) - oracle.gelu(-x), x, rtol=0, atol=1e-15)


def test_ablation_ordering(tiny):
    """Table 3 direction and the eq. 8 argument: on outlier inputs the full
    method beats smoothing-only W4A4, which beats plain W4A4."""
    L, X, a, p = tiny
    W = oracle.bf16_bits_to_f64(L.W).T
    b = oracle.bf16_bits_to_f64(L.b)
    ref = X @ W + b
    e_full = _rel(oracle.layer_forward(L.X, p)["Y"], ref)
    p0 = oracle.pack_weights(L.W, a, 0, bias_bits=L.b)
    e_smooth = _rel(oracle.layer_forward(L.X, p0)["Y"], ref)
    pn = oracle.pack_weights(L.W, a, 0, bias_bits=L.b, smooth=False)
    e_plain = _rel(oracle.layer_forward(L.X, pn)["Y"], ref)
    assert e_full < e_smooth < e_plain
    assert e_full < 0.08


def test_product_error_bound_eq6(tiny):
    L, X, a, p = tiny
    xc, s_x, _, xhat = oracle.quantize_act(L.X, p["inv_lambda"], p["L1b"])
    Qx = oracle.dequantize_groups(xc, s_x)
    R32 = oracle.round_f32(p["R"])
    QR = oracle.dequantize_groups(p["wcodes"], p["s_w"]).T
    lhs = np.linalg.norm(xhat @ R32 - Qx @ QR)
    dW = np.linalg.norm(R32 - QR)
    dX = np.linalg.norm(xhat - Qx)
    rhs = np.linalg.norm(xhat) * dW + dX * (np.linalg.norm(R32) + dW)
    assert lhs <= rhs


def test_lora_identity_eq13():
    spec = synth.layer_spec("lora", 64, 256, 128, 8, 77, lora_rank=4, tiny=True)
    L = synth.make_layer(spec)
    X = oracle.bf16_bits_to_f64(L.X)
    a = oracle.calib_absmax(X)
    p = oracle.pack_weights(L.W, a, 8, bias_bits=L.b, lora_A_bits=L.A, lora_B_bits=L.B)
    A = oracle.bf16_bits_to_f64(L.A)
    B = oracle.bf16_bits_to_f64(L.B)
    lam = p["lam"]
    W = oracle.bf16_bits_to_f64(L.W).T
    # D (W + A B) = D W + (D A) B
    assert _rel(lam[:, None] * (W + A @ B), p["Wt"] + (lam[:, None] * A) @ B) < 1e-12
    # the stored branch holds [L1 | D A] and [L2 ; B]
    assert p["L1b"].shape[1] == 12 and p["L2b"].shape[0] == 12
    assert np.array_equal(p["L1b"][:, 8:], oracle.round_bf16(lam[:, None] * A))
    assert np.array_equal(p["L2b"][8:], B)
    # before quantisation the adapted layer is X(W + AB) + b
    b = oracle.bf16_bits_to_f64(L.b)
    Xt = X / lam[None, :]
    y = Xt @ (p["Wt"] - p["L1"] @ p["L2"]) + (Xt @ np.hstack([p["L1"], lam[:, None] * A])) @ \
        np.vstack([p["L2"], B]) + b
    assert _rel(y, X @ (W + A @ B) + b) < 1e-12


def test_leading_svd_matches_full_svd(tiny):
    """The ARPACK path used for large layers agrees with LAPACK's full SVD."""
    L, X, a, p = tiny
    q = oracle.pack_weights(L.W, a, 16, bias_bits=L.b, svd="leading")
    assert np.max(np.abs(q["sigma"] - p["sigma"]) / p["sigma"]) < 1e-12
    assert np.array_equal(np.abs(q["L1b"]), np.abs(p["L1b"]))
    assert np.array_equal(q["wq"], p["wq"]) and np.array_equal(q["s_w"], p["s_w"])


def _lora_identity_err(p, X, W, A, B, b, s):
    """Relative error between the unquantised two-branch layer built from the
    stored factors (eq. 7 with quantisation off: [L1 | s D A] and [L2 ; B]
    joined to the residual) and the adapted layer's definition X (W + s A B) + b
    (eq. 13)."""
    R = p["Wt"] - p["L1b"][:, :p["rank"] - A.shape[1]] @ p["L2b"][:p["rank"] - A.shape[1]]
    y = oracle.two_branch_unquantized(X, p["lam"], p["L1b"], p["L2b"], R, b)
    return _rel(y, X @ (W + float(np.float32(s)) * (A @ B)) + b)


def _lora_placement_ok(p, lam, A, B, s, r):
    """eq. 13 puts the adapter on the smoothed side: the stored low-rank
    factors end with bf16(s D A) and with B unchanged."""
    return (np.array_equal(p["L1b"][:, r:], oracle.round_bf16(lam[:, None] * A * float(np.float32(s))))
            and np.array_equal(p["L2b"][r:], B))


@pytest.mark.parametrize("scale", [0.3, 2.5, -0.75])
def test_lora_scale_eq13(scale):
    """LoRA scale s != 1: D (W + s A B) = D W + (s D A) B (eq. 13), the stored
    factors hold s on the A side, and two planted mistakes fail the checks:
    the scale applied to B instead, and the scale dropped."""
    spec = synth.layer_spec("lora_s", 64, 256, 128, 8, 78, lora_rank=4, tiny=True)
    L = synth.make_layer(spec)
    X = oracle.bf16_bits_to_f64(L.X)
    a = oracle.calib_absmax(X)
    A = oracle.bf16_bits_to_f64(L.A) * 40.0          # an adapter term that matters
    B = oracle.bf16_bits_to_f64(L.B) * 40.0
    Ab, Bb = oracle.round_bf16_bits(A), oracle.round_bf16_bits(B)
    A, B = oracle.bf16_bits_to_f64(Ab), oracle.bf16_bits_to_f64(Bb)
    W = oracle.bf16_bits_to_f64(L.W).T
    b = oracle.bf16_bits_to_f64(L.b)
    p = oracle.pack_weights(L.W, a, 8, bias_bits=L.b, lora_A_bits=Ab, lora_B_bits=Bb,
                            lora_scale=scale)
    lam = p["lam"]
    s32 = float(np.float32(scale))
    assert _rel(lam[:, None] * (W + s32 * A @ B), p["Wt"] + (s32 * lam[:, None] * A) @ B) < 1e-12
    assert _lora_placement_ok(p, lam, A, B, scale, 8)
    # only the bf16 rounding of the factors separates the two (eq. 10 residual
    # is taken against the stored SVD factors, so that part is exact)
    err = _lora_identity_err(p, X, W, A, B, b, scale)
    assert err < 2.0 ** -8, err
    # mistake 1: the scale applied to B (same product, wrong placement)
    bad = dict(p)
    bad["L1b"] = np.hstack([p["L1b"][:, :8], oracle.round_bf16(lam[:, None] * A)])
    bad["L2b"] = np.vstack([p["L2b"][:8], oracle.round_bf16(s32 * B)])
    assert not _lora_placement_ok(bad, lam, A, B, scale, 8)
    # mistake 2: the scale dropped (the layer no longer matches its definition)
    drop = dict(p)
    drop["L1b"] = np.hstack([p["L1b"][:, :8], oracle.round_bf16(lam[:, None] * A)])
    assert _lora_identity_err(drop, X, W, A, B, b, scale) > 1e-2
