"""Pins of the oracle's calibration refinement (SVDQuant review section 5:
alpha chosen by the calibrated layer-output error; protected factors
re-fitted to W~ - Q(R), the residual recomputed against W~)."""
import numpy as np
import pytest

import oracle
import synth


@pytest.fixture(scope="module")
def tiny():
    return synth.make_layer(synth.WORKLOADS["tiny"])


def test_single_alpha_without_refinement_is_the_plain_pack(tiny):
    L = tiny
    p, errs = oracle.pack_weights_calibrated(L.W, L.X, 16, alphas=(0.5,), iters=0, bias_bits=L.b)
    q = oracle.pack_weights(L.W, oracle.calib_absmax(oracle.bf16_bits_to_f64(L.X)), 16,
                            bias_bits=L.b)
    for k in ("inv_lambda", "wq", "s_w", "L1b", "L2b", "bias"):
        assert np.array_equal(p[k], q[k]), k
    assert len(errs) == 1


def test_error_is_the_dense_dequantised_product(tiny):
    """layer_output_error against the plain definition: deq(Q(X~)) deq(Q(R))
    + Z L2 as dense fp64 matrices, compared with X W."""
    L = tiny
    p = oracle.pack_weights(L.W, oracle.calib_absmax(oracle.bf16_bits_to_f64(L.X)), 16)
    xc, s_x, Z, _ = oracle.quantize_act(L.X, p["inv_lambda"], p["L1b"])
    Xq = oracle.dequantize_groups(xc, s_x)                     # [M, K]
    Rq = oracle.dequantize_groups(p["wcodes"], p["s_w"])       # [N, K]
    Yq = Xq @ Rq.T + Z @ p["L2b"]
    ref = oracle.bf16_bits_to_f64(L.X) @ oracle.bf16_bits_to_f64(L.W).T
    expect = np.linalg.norm(Yq - ref) / np.linalg.norm(ref)
    assert oracle.layer_output_error(L.X, p, L.W) == pytest.approx(expect, rel=1e-12)


def test_refined_factors_are_the_best_rank_r_fit_of_w_minus_qr(tiny):
    L = tiny
    p0 = oracle.pack_weights(L.W, oracle.calib_absmax(oracle.bf16_bits_to_f64(L.X)), 16)
    p1 = oracle.refine_factors(p0)
    T = p0["Wt"] - oracle.dequantize_groups(p0["wcodes"], p0["s_w"]).T
    S = np.linalg.svd(T, compute_uv=False)
    resid = np.linalg.norm(T - p1["L1"] @ p1["L2"]) ** 2
    # Eckart-Young for T itself: a fit of W~ or of W~ + Q(R), or of the wrong
    # rank, would leave a larger remainder of T than its tail energy
    assert resid == pytest.approx(np.sum(S[16:] ** 2), rel=1e-9)
    # the residual is recomputed against W~ and the stored bf16 factors
    err = np.max(np.abs(p1["L1b"] @ p1["L2b"] + p1["R"] - p0["Wt"]))
    assert err <= 1e-14 * np.max(np.abs(p0["Wt"]))


def test_refinement_lowers_the_calibrated_error_on_outlier_data(tiny):
    L = tiny
    _, e0 = oracle.pack_weights_calibrated(L.W, L.X, 16, alphas=(0.5,), iters=0)
    _, e1 = oracle.pack_weights_calibrated(L.W, L.X, 16, alphas=(0.5,), iters=1)
    assert e1[0] < e0[0]


def test_the_smallest_error_wins(tiny):
    L = tiny
    alphas = (0.3, 0.5, 0.7)
    p, errs = oracle.pack_weights_calibrated(L.W, L.X, 16, alphas=alphas, iters=0)
    assert p["alpha"] == alphas[int(np.argmin(errs))]
    for a, e in zip(alphas, errs):
        q, (e2,) = oracle.pack_weights_calibrated(L.W, L.X, 16, alphas=(a,), iters=0)
        assert e2 == e
