"""The library's host pack against the oracle on seeded random shapes, by
the two-level rule for factors that any SVD may return up to sign and
rounding: the singular values agree to 1e-10, and, given the library's own
exported bf16 factors, the oracle's residual quantisation (eq. 10, then
eq. 1 per group) reproduces the library's weight codes and scales bit for
bit."""
import numpy as np
import pytest

import oracle
import synth
import w4a4_quantized_gemm_smooth_b200 as S


def _cases(n=8, seed=2024):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        K = 64 * int(rng.integers(1, 13))
        N = 8 * int(rng.integers(2, 51))
        rmax = min(32, (min(K, N) - 1) // 8 * 8)
        r = 8 * int(rng.integers(0, rmax // 8 + 1))
        alpha = float(rng.choice([0.5, 0.4, 0.6]))
        out.append((K, N, r, alpha, 5000 + i))
    return out


@pytest.mark.parametrize("K,N,r,alpha,seed", _cases())
def test_host_pack_two_level_parity(K, N, r, alpha, seed):
    L = synth.make_layer(synth.layer_spec(f"rp{seed}", 32, K, N, r, seed, tiny=(K <= 512)))
    a = S.svdq_calib_absmax(L.X)
    w = S.svdq_pack_weights_host(L.W, a, r, alpha=alpha, bias_bits=L.b)
    e = w.export()
    W = oracle.bf16_bits_to_f64(L.W).T                              # [K, N]
    lam = oracle.smoothing_lambda(a.astype(np.float64), np.max(np.abs(W), axis=1), alpha)
    assert np.array_equal(e["inv_lambda"].astype(np.float64), oracle.round_f32(1.0 / lam))
    Wt = lam[:, None] * W
    sv = np.linalg.svd(Wt, compute_uv=False)
    assert np.max(np.abs(e["sigma"] - sv[:r + 1]) / sv[:r + 1]) < 1e-10
    L1b = oracle.bf16_bits_to_f64(e["L1"])[:, :r]
    L2b = oracle.bf16_bits_to_f64(e["L2"])[:r]
    _, codes, s_w = oracle.residual_quantize(Wt, L1b, L2b)
    assert np.array_equal(e["wq"], oracle.pack_nibbles(codes))
    assert np.array_equal(e["s_w"].astype(np.float64), s_w)
    w.free()


def _residual_from_library(L, a, e, r, alpha):
    W = oracle.bf16_bits_to_f64(L.W).T
    lam = oracle.smoothing_lambda(a.astype(np.float64), np.max(np.abs(W), axis=1), alpha)
    assert np.array_equal(e["inv_lambda"].astype(np.float64), oracle.round_f32(1.0 / lam))
    L1b = oracle.bf16_bits_to_f64(e["L1"])[:, :r]
    L2b = oracle.bf16_bits_to_f64(e["L2"])[:r]
    R, _, _ = oracle.residual_quantize(lam[:, None] * W, L1b, L2b)
    return oracle.round_f32(R.T)


@pytest.mark.parametrize("K,N,r,alpha,seed", _cases(6, seed=77))
def test_w8a8_host_pack_two_level_parity(K, N, r, alpha, seed):
    L = synth.make_layer(synth.layer_spec(f"r8{seed}", 32, K, N, r, seed, tiny=(K <= 512)))
    a = S.svdq_calib_absmax(L.X)
    w = S.svdq_pack_weights_w8a8(L.W, a, r, alpha=alpha, bias_bits=L.b, to_device=False)
    e = w.export()
    codes8, s_w8 = oracle.quantize_rows_int8(_residual_from_library(L, a, e, r, alpha))
    assert np.array_equal(e["wq8"].astype(np.int64), codes8)
    assert np.array_equal(e["s_w8"].astype(np.float64), s_w8)
    w.free()


@pytest.mark.parametrize("K,N,r,alpha,seed", _cases(6, seed=78))
def test_nvfp4_host_pack_two_level_parity(K, N, r, alpha, seed):
    L = synth.make_layer(synth.layer_spec(f"r4{seed}", 32, K, N, r, seed, tiny=(K <= 512)))
    a = S.svdq_calib_absmax(L.X)
    w = S.svdq_pack_weights_nvfp4(L.W, a, r, alpha=alpha, bias_bits=L.b, to_device=False)
    e = w.export()
    codes, b, s = oracle.quantize_nvfp4_rows(_residual_from_library(L, a, e, r, alpha))
    assert np.array_equal(e["wq4"], oracle.pack_nibbles(codes))
    assert np.array_equal(e["sf4"], oracle.e4m3_bits(b))
    assert np.array_equal(e["s_w4"].astype(np.float64), s)
    w.free()


def _gptq_cases(n=4, seed=99):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        K = 64 * int(rng.integers(1, 9))
        N = 8 * int(rng.integers(2, 30))
        r = 8 * int(rng.integers(0, min(4, (min(K, N) - 1) // 8) + 1))
        out.append((K, N, r, 600 + i))
    return out


@pytest.mark.parametrize("K,N,r,seed", _gptq_cases())
def test_gptq_host_pack_two_level_parity(K, N, r, seed):
    """The calibrated pack with GPTQ rounding (one alpha, no refinement):
    given the library's factors and the calibration Hessian, the oracle's
    GPTQ gives the library's codes and scales bit for bit."""
    L = synth.make_layer(synth.layer_spec(f"gq{seed}", 96, K, N, r, seed, tiny=(K <= 512)))
    w, _ = S.svdq_pack_weights_calibrated(L.W, L.X, r, alphas=(0.5,), refine_iters=0,
                                          bias_bits=L.b, to_device=False, gptq=True)
    e = w.export()
    W = oracle.bf16_bits_to_f64(L.W).T
    a = oracle.calib_absmax(oracle.bf16_bits_to_f64(L.X))
    lam = oracle.smoothing_lambda(a, np.max(np.abs(W), axis=1), 0.5)
    assert np.array_equal(e["inv_lambda"].astype(np.float64), oracle.round_f32(1.0 / lam))
    L1b = oracle.bf16_bits_to_f64(e["L1"])[:, :r]
    L2b = oracle.bf16_bits_to_f64(e["L2"])[:r]
    R, _, _ = oracle.residual_quantize(lam[:, None] * W, L1b, L2b)
    codes, s_w = oracle.gptq_quantize_residual(R, oracle.gptq_hessian(L.X, e["inv_lambda"]))
    assert np.array_equal(e["wq"], oracle.pack_nibbles(codes))
    assert np.array_equal(e["s_w"].astype(np.float64), s_w)
    w.free()


@pytest.mark.parametrize("K,N,r,seed", [c for c in _gptq_cases(6, seed=101) if c[2] > 0][:4])
def test_refined_host_pack_two_level_parity(K, N, r, seed):
    """The calibrated pack with one alternating refinement: the library's
    final (refined) factors give, through the oracle's residual
    quantisation, the library's codes and scales bit for bit."""
    L = synth.make_layer(synth.layer_spec(f"rf{seed}", 96, K, N, r, seed, tiny=(K <= 512)))
    w, _ = S.svdq_pack_weights_calibrated(L.W, L.X, r, alphas=(0.5,), refine_iters=1,
                                          bias_bits=L.b, to_device=False)
    e = w.export()
    W = oracle.bf16_bits_to_f64(L.W).T
    a = oracle.calib_absmax(oracle.bf16_bits_to_f64(L.X))
    lam = oracle.smoothing_lambda(a, np.max(np.abs(W), axis=1), 0.5)
    Wt = lam[:, None] * W
    L1b = oracle.bf16_bits_to_f64(e["L1"])[:, :r]
    L2b = oracle.bf16_bits_to_f64(e["L2"])[:r]
    _, codes, s_w = oracle.residual_quantize(Wt, L1b, L2b)
    assert np.array_equal(e["wq"], oracle.pack_nibbles(codes))
    assert np.array_equal(e["s_w"].astype(np.float64), s_w)
    w.free()
