"""Pins of the oracle's GPTQ residual rounding (SVDQuant review section 8:
"residual weights use GPTQ"; the published algorithm of Frantar et al.).
The Cholesky form is checked against the closed form for a diagonal Hessian
(plain rounding), against an independent optimal-brain-surgeon form that
re-inverts the remaining Hessian at every step, and for the property GPTQ is
for: a smaller calibrated layer error than plain rounding."""
import numpy as np
import pytest

import oracle
import synth


def _plain(R):
    N = R.shape[1]
    K = R.shape[0]
    codes, s = oracle.quantize_groups(oracle.round_f32(R.T).reshape(N, K // 64, 64))
    return codes.reshape(N, K), s.T


def test_diagonal_hessian_is_plain_rounding():
    rng = np.random.default_rng(10)
    R = rng.standard_normal((192, 6)) * 0.05
    H = np.diag(rng.uniform(0.5, 4.0, 192))
    c, s = oracle.gptq_quantize_residual(R, H)
    c0, s0 = _plain(R)
    assert np.array_equal(c, c0) and np.array_equal(s, s0)


def _obs_reference(R, H, damp=0.01):
    """Sequential optimal-brain-surgeon updates with the inverse of the
    remaining (dampened) Hessian recomputed at every step."""
    R = np.array(R, dtype=np.float64, copy=True)
    K, N = R.shape
    Hd = H + damp * np.mean(np.diag(H)) * np.eye(K)
    codes = np.zeros((N, K), dtype=np.int64)
    s_w = np.zeros((K // 64, N))
    for k in range(K):
        g = k // 64
        if k % 64 == 0:
            _, s_w[g] = oracle.quantize_groups(oracle.round_f32(R[k:k + 64].T))
        s = s_w[g]
        w32 = oracle.round_f32(R[k])
        q = np.zeros(N, dtype=np.int64)
        for n in range(N):
            if s[n] > 0:
                # round half to even of w / s, decided by exact comparisons
                q[n] = int(np.clip(np.rint(w32[n] / s[n]), -8, 7))
                lo, hi = (q[n] - 0.5) * s[n], (q[n] + 0.5) * s[n]
                if w32[n] > hi or (w32[n] == hi and q[n] % 2):
                    q[n] += 1
                elif w32[n] < lo or (w32[n] == lo and q[n] % 2):
                    q[n] -= 1
                q[n] = int(np.clip(q[n], -8, 7))
        codes[:, k] = q
        Hinv = np.linalg.inv(Hd[k:, k:])
        delta = (R[k] - q * s) / Hinv[0, 0]
        R[k + 1:] -= np.outer(Hinv[1:, 0], delta)
    return codes, s_w


def test_cholesky_form_matches_the_sequential_obs_form():
    rng = np.random.default_rng(11)
    X = rng.standard_normal((300, 128)) @ rng.standard_normal((128, 128)) * 0.3   # correlated
    H = X.T @ X
    R = rng.standard_normal((128, 4)) * 0.05
    c, s = oracle.gptq_quantize_residual(R, H)
    c1, s1 = _obs_reference(R, H)
    assert np.array_equal(s, s1)
    assert np.array_equal(c, c1)


def test_gptq_lowers_the_calibrated_error():
    L = synth.make_layer(synth.WORKLOADS["tiny"])
    _, e_rtn = oracle.pack_weights_calibrated(L.W, L.X, 16, alphas=(0.5,), iters=0)
    _, e_gptq = oracle.pack_weights_calibrated(L.W, L.X, 16, alphas=(0.5,), iters=0, gptq=True)
    assert e_gptq[0] < e_rtn[0]


def test_dead_channel_keeps_plain_rounding():
    """A channel the calibration never activates (H_kk = 0, its row and
    column zero) passes no error on and is rounded plainly."""
    rng = np.random.default_rng(12)
    X = rng.standard_normal((200, 64))
    X[:, 0] = 0.0
    H = X.T @ X
    R = rng.standard_normal((64, 3)) * 0.05
    c, _ = oracle.gptq_quantize_residual(R, H)
    c0, _ = _plain(R)
    assert np.array_equal(c[:, 0], c0[:, 0])
