"""The library's calibrated pack (svdq_pack_weights_calibrated, host only)
against the oracle's pack_weights_calibrated: the candidates' calibrated
errors, the chosen alpha, and the packed layer (lambda, factors up to sign,
residual codes and scales bit for bit)."""
import numpy as np
import pytest

import oracle
import synth
import w4a4_quantized_gemm_smooth_b200 as S
from helpers import column_signs


@pytest.mark.parametrize("case", ["tiny", "lora", "tall"])
def test_calibrated_pack_matches_oracle(case):
    if case == "tiny":
        spec = synth.WORKLOADS["tiny"]
    elif case == "lora":
        spec = synth.layer_spec("cal_lora", 128, 384, 256, 16, 41, lora_rank=8)
    else:
        spec = synth.layer_spec("cal_tall", 96, 640, 192, 24, 42)
    L = synth.make_layer(spec)
    alphas = (0.3, 0.5, 0.7)
    w, errs = S.svdq_pack_weights_calibrated(L.W, L.X, spec.rank, alphas=alphas, refine_iters=1,
                                             bias_bits=L.b, lora_A_bits=L.A, lora_B_bits=L.B,
                                             to_device=False)
    p, errs_o = oracle.pack_weights_calibrated(L.W, L.X, spec.rank, alphas=alphas, iters=1,
                                               bias_bits=L.b, lora_A_bits=L.A, lora_B_bits=L.B)
    assert np.allclose(errs, errs_o, rtol=1e-6, atol=0)
    assert alphas[int(np.argmin(errs))] == p["alpha"]
    e = w.export()
    assert np.array_equal(e["inv_lambda"].astype(np.float64), p["inv_lambda"])
    sg = column_signs(e["L1"], p["L1b"])
    assert np.array_equal(oracle.bf16_bits_to_f64(e["L1"]) * sg[None, :], p["L1b"])
    assert np.array_equal(oracle.bf16_bits_to_f64(e["L2"]) * sg[:, None], p["L2b"])
    assert np.array_equal(e["wq"], p["wq"])
    assert np.array_equal(e["s_w"].astype(np.float64), p["s_w"])
    assert np.array_equal(e["bias"], L.b)
    w.free()


@pytest.mark.parametrize("case", ["tiny", "tall"])
def test_gptq_pack_matches_oracle(case):
    """GPTQ rounding of the residual (with one refinement step, which rounds
    the refined residual by GPTQ again): the library's host Cholesky and the
    oracle's LAPACK one give the same codes and scales."""
    if case == "tiny":
        spec = synth.WORKLOADS["tiny"]
    else:
        spec = synth.layer_spec("gq_tall", 96, 640, 192, 24, 43)
    L = synth.make_layer(spec)
    alphas = (0.4, 0.6)
    w, errs = S.svdq_pack_weights_calibrated(L.W, L.X, spec.rank, alphas=alphas, refine_iters=1,
                                             bias_bits=L.b, to_device=False, gptq=True)
    p, errs_o = oracle.pack_weights_calibrated(L.W, L.X, spec.rank, alphas=alphas, iters=1,
                                               bias_bits=L.b, gptq=True)
    assert np.allclose(errs, errs_o, rtol=1e-6, atol=0)
    assert alphas[int(np.argmin(errs))] == p["alpha"]
    e = w.export()
    assert np.array_equal(e["wq"], p["wq"])
    assert np.array_equal(e["s_w"].astype(np.float64), p["s_w"])
    # and GPTQ beats rounding to nearest on the calibrated error
    _, errs_rtn = S.svdq_pack_weights_calibrated(L.W, L.X, spec.rank, alphas=alphas, refine_iters=1,
                                                 to_device=False)
    assert min(errs) < min(errs_rtn)
    w.free()


def test_one_alpha_without_refinement_is_the_plain_pack():
    L = synth.make_layer(synth.WORKLOADS["tiny"])
    w, errs = S.svdq_pack_weights_calibrated(L.W, L.X, 16, alphas=(0.5,), refine_iters=0,
                                             bias_bits=L.b, to_device=False)
    w0 = S.svdq_pack_weights_host(L.W, S.svdq_calib_absmax(L.X), 16, bias_bits=L.b)
    e, e0 = w.export(), w0.export()
    for k in e:
        assert np.array_equal(e[k], e0[k]), k
    assert errs.shape == (1,) and 0 < errs[0] < 1
    w.free()
    w0.free()


def test_calibrated_pack_argument_errors():
    L = synth.make_layer(synth.WORKLOADS["tiny"])
    for bad in ((0.5, 1.0), (0.0,), ()):
        with pytest.raises(S.SVDQError):
            S.svdq_pack_weights_calibrated(L.W, L.X, 16, alphas=bad, to_device=False)
    with pytest.raises(S.SVDQError):
        S.svdq_pack_weights_calibrated(L.W, L.X, 16, refine_iters=-1, to_device=False)
