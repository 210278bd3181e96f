"""GPU parity of the W8A8 comparator (svdq_quantize_act_w8a8 then
svdq_linear_w8a8) against the oracle's W8A8 functions on the same seeded
inputs.

Bar: int8 activation codes and per-token scales bit-exact; weight codes and
per-channel scales bit-exact; Z within one bf16 ulp plus the fp32
accumulation bound; Y within 2e-3 relative Frobenius error of the oracle's
bf16 Y computed from the GPU's own Z (the oracle's codes and scales equal the
GPU's)."""
import numpy as np
import pytest
import torch

import oracle
import synth
import w4a4_quantized_gemm_smooth_b200 as S
from helpers import Y_REL_FRO, check_z, column_signs, rel_fro

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "gpu tests need a CUDA device"
    S.lib()


def _to_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)) \
        .view(torch.bfloat16).cuda()


def _bits(t):
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _run(w, Xb, epilogue):
    lin = S.W8A8Linear(w, epilogue)
    xq, s_x, Z, Y = lin.buffers(Xb.shape[0])
    lin.forward(_to_dev(Xb), out=Y)
    torch.cuda.synchronize()
    S.svdq_get_device_error(w)
    return xq.cpu().numpy().astype(np.int64), s_x.cpu().numpy().astype(np.float64), Z, _bits(Y)


def check_w8a8(spec, epilogue=S.EPI_NONE, X_bits=None):
    L = synth.make_layer(spec)
    Xb = L.X if X_bits is None else X_bits
    a = S.svdq_calib_absmax(Xb)
    w = S.svdq_pack_weights_w8a8(L.W, a, spec.rank, bias_bits=L.b)
    p = oracle.pack_weights_w8a8(L.W, a.astype(np.float64), spec.rank, bias_bits=L.b)
    e = w.export()
    assert np.array_equal(e["wq8"].astype(np.int64), p["wcodes8"]), "weight codes"
    assert np.array_equal(e["s_w8"].astype(np.float64), p["s_w8"]), "weight scales"
    r = w.rank
    signs = column_signs(e["L1"], p["L1b"]) if r else np.zeros(0)
    xq, s_x, Z, Yb = _run(w, Xb, epilogue)
    xc, sxo, Zo, xhat = oracle.quantize_act_w8a8(Xb, p["inv_lambda"], p["L1b"])
    assert np.array_equal(xq, xc), "activation codes"
    assert np.array_equal(s_x, sxo), "activation scales"
    Zg = check_z(_bits(Z), Zo, xhat, p["L1b"], signs) if r else np.zeros((Xb.shape[0], 0))
    _, Yo = oracle.linear_w8a8(xc, sxo, Zg, p["wcodes8"], p["s_w8"], p["L2b"], p["bias"],
                               apply_gelu=(epilogue == S.EPI_GELU))
    err = rel_fro(oracle.bf16_bits_to_f64(Yb), Yo)
    assert err <= Y_REL_FRO, err
    w.free()
    return err


@pytest.mark.parametrize("M,K,N,r,epi", [
    (256, 512, 512, 16, S.EPI_NONE),       # the outlier workload at small size
    (130, 320, 600, 16, S.EPI_NONE),       # ragged M and N, 5 K groups
    (1, 64, 136, 8, S.EPI_NONE),           # one token, one K group
    (390, 1152, 1152, 32, S.EPI_GELU),     # PixArt width, GELU, rank 32
    (257, 768, 512, 0, S.EPI_NONE),        # no low-rank branch
    (512, 3072, 3072, 16, S.EPI_NONE),     # FLUX width, the eight-bit setting's rank
])
def test_w8a8_matches_oracle(M, K, N, r, epi):
    spec = synth.layer_spec(f"w8_{M}_{K}_{N}_{r}", M, K, N, r, 700 + M + K + r,
                            tiny=(K <= 512))
    check_w8a8(spec, epi)


def test_w8a8_row_pitch():
    """Y written into a wider buffer (ldy > N): the columns past N stay untouched."""
    spec = synth.layer_spec("w8_ldy", 200, 512, 264, 16, 74, tiny=True)
    L = synth.make_layer(spec)
    a = S.svdq_calib_absmax(L.X)
    w = S.svdq_pack_weights_w8a8(L.W, a, 16, bias_bits=L.b)
    lin = S.W8A8Linear(w)
    xq, s_x, Z, Y = lin.buffers(200)
    full = torch.full((200, 320), -7.0, dtype=torch.bfloat16, device="cuda")
    lin.forward(_to_dev(L.X), out=full[:, :264])
    lin.forward(_to_dev(L.X), out=Y)
    torch.cuda.synchronize()
    S.svdq_get_device_error(w)
    assert np.array_equal(_bits(full[:, :264]), _bits(Y))
    assert torch.all(full[:, 264:] == -7.0)
    w.free()


def test_w8a8_zero_and_single_outlier_tokens():
    spec = synth.layer_spec("w8_edge", 96, 256, 264, 8, 71, tiny=True)
    L = synth.make_layer(spec)
    X = L.X.copy()
    X[5] = 0                                   # all-zero token: s = 0, codes 0
    X[17, :] = 0
    X[17, 3] = 0x4000                           # one channel only (2.0)
    check_w8a8(spec, X_bits=X)


def test_w8a8_full_size_qkv():
    """The FLUX QKV projection with the eight-bit setting's rank 16, all
    4608 tokens; the oracle checks sampled rows over every column and the
    weight codes of sampled columns."""
    spec = synth.layer_spec("w8_flux_qkv", 4608, 3072, 9216, 16, 1)
    L = synth.make_layer(spec)
    M, N = 4608, 9216
    a = S.svdq_calib_absmax(L.X)
    w = S.svdq_pack_weights_w8a8(L.W, a, 16, bias_bits=L.b)
    e = w.export()
    rng = np.random.default_rng(5)
    C = np.unique(np.concatenate([[0, 255, 256, N - 1], rng.choice(N, 96, replace=False)]))
    Wl = oracle.bf16_bits_to_f64(L.W)
    lam_o = oracle.smoothing_lambda(a.astype(np.float64), np.max(np.abs(Wl), axis=0))
    assert np.array_equal(e["inv_lambda"].astype(np.float64), oracle.round_f32(1.0 / lam_o))
    L1 = oracle.bf16_bits_to_f64(e["L1"])
    L2 = oracle.bf16_bits_to_f64(e["L2"])
    R_C, _, _ = oracle.residual_quantize(lam_o[:, None] * Wl[C].T, L1, L2[:, C])
    codes_C, sw_C = oracle.quantize_rows_int8(oracle.round_f32(R_C.T))
    assert np.array_equal(e["wq8"][C].astype(np.int64), codes_C), "weight codes"
    assert np.array_equal(e["s_w8"][C].astype(np.float64), sw_C), "weight scales"
    xq, s_x, Z, Yb = _run(w, L.X, S.EPI_NONE)
    R = np.unique(np.concatenate([[0, 127, 128, M - 1], rng.choice(M, 160, replace=False)]))
    xc, sxo, Zo, xhat = oracle.quantize_act_w8a8(L.X[R], e["inv_lambda"].astype(np.float64), L1)
    assert np.array_equal(xq[R], xc), "activation codes"
    assert np.array_equal(s_x[R], sxo), "activation scales"
    Zg = check_z(_bits(Z)[R], Zo, xhat, L1, np.ones(16))
    _, Yo = oracle.linear_w8a8(xc, sxo, Zg, e["wq8"].astype(np.int64),
                               e["s_w8"].astype(np.float64), L2,
                               oracle.bf16_bits_to_f64(e["bias"]))
    err = rel_fro(oracle.bf16_bits_to_f64(Yb[R]), Yo)
    assert err <= Y_REL_FRO, err
    w.free()
