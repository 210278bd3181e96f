"""GPU parity of the cross-layer fusion: svdq_linear_quantize_next (fc1's
epilogue emits fc2's activation side) against the unfused calls on the GPU
and against the oracle's activation pass applied to fc1's output.

Bar: fc2's INT4 codes and scales bit-exact, both against svdq_quantize_act
on the GPU's own unfused fc1 output H and against the oracle's quantiser on
H; Z within one bf16 ulp plus the fp32 accumulation bound of the oracle's
exact Z; fc2's output within 2e-3 relative Frobenius error of the oracle's
bf16 Y computed from the fused path's own codes, scales and Z.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import w4a4_quantized_gemm_smooth_b200 as S
from helpers import Y_REL_FRO, rel_fro, z_tolerance

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


def _pair(M, K, N, N2, r1, r2, seed, epi):
    """fc1 [N, K] and fc2 [N2, N]; fc2 is calibrated on the GPU's unfused fc1
    output (the activation it sees in the chained pair)."""
    L1 = synth.make_layer(synth.layer_spec(f"p1_{M}_{K}_{N}", M, K, N, r1, seed, tiny=(K <= 512)))
    L2 = synth.make_layer(synth.layer_spec(f"p2_{N}_{N2}", M, N, N2, r2, seed + 1,
                                           tiny=(N <= 512)))
    w1 = S.svdq_pack_weights(L1.W, S.svdq_calib_absmax(L1.X), r1, bias_bits=L1.b)
    lin1 = S.SVDQLinear(w1, epi)
    X = _to_dev(L1.X)
    H = lin1(X).clone()
    torch.cuda.synchronize()
    Hb = _bits(H)
    w2 = S.svdq_pack_weights(L2.W, S.svdq_calib_absmax(Hb), r2, bias_bits=L2.b)
    return w1, w2, lin1, H, Hb


def _fused(w1, w2, lin1, epi):
    M = lin1.xq.shape[0]
    N, r2 = w1.N, w2.rank
    xq2 = torch.full((M, N // 2), 0xAB, dtype=torch.uint8, device="cuda")
    s_x2 = torch.full((N // 64, M), -1.0, dtype=torch.float32, device="cuda")
    Z2 = torch.empty((M, r2), dtype=torch.bfloat16, device="cuda") if r2 else None
    nws = S.svdq_linear_quantize_next_workspace(w1, w2, M)
    tiles_n = -(-N // (128 if N <= 128 or 0 < N % 256 <= 128 else 256))
    assert nws == 4 * tiles_n * M * r2
    ws = torch.full((max(nws // 4, 1),), 3.0, dtype=torch.float32, device="cuda") if r2 else None
    S.svdq_linear_quantize_next(w1, w2, lin1.xq, lin1.s_x, lin1.Z, xq2, s_x2, Z2, ws, epi)
    torch.cuda.synchronize()
    S.svdq_get_device_error(w1)
    return xq2, s_x2, Z2


def check_pair(M, K, N, N2, r1, r2, seed, epi=S.EPI_GELU, rows=None):
    w1, w2, lin1, H, Hb = _pair(M, K, N, N2, r1, r2, seed, epi)
    xq2, s_x2, Z2 = _fused(w1, w2, lin1, epi)
    # the unfused activation pass on the GPU's own H
    lin2 = S.SVDQLinear(w2)
    uq, us, uZ, _ = lin2.buffers(M)
    S.svdq_quantize_act(w2, H, uq, us, uZ)
    torch.cuda.synchronize()
    assert torch.equal(xq2, uq), "codes differ from the unfused activation pass"
    assert torch.equal(s_x2, us), "scales differ from the unfused activation pass"
    # the oracle's activation pass on H (sampled rows at full size)
    R = np.arange(M) if rows is None else rows
    e2 = w2.export()
    L1b = oracle.bf16_bits_to_f64(e2["L1"])
    codes, s_o, Z_o, xhat = oracle.quantize_act(Hb[R], e2["inv_lambda"].astype(np.float64), L1b)
    gq = xq2.cpu().numpy()
    assert np.array_equal(gq[R], oracle.pack_nibbles(codes)), "codes vs oracle"
    assert np.array_equal(s_x2.cpu().numpy()[:, R].astype(np.float64), s_o), "scales vs oracle"
    if r2:
        Zg = oracle.bf16_bits_to_f64(_bits(Z2)[R])
        tol = 2.0 ** -7 * np.abs(Z_o) + z_tolerance(xhat, L1b, N) + 1e-30
        bad = np.abs(Zg - Z_o) > tol
        assert not bad.any(), f"{bad.sum()} Z entries out of tolerance"
        Zu = oracle.bf16_bits_to_f64(_bits(uZ)[R])
        assert np.all(np.abs(Zg - Zu) <= 2.0 ** -7 * np.abs(Zu) + 2 * z_tolerance(xhat, L1b, N) + 1e-30)
    # fc2 on the fused path's own activation side, against the oracle
    Y2 = torch.empty((M, N2), dtype=torch.bfloat16, device="cuda")
    S.svdq_linear(w2, xq2, s_x2, Z2, Y2)
    torch.cuda.synchronize()
    S.svdq_get_device_error(w2)
    _, Yo = oracle.linear(codes, s_o, (Zg if r2 else np.zeros((len(R), 0))),
                          oracle.unpack_nibbles(e2["wq"]), e2["s_w"].astype(np.float64),
                          oracle.bf16_bits_to_f64(e2["L2"]), oracle.bf16_bits_to_f64(e2["bias"]))
    err = rel_fro(oracle.bf16_bits_to_f64(_bits(Y2)[R]), Yo)
    assert err <= Y_REL_FRO, err
    w1.free()
    w2.free()
    return err


@pytest.mark.parametrize("M,K,N,N2,r1,r2,epi", [
    (256, 512, 768, 256, 32, 32, S.EPI_GELU),   # 128 x 256 tiles, two L1 parts per tile
    (200, 256, 320, 192, 16, 16, S.EPI_GELU),   # 128 x 128 tiles, ragged M, partial last tile
    (130, 512, 512, 136, 8, 24, S.EPI_NONE),    # rank 24 (padded to 32), no GELU
    (96, 256, 384, 128, 0, 16, S.EPI_GELU),     # fc1 without a low-rank branch
    (160, 256, 256, 128, 16, 0, S.EPI_GELU),    # fc2 without a low-rank branch: no Z
    (1, 64, 128, 64, 8, 8, S.EPI_GELU),         # one token
])
def test_fused_next_matches_unfused_and_oracle(M, K, N, N2, r1, r2, epi):
    check_pair(M, K, N, N2, r1, r2, 900 + M + N, epi)


def test_fused_next_flux_mlp_pair():
    """The FLUX feed-forward pair (fc1 3072 -> 12288 with GELU, fc2 12288 ->
    3072, rank 32), all 4608 tokens on the GPU, the oracle on sampled rows."""
    rng = np.random.default_rng(7)
    rows = np.unique(np.concatenate([[0, 127, 128, 4607], rng.choice(4608, 24, replace=False)]))
    err = check_pair(4608, 3072, 12288, 3072, 32, 32, 2, rows=rows)
    assert err < 1.5e-3


def test_mlp_module_fused_equals_unfused():
    """SVDQMLP: the fused and the unfused chains give the same fc2 codes, so
    their outputs differ only through Z's summation order."""
    w1, w2, lin1, H, Hb = _pair(256, 512, 768, 384, 32, 32, 31, S.EPI_GELU)
    mlp = S.SVDQMLP(w1, w2)
    X = _to_dev(synth.make_layer(synth.layer_spec("p1_256_512_768", 256, 512, 768, 32, 31,
                                                  tiny=True)).X)
    Yf = mlp(X, fused=True).clone()
    qf = mlp.fc2.xq.clone()
    Yu = mlp(X, fused=False).clone()
    qu = mlp.fc2.xq.clone()
    torch.cuda.synchronize()
    assert torch.equal(qf, qu)
    assert rel_fro(oracle.bf16_bits_to_f64(_bits(Yf)), oracle.bf16_bits_to_f64(_bits(Yu))) < 1e-3
    assert torch.equal(mlp.H, H)         # the unfused chain stored fc1's Y bit for bit
    w1.free()
    w2.free()


def test_fused_next_rejects_mismatched_layers():
    w1, w2, lin1, H, Hb = _pair(64, 256, 320, 128, 16, 16, 41, S.EPI_GELU)
    L = synth.make_layer(synth.layer_spec("bad", 64, 256, 128, 16, 42, tiny=True))
    w_bad = S.svdq_pack_weights(L.W, S.svdq_calib_absmax(L.X), 16, bias_bits=L.b)   # K = 256 != 320
    xq2 = torch.empty((64, 160), dtype=torch.uint8, device="cuda")
    s_x2 = torch.empty((5, 64), dtype=torch.float32, device="cuda")
    Z2 = torch.empty((64, 16), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty((S.svdq_linear_quantize_next_workspace(w1, w2, 64) // 4,),
                     dtype=torch.float32, device="cuda")
    with pytest.raises(S.SVDQError) as e:
        S.svdq_linear_quantize_next(w1, w_bad, lin1.xq, lin1.s_x, lin1.Z, xq2, s_x2, Z2, ws)
    assert e.value.status == 2              # SVDQ_ERR_SHAPE
    with pytest.raises(S.SVDQError) as e:
        S.svdq_linear_quantize_next(w1, w2, lin1.xq, lin1.s_x, lin1.Z, xq2, s_x2, Z2, None)
    assert e.value.status == 1              # SVDQ_ERR_INVALID_ARG: no workspace
    with pytest.raises(S.SVDQError) as e:
        S.svdq_linear_quantize_next(w1, w2, lin1.xq, lin1.s_x, lin1.Z, xq2, s_x2, Z2, ws[:-4])
    assert e.value.status == 2              # SVDQ_ERR_SHAPE: workspace too small
    for w in (w1, w2, w_bad):
        w.free()
