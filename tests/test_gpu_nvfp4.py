"""GPU parity of the NVFP4 variant (svdq_quantize_act_nvfp4 then
svdq_linear_nvfp4) against the oracle's NVFP4 functions on the same seeded
inputs.

Bar: E2M1 activation codes, E4M3 group-scale bytes (in the tensor-core atom
layout) and row scales bit-exact; Z within one bf16 ulp plus the fp32
accumulation bound; Y within 2e-3 relative Frobenius error of the oracle's
bf16 Y computed from the GPU's own codes, scales and Z."""
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


def atom_to_rows(sf_atoms, rows, K):
    """Group-scale bytes in the atom layout -> [rows, K/16] (layout rule of
    include/svdq.h: atom (a, kb) at (a K/64 + kb) 512, row r at 16 (r % 32) +
    4 (r / 32), group j of the K block at + j)."""
    nkb = K // 64
    out = np.zeros((rows, K // 16), np.uint8)
    for r in range(rows):
        a, rr = divmod(r, 128)
        for kb in range(nkb):
            base = (a * nkb + kb) * 512 + 16 * (rr % 32) + 4 * (rr // 32)
            out[r, 4 * kb:4 * kb + 4] = sf_atoms[base:base + 4]
    return out


def e4m3_value(bits):
    return torch.from_numpy(np.ascontiguousarray(bits)).view(torch.float8_e4m3fn) \
        .to(torch.float32).numpy().astype(np.float64)


def _run(w, Xb, epilogue):
    lin = S.NVFP4Linear(w, epilogue)
    xq, sfa, s_x, Z, Y = lin.buffers(Xb.shape[0])
    lin.forward(_to_dev(Xb), out=Y)
    torch.cuda.synchronize()
    S.svdq_get_device_error(w)
    return (xq.cpu().numpy(), sfa.cpu().numpy(), s_x.cpu().numpy().astype(np.float64),
            (_bits(Z) if Z is not None else None), _bits(Y))


def check_nvfp4(spec, epilogue=S.EPI_NONE, X_bits=None, rows=None):
    L = synth.make_layer(spec)
    Xb = L.X if X_bits is None else X_bits
    M, K = Xb.shape
    a = S.svdq_calib_absmax(Xb)
    w = S.svdq_pack_weights_nvfp4(L.W, a, spec.rank, bias_bits=L.b)
    e = w.export()
    r = w.rank
    xq, sfa, s_x, Zb, Yb = _run(w, Xb, epilogue)
    R = np.arange(M) if rows is None else rows
    L1 = oracle.bf16_bits_to_f64(e["L1"])
    L2 = oracle.bf16_bits_to_f64(e["L2"])
    xc, xb, xs, Zo, xhat = oracle.quantize_act_nvfp4(Xb[R], e["inv_lambda"].astype(np.float64), L1)
    # activation side, bit-exact
    assert np.array_equal(xq[R], oracle.pack_nibbles(xc)), "activation codes"
    sf_rows = atom_to_rows(sfa, ((M + 127) // 128) * 128, K)
    assert np.array_equal(sf_rows[R], oracle.e4m3_bits(xb)), "activation group scales"
    assert not sf_rows[M:].any(), "padding rows of the scale atoms"
    assert np.array_equal(s_x[R], xs), "activation row scales"
    if r:
        Zg = oracle.bf16_bits_to_f64(Zb[R])
        tol = 2.0 ** -7 * np.abs(Zo) + z_tolerance(xhat, L1, K) + 1e-30
        assert not (np.abs(Zg - Zo) > tol).any(), "Z"
    else:
        Zg = np.zeros((len(R), 0))
    # product, from the GPU's own codes and scales
    gcodes = oracle.unpack_nibbles(xq[R])
    gb = e4m3_value(sf_rows[R])
    wcodes = oracle.unpack_nibbles(e["wq4"])
    wb = e4m3_value(e["sf4"])
    _, Yo = oracle.linear_nvfp4(gcodes, gb, s_x[R], Zg, wcodes, wb, e["s_w4"].astype(np.float64),
                                L2, oracle.bf16_bits_to_f64(e["bias"]),
                                apply_gelu=(epilogue == S.EPI_GELU))
    err = rel_fro(oracle.bf16_bits_to_f64(Yb[R]), Yo)
    assert err <= Y_REL_FRO, err
    w.free()
    return err


@pytest.mark.parametrize("M,K,N,r,epi", [
    (256, 512, 512, 16, S.EPI_NONE),       # the outlier workload at small size
    (130, 320, 136, 8, S.EPI_NONE),        # ragged M and N, odd number of 64-K blocks
    (1, 64, 128, 8, S.EPI_NONE),           # one token, one K block
    (390, 1152, 1152, 32, S.EPI_GELU),     # PixArt width, GELU
    (257, 768, 512, 0, S.EPI_NONE),        # no low-rank branch
    (512, 3072, 3072, 32, S.EPI_NONE),     # FLUX width
])
def test_nvfp4_matches_oracle(M, K, N, r, epi):
    spec = synth.layer_spec(f"f4_{M}_{K}_{N}_{r}", M, K, N, r, 800 + M + K + r,
                            tiny=(K <= 512))
    check_nvfp4(spec, epi)


def test_nvfp4_row_pitch():
    """Y written into a wider buffer (ldy > N): the columns past N stay untouched."""
    spec = synth.layer_spec("f4_ldy", 200, 512, 264, 16, 84, tiny=True)
    L = synth.make_layer(spec)
    a = S.svdq_calib_absmax(L.X)
    w = S.svdq_pack_weights_nvfp4(L.W, a, 16, bias_bits=L.b)
    lin = S.NVFP4Linear(w)
    xq, sfa, s_x, Z, Y = lin.buffers(200)
    full = torch.full((200, 320), -7.0, dtype=torch.bfloat16, device="cuda")
    lin.forward(_to_dev(L.X), out=full[:, :264])
    lin.forward(_to_dev(L.X), out=Y)
    torch.cuda.synchronize()
    S.svdq_get_device_error(w)
    assert np.array_equal(_bits(full[:, :264]), _bits(Y))
    assert torch.all(full[:, 264:] == -7.0)
    w.free()


def test_nvfp4_zero_and_single_outlier_tokens():
    spec = synth.layer_spec("f4_edge", 96, 256, 264, 8, 81, tiny=True)
    L = synth.make_layer(spec)
    X = L.X.copy()
    X[5] = 0
    X[17, :] = 0
    X[17, 3] = 0x4000
    check_nvfp4(spec, X_bits=X)


def test_nvfp4_full_size_qkv():
    """The FLUX QKV projection, all 4608 tokens, rank 32; sampled rows."""
    spec = synth.WORKLOADS["flux_qkv"]
    rng = np.random.default_rng(6)
    rows = np.unique(np.concatenate([[0, 127, 128, 4607], rng.choice(4608, 96, replace=False)]))
    err = check_nvfp4(spec, rows=rows)
    assert err < 1.5e-3
