"""GPU parity: the C-ABI library (pack, svdq_quantize_act, svdq_linear,
svdq_debug_partials) against the fp64 oracle on the same seeded inputs.

Bar (SVDQuant layer contract): INT4 codes, fp32 scales and int32 group
partials bit-exact; weight codes and scales bit-exact; Z within one bf16 ulp
plus the fp32 accumulation bound; Y within 2e-3 relative Frobenius error of
the oracle's bf16 Y.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import w4a4_quantized_gemm_smooth_b200 as S
from helpers import Y_REL_FRO, check_z, column_signs, rel_fro

pytestmark = pytest.mark.gpu


def to_dev(bits, ld=None):
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    if ld is not None and ld != bits.shape[1]:
        full = torch.zeros((bits.shape[0], ld), dtype=torch.bfloat16)
        full[:, :bits.shape[1]] = t
        return full.cuda()[:, :bits.shape[1]]
    return t.cuda()


def to_bits(t):
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "gpu tests need a CUDA device"
    S.lib()


def check_layer(spec, epilogue=S.EPI_NONE, rows_sample=None, partial_blocks=None,
                svd=None, X_bits=None, ldy=None, lora_scale=1.0, W_bits=None, absmax=None,
                pack_check=None):
    L = synth.make_layer(spec)
    Xb = L.X if X_bits is None else X_bits
    Wb = L.W if W_bits is None else W_bits
    a = S.svdq_calib_absmax(Xb) if absmax is None else absmax
    w = S.svdq_pack_weights(Wb, a, spec.rank, bias_bits=L.b, lora_A_bits=L.A,
                            lora_B_bits=L.B, lora_scale=lora_scale)
    p = oracle.pack_weights(Wb, a.astype(np.float64), spec.rank, bias_bits=L.b,
                            lora_A_bits=L.A, lora_B_bits=L.B, lora_scale=lora_scale, svd=svd)
    if pack_check is not None:
        pack_check(p)
    e = w.export()
    if spec.lora_rank:
        # the adapter columns carry no sign ambiguity: bit-exact (eq. 13,
        # the scale on the smoothed A side)
        r0 = spec.rank
        assert np.array_equal(oracle.bf16_bits_to_f64(e["L1"])[:, r0:], p["L1b"][:, r0:])
        assert np.array_equal(oracle.bf16_bits_to_f64(e["L2"])[r0:], p["L2b"][r0:])
    # weights
    assert np.array_equal(e["inv_lambda"].astype(np.float64), p["inv_lambda"])
    assert np.array_equal(e["wq"], p["wq"])
    assert np.array_equal(e["s_w"].astype(np.float64), p["s_w"])
    signs = column_signs(e["L1"], p["L1b"]) if w.rank else np.zeros(0)
    # activation pass
    M, K, N = Xb.shape[0], spec.K, spec.N
    X = to_dev(Xb)
    lin = S.SVDQLinear(w, epilogue)
    xq, s_x, Z, Y = lin.buffers(M)
    if ldy is not None:
        Yfull = torch.empty((M, ldy), dtype=torch.bfloat16, device="cuda")
        Y = Yfull[:, :N]
    lin.forward(X, out=Y)
    torch.cuda.synchronize()
    S.svdq_get_device_error(w)
    xc, sxo, Zo, xhat = oracle.quantize_act(Xb, p["inv_lambda"], p["L1b"])
    assert np.array_equal(xq.cpu().numpy(), oracle.pack_nibbles(xc)), "activation codes"
    assert np.array_equal(s_x.cpu().numpy().astype(np.float64), sxo), "activation scales"
    if w.rank:
        check_z(to_bits(Z), Zo, xhat, p["L1b"], signs)
    # output
    rows = np.arange(M) if rows_sample is None else rows_sample
    _, Yo = oracle.linear(xc, sxo, Zo, p["wcodes"], p["s_w"], p["L2b"], p["bias"],
                          apply_gelu=(epilogue == S.EPI_GELU), rows=rows)
    Yg = oracle.bf16_bits_to_f64(to_bits(Y))[rows]
    err = rel_fro(Yg, Yo)
    assert err <= Y_REL_FRO, err
    # int32 partials from the tensor-core path
    blocks = partial_blocks or [(0, min(M, 256), 0, min(N, 256))]
    for (r0, nr, c0, nc) in blocks:
        P = torch.empty((K // 64, nr, nc), dtype=torch.int32, device="cuda")
        S.svdq_debug_partials(w, M, xq, r0, nr, c0, nc, P)
        torch.cuda.synchronize()
        Po = oracle.group_partials(xc, p["wcodes"], np.arange(r0, r0 + nr), np.arange(c0, c0 + nc))
        assert np.array_equal(P.cpu().numpy().astype(np.int64), Po), f"partials {r0},{c0}"
    S.svdq_get_device_error(w)
    w.free()
    return err


def test_tiny_layer():
    spec = synth.WORKLOADS["tiny"]
    err = check_layer(spec, partial_blocks=[(0, 256, 0, 512)])
    assert err < 1e-3


def test_tiny_layer_gelu_epilogue():
    check_layer(synth.WORKLOADS["tiny"], epilogue=S.EPI_GELU)


@pytest.mark.parametrize("M,K,N,r", [
    (200, 512, 384, 16),     # ragged M
    (130, 320, 136, 24),     # ragged M, K not a multiple of 256, N not of 128, r not of 16
    (1, 64, 128, 8),         # one token, one group
    (333, 1152, 256, 64),    # PixArt width, rank 64
    (128, 256, 128, 0),      # no low-rank branch
    (130, 8256, 136, 8),     # K too long for the correction operand of 128-column tiles
])
def test_ragged_and_small_shapes(M, K, N, r):
    spec = synth.layer_spec(f"e{M}_{K}_{N}_{r}", M, K, N, r, 100 + M + K + N + r, tiny=True)
    check_layer(spec, partial_blocks=[(0, M, 0, N), (M - 1, 1, N - 1, 1)])


@pytest.mark.parametrize("M,K,r", [
    (4773, 1152, 64),   # 150 token blocks, ragged last block, rank 64
    (4773, 1152, 0),    # the same without a branch
    (4800, 4608, 32),   # long K
    (9472, 512, 16),    # 296 token blocks of a single stage each
])
def test_more_token_blocks_than_sms(M, K, r):
    """More 32-token blocks than SMs (more than one wave of the activation
    pass), the ragged last block included.  Every row's codes, scales and Z
    are compared."""
    spec = synth.layer_spec(f"p{M}_{K}_{r}", M, K, 128, r, 300 + M + K + r, tiny=True)
    rows = np.sort(np.random.default_rng(M + K + r).choice(M, 192, replace=False))
    check_layer(spec, rows_sample=rows, partial_blocks=[(M - 128, 128, 0, 128)])


def test_layer_from_host_buffers():
    """svdq_linear_host: X read from host memory (pinned and pageable, row
    stride above K), Y written to host memory (row stride above N, the
    padding untouched); the same bits as the device calls on the same X."""
    spec = synth.layer_spec("hostbuf", 333, 1152, 136, 32, 77, tiny=True)
    L = synth.make_layer(spec)
    a = S.svdq_calib_absmax(L.X)
    w = S.svdq_pack_weights(L.W, a, spec.rank, bias_bits=L.b)
    M, K, N = spec.M, spec.K, spec.N
    X = to_dev(L.X)
    for epi in (S.EPI_NONE, S.EPI_GELU):
        Yref = S.SVDQLinear(w, epi).forward(X).cpu()
        for pinned in (True, False):
            Xh = torch.zeros((M, K + 64), dtype=torch.bfloat16, pin_memory=pinned)
            Xh[:, :K] = X.cpu()
            Yh = torch.full((M, N + 8), float("nan"), dtype=torch.bfloat16, pin_memory=pinned)
            ws = torch.empty(S.svdq_linear_host_workspace(w, M), dtype=torch.uint8, device="cuda")
            S.svdq_linear_host(w, Xh[:, :K], Yh[:, :N], ws, epi)
            torch.cuda.synchronize()
            S.svdq_get_device_error(w)
            assert torch.equal(Yh[:, :N], Yref), (epi, pinned)
            assert torch.isnan(Yh[:, N:].float()).all()
    # a workspace one byte short is refused before anything is enqueued
    short = torch.empty(S.svdq_linear_host_workspace(w, M) - 1, dtype=torch.uint8, device="cuda")
    Yh = torch.empty((M, N), dtype=torch.bfloat16)
    with pytest.raises(S.SVDQError):
        S.svdq_linear_host(w, X.cpu(), Yh, short)
    w.free()


def test_ragged_output_stride():
    spec = synth.layer_spec("ldy", 96, 256, 196, 16, 7, tiny=True)
    check_layer(spec, ldy=200)


@pytest.mark.parametrize("lora_scale", [1.0, 0.3, -2.5])
def test_lora_branch(lora_scale):
    spec = synth.layer_spec("lora", 256, 512, 384, 16, 21, lora_rank=16)
    check_layer(spec, lora_scale=lora_scale)


def test_weight_group_of_minus_eight_codes():
    """A weight group whose residual codes are all -8.  Channels 64..127 get
    smoothing factors of 2^-127 (activation statistic 2^-149 against a weight
    of 2^105 in column 0), so column 1's weights of -2^-19 there become
    residuals of -2^-146 = -8 s with the group scale s = fl32(2^-146 / 7) =
    2^-149, the smallest fp32 subnormal (the clamp to [-8, 7] keeps -8).  The
    layer then keeps two's-complement weight codes on the device, and the
    GEMM's per-group correction for that group takes its largest digit
    (-sum_k q_w = 512 = 64 * 8).  The activations of those channels are
    +-2^-133 (bf16's smallest subnormal) times the factor 2^127, so the
    partials there are non-zero."""
    M, K, N = 256, 256, 256
    spec = synth.layer_spec("minus8", M, K, N, 0, 91, tiny=True)
    L = synth.make_layer(spec)
    W = L.W.copy()
    X = L.X.copy()
    ch = slice(64, 128)
    W[0, ch] = 0x7400                          # 2^105
    W[1, ch] = 0xB600                          # -2^-19
    X[:, ch] = 0
    rng = np.random.default_rng(92)
    pick = rng.random((M, 64)) < 0.3
    X[:, ch] = np.where(pick, np.where(rng.random((M, 64)) < 0.5, 0x0001, 0x8001), 0).astype(X.dtype)
    a = S.svdq_calib_absmax(X)
    a[ch] = np.float32(2.0 ** -149)

    def pack_check(p):
        codes = p["wcodes"]
        assert np.all(codes[1, ch] == -8), "the planted group is all -8"
        assert p["s_w"][1, 1] == 2.0 ** -149
    check_layer(spec, X_bits=X, W_bits=W, absmax=a, pack_check=pack_check,
                partial_blocks=[(0, 256, 0, 256)])


def test_zero_rows_and_groups():
    spec = synth.layer_spec("zeros", 160, 256, 128, 8, 9, tiny=True)
    L = synth.make_layer(spec)
    X = L.X.copy()
    X[5] = 0                    # an all-zero token
    X[7, 64:128] = 0            # one all-zero group
    X[9, :64] = 0x8000          # negative zeros
    check_layer(spec, X_bits=X)


def test_argument_errors_launch_nothing():
    spec = synth.layer_spec("args", 64, 128, 64, 8, 3, tiny=True)
    L = synth.make_layer(spec)
    w = S.svdq_pack_weights(L.W, S.svdq_calib_absmax(L.X), 8, bias_bits=L.b)
    lib = S.lib()
    X = to_dev(L.X)
    xq = torch.empty((64, 64), dtype=torch.uint8, device="cuda")
    s_x = torch.empty((2, 64), dtype=torch.float32, device="cuda")
    Z = torch.empty((64, 8), dtype=torch.bfloat16, device="cuda")
    Y = torch.empty((64, 64), dtype=torch.bfloat16, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    import ctypes
    vp = ctypes.c_void_p
    # misaligned X (offset by one element)
    assert lib.svdq_quantize_act(w.handle, 63, vp(X.data_ptr() + 2), 128, vp(xq.data_ptr()),
                                 vp(s_x.data_ptr()), vp(Z.data_ptr()), vp(st)) == 3
    # ldx too small
    assert lib.svdq_quantize_act(w.handle, 64, vp(X.data_ptr()), 64, vp(xq.data_ptr()),
                                 vp(s_x.data_ptr()), vp(Z.data_ptr()), vp(st)) == 2
    # missing Z with rank > 0
    assert lib.svdq_linear(w.handle, 64, vp(xq.data_ptr()), vp(s_x.data_ptr()), None,
                           vp(Y.data_ptr()), 64, 0, vp(st)) == 1
    # bad epilogue
    assert lib.svdq_linear(w.handle, 64, vp(xq.data_ptr()), vp(s_x.data_ptr()),
                           vp(Z.data_ptr()), vp(Y.data_ptr()), 64, 7, vp(st)) == 1
    # M == 0 is a no-op
    assert lib.svdq_linear(w.handle, 0, None, None, None, None, 64, 0, vp(st)) == 0
    # partial block outside the output
    assert lib.svdq_debug_partials(w.handle, 64, vp(xq.data_ptr()), 60, 8, 0, 4,
                                   vp(Y.data_ptr()), vp(st)) == 2
    torch.cuda.synchronize()
    S.svdq_get_device_error(w)
    w.free()


def test_save_load_roundtrip(tmp_path):
    spec = synth.layer_spec("sl", 128, 256, 192, 16, 31, lora_rank=8)
    L = synth.make_layer(spec)
    w = S.svdq_pack_weights(L.W, S.svdq_calib_absmax(L.X), 16, bias_bits=L.b,
                            lora_A_bits=L.A, lora_B_bits=L.B)
    path = str(tmp_path / "l.svdq")
    w.save(path)
    w2 = S.svdq_weights_load(path)
    e1, e2 = w.export(), w2.export()
    for k in e1:
        assert np.array_equal(e1[k], e2[k]), k
    X = to_dev(L.X)
    Y1 = S.SVDQLinear(w)(X).clone()
    Y2 = S.SVDQLinear(w2)(X).clone()
    torch.cuda.synchronize()
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))
    w.free()
    w2.free()


@pytest.mark.parametrize("gptq", [False, True])
def test_calibrated_pack_layer(gptq):
    """A layer packed with the calibrated alpha search and one refinement
    (and GPTQ rounding of the residual) runs through the hot path like any
    other."""
    spec = synth.layer_spec("calgpu", 192, 640, 320, 24, 55)
    L = synth.make_layer(spec)
    w, errs = S.svdq_pack_weights_calibrated(L.W, L.X, 24, refine_iters=1, bias_bits=L.b,
                                             gptq=gptq)
    p, errs_o = oracle.pack_weights_calibrated(L.W, L.X, 24, iters=1, bias_bits=L.b, gptq=gptq)
    assert np.allclose(errs, errs_o, rtol=1e-6, atol=0)
    X = to_dev(L.X)
    lin = S.SVDQLinear(w)
    xq, s_x, Z, Y = lin.buffers(L.X.shape[0])
    lin.forward(X, out=Y)
    torch.cuda.synchronize()
    S.svdq_get_device_error(w)
    xc, sxo, Zo, xhat = oracle.quantize_act(L.X, p["inv_lambda"], p["L1b"])
    assert np.array_equal(xq.cpu().numpy(), oracle.pack_nibbles(xc))
    assert np.array_equal(s_x.cpu().numpy().astype(np.float64), sxo)
    signs = column_signs(w.export()["L1"], p["L1b"])
    check_z(to_bits(Z), Zo, xhat, p["L1b"], signs)
    _, Yo = oracle.linear(xc, sxo, Zo, p["wcodes"], p["s_w"], p["L2b"], p["bias"])
    assert rel_fro(oracle.bf16_bits_to_f64(to_bits(Y)), Yo) <= Y_REL_FRO
    w.free()
