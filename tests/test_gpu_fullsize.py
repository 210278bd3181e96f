"""GPU parity at the full workload sizes, in the launch configuration the
bench times (svdq_quantize_act then svdq_linear over all M tokens).

The oracle cannot redo a full-size layer in seconds, so it checks samples
that it computes one by one:
  * lambda for every channel; weight codes and scales of sampled output
    columns, re-derived from the library's exported bf16 factors (the
    residual and its quantisation are column-separable);
  * activation codes, scales and Z of sampled token rows (bit-exact / Z
    tolerance), from the same X bytes;
  * Y of the sampled rows over every output column (relative Frobenius
    <= 2e-3 against the oracle's bf16 Y from the GPU's codes, scales and Z);
  * int32 group partials of four whole output tiles (the first and last
    corners and two seeded interior tiles), bit-exact.
The FLUX MLP pair runs as a chain: fc1 with the GELU epilogue writes H, and
fc2 quantises H with its own fused activation kernel.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import w4a4_quantized_gemm_smooth_b200 as S
from helpers import Y_REL_FRO, check_z, rel_fro

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


def _sample(n, k, seed, tile):
    """Sorted unique indices: both ends, the last tile's edge, and k random."""
    rng = np.random.default_rng(seed)
    fixed = [0, 1, min(tile - 1, n - 1), min(tile, n - 1), n - 1, max(n - tile, 0)]
    pick = rng.choice(n, size=min(k, n), replace=False)
    return np.unique(np.concatenate([fixed, pick]).astype(np.int64))


def check_full(spec, X_bits=None, epilogue=S.EPI_NONE, sigma=False, n_rows=192, n_cols=160):
    L = synth.make_layer(spec)
    Xb = L.X if X_bits is None else X_bits
    M, K, N, r = Xb.shape[0], spec.K, spec.N, spec.rank
    a = S.svdq_calib_absmax(Xb)
    w = S.svdq_pack_weights(L.W, a, r, bias_bits=L.b, lora_A_bits=L.A, lora_B_bits=L.B)
    e = w.export()
    rt = e["L1"].shape[1]
    assert rt == r + spec.lora_rank

    # smoothing factors, every channel (review section 3.1, eq. 4)
    Wl = oracle.bf16_bits_to_f64(L.W)                       # [N, K]
    lam = oracle.smoothing_lambda(a.astype(np.float64), np.max(np.abs(Wl), axis=0))
    assert np.array_equal(e["inv_lambda"].astype(np.float64), oracle.round_f32(1.0 / lam))

    # residual codes and scales of sampled columns, given the library's factors
    L1 = oracle.bf16_bits_to_f64(e["L1"])                   # [K, rt]
    L2 = oracle.bf16_bits_to_f64(e["L2"])                   # [rt, N]
    C = _sample(N, n_cols, spec.seed + 11, 256)
    WtC = lam[:, None] * Wl[C].T
    _, codes_C, sw_C = oracle.residual_quantize(WtC, L1[:, :r], L2[:r, C])
    assert np.array_equal(e["wq"][C], oracle.pack_nibbles(codes_C)), "weight codes"
    assert np.array_equal(e["s_w"][:, C].astype(np.float64), sw_C), "weight scales"
    if sigma:
        Wt = lam[:, None] * Wl.T
        U, Sg, Vt = oracle.leading_svd(Wt, r + 1)
        assert np.max(np.abs(e["sigma"] - Sg) / Sg) < 1e-10
        prod = U[:, :r] @ (Sg[:r, None] * Vt[:r, C])
        assert np.linalg.norm(L1[:, :r] @ L2[:r, C] - prod) / np.linalg.norm(WtC) < 1e-2

    # the hot path over the whole batch
    X = _to_dev(Xb)
    lin = S.SVDQLinear(w, epilogue)
    xq, s_x, Z, Y = lin.buffers(M)
    lin.forward(X, out=Y)
    torch.cuda.synchronize()
    S.svdq_get_device_error(w)
    xq_h, sx_h = xq.cpu().numpy(), s_x.cpu().numpy()

    # activation side on sampled rows (review section 6.1)
    R = _sample(M, n_rows, spec.seed + 7, 128)
    xc, sxo, Zo, xhat = oracle.quantize_act(Xb[R], e["inv_lambda"].astype(np.float64), L1)
    assert np.array_equal(xq_h[R], oracle.pack_nibbles(xc)), "activation codes"
    assert np.array_equal(sx_h[:, R].astype(np.float64), sxo), "activation scales"
    Zg_bits = _bits(Z)
    if rt:
        check_z(Zg_bits[R], Zo, xhat, L1, np.ones(rt))

    # Y of the sampled rows, every column, from the GPU's own codes/scales/Z
    wcodes = oracle.unpack_nibbles(e["wq"])
    Zg = oracle.bf16_bits_to_f64(Zg_bits)[R] if rt else np.zeros((len(R), 0))
    _, Yo = oracle.linear(xc, sxo, Zg, wcodes, e["s_w"].astype(np.float64), L2,
                          oracle.bf16_bits_to_f64(e["bias"]),
                          apply_gelu=(epilogue == S.EPI_GELU))
    Yb = _bits(Y)
    err = rel_fro(oracle.bf16_bits_to_f64(Yb[R]), Yo)
    assert err <= Y_REL_FRO, err

    # int32 partials of four whole tiles: both corners and two seeded others
    BN = 256 if N > 128 and (N % 256 == 0 or N % 256 > 128) else 128
    tm, tn = -(-M // 128), -(-N // BN)
    rng = np.random.default_rng(spec.seed + 13)
    picks = [(0, 0), (tm - 1, tn - 1)]
    while len(picks) < min(4, tm * tn):
        t = (int(rng.integers(tm)), int(rng.integers(tn)))
        if t not in picks:
            picks.append(t)
    tiles = [(128 * i, BN * j) for i, j in picks]
    for r0, c0 in tiles:
        nr, nc = min(128, M - r0), min(BN, N - c0)
        P = torch.empty((K // 64, nr, nc), dtype=torch.int32, device="cuda")
        S.svdq_debug_partials(w, M, xq, r0, nr, c0, nc, P)
        torch.cuda.synchronize()
        rows = np.arange(r0, r0 + nr)
        Po = oracle.group_partials(oracle.unpack_nibbles(xq_h[rows]), wcodes, None,
                                   np.arange(c0, c0 + nc))
        assert np.array_equal(P.cpu().numpy().astype(np.int64), Po), f"partials {r0},{c0}"
    S.svdq_get_device_error(w)
    w.free()
    return Yb, err


def test_flux_qkv_full():
    _, err = check_full(synth.WORKLOADS["flux_qkv"], sigma=True)
    assert err < 1.5e-3


def test_flux_mlp_chain_full():
    """fc1 (GELU epilogue) -> H -> fc2, each at full size."""
    H, _ = check_full(synth.WORKLOADS["flux_mlp_fc1"], epilogue=S.EPI_GELU)
    check_full(synth.WORKLOADS["flux_mlp_fc2"], X_bits=H)


@pytest.mark.parametrize("name", ["flux_ss_in", "flux_ss_out"])
def test_flux_single_stream_with_lora_full(name):
    check_full(synth.WORKLOADS[name])


@pytest.mark.parametrize("spec", synth.pixart_points(), ids=lambda p: p.name)
def test_pixart_points_full(spec):
    """Every point of the PixArt-Sigma-like sweep (review section 9.2): 4
    shapes x M in {256, 1024, 4096, 16384} x rank in {16, 32, 64}."""
    check_full(spec, n_rows=96, n_cols=96)
