"""GPU parity of the activation quantisers on planted edge cases (SVDQuant
review section 2.2, eq. 1: round to the grid, clamp, the all-zero group set
aside), for every kernel that quantises activations: svdq_quantize_act
(W4A4), the W8A8 and NVFP4 activation passes, and the epilogue of
svdq_linear_quantize_next (the next layer's W4A4 codes from a layer's
output tile).

The smoothing factors are made exact powers of two (act_absmax = 4^e
max|W_k|, so lambda = 2^e and x~ = x 2^-e exactly): planted bf16 values
survive smoothing unchanged (e = 0) or move into fp32's subnormal range
(e = 16).  The planted cases:
  exact ties          x / s = k + 1/2 exactly (round half to even decides);
  near a half         0 < |x / s - (k + 1/2)| <= 2^-20 (W4A4) or 2^-15 (W8A8):
                      the fast reciprocal path must hand over to the exact one;
  tiny scale          s < 2^-64 (the exact path on rescaled values);
  subnormal scale     s subnormal with |x / s| >= 7.5 (the clamp to [-8, 7]
                      acts: +8 -> 7, -8 stays) and the int8 analogue;
  underflowing scale  group maximum 2^-149: s = fl32(m / 7) = 0, codes 0;
  zero groups         +0 and -0.
Each range is asserted on the host from the oracle's own scales (exact
rational quotients) before the GPU results are compared bit for bit.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth
import w4a4_quantized_gemm_smooth_b200 as S

pytestmark = pytest.mark.gpu

K = 512                 # 8 groups of 64; groups 6 and 7 have lambda = 2^16
SUB_GROUPS = (6, 7)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "gpu tests need a CUDA device"
    S.lib()


def _to_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)) \
        .view(torch.bfloat16).cuda()


def _bits(t):
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def bf(x):
    """bf16 bits of values that are exact bf16 numbers (asserted)."""
    x = np.asarray(x, dtype=np.float64)
    b = oracle.round_bf16_bits(x)
    assert np.array_equal(oracle.bf16_bits_to_f64(b), x), "planted value not a bf16 number"
    return b


def _absmax_for(W_bits, sub_groups=SUB_GROUPS, Kk=K):
    """act_absmax giving lambda = 1, or 2^16 on the channels of sub_groups."""
    w = np.max(np.abs(oracle.bf16_bits_to_f64(W_bits)), axis=0)         # [K]
    a = w.copy()
    for g in sub_groups:
        a[64 * g:64 * g + 64] *= 2.0 ** 32
    a32 = a.astype(np.float32)
    assert np.array_equal(a32.astype(np.float64), a)
    return a32


def _fr(x):
    return Fraction(float(x))


# ------------------------------------------------------------------ W4A4
def _w4_group_patterns():
    """Planted 64-value groups (values of x~, as bf16 numbers before the
    2^-16 of groups 6-7 is applied), by kind."""
    out = {}
    j = 2.0 ** -3
    ties = [7.0 * j] + [s * (k + 0.5) * j for k in range(7) for s in (1, -1)]
    out["ties"] = ties
    # near a half: m / 7 inexact and x = m / 2 gives x / s = 3.5 (1 + d), |d| <= 2^-24
    out["near_a"] = [1.0, 0.5, -0.5, 0.25]
    out["near_b"] = [1.25, 0.625, -0.625]
    out["near_c"] = [1.5, 0.75, -0.75, 0.1875]
    out["tiny"] = [2.0 ** -70] + [s * k * 2.0 ** -73 for k in (1, 3, 7, 28, 55) for s in (1, -1)]
    out["zero"] = [0.0, -0.0]
    # lambda = 2^16 groups: x~ = x 2^-16
    out["subnormal_clamp"] = [2.0 ** -130, -(2.0 ** -130), 3 * 2.0 ** -133, -(2.0 ** -133)]
    out["underflow"] = [2.0 ** -133, -(2.0 ** -133)]
    return out


def _fill_group(row, g, vals, rng):
    """Values of a planted group, the rest of the group zero, in shuffled columns."""
    cols = 64 * g + rng.permutation(64)[:len(vals)]
    row[64 * g:64 * g + 64] = 0.0
    row[cols] = vals


def _w4_X(M, rng):
    """Token rows: random data (0.1 ~ N(0,1)), then the planted groups."""
    X = rng.standard_normal((M, K)) * 0.1
    X[:, 64 * 6:] *= 0.0            # lambda = 2^16 channels: planted values only
    P = _w4_group_patterns()
    plan = [  # (token, group, kind)
        (0, 0, "ties"), (0, 1, "near_a"), (0, 2, "near_b"), (0, 3, "near_c"), (0, 4, "tiny"),
        (0, 5, "zero"), (0, 6, "subnormal_clamp"), (0, 7, "underflow"),
        (1, 0, "near_c"), (1, 1, "ties"), (1, 2, "tiny"), (1, 3, "near_a"), (1, 6, "underflow"),
        (1, 7, "subnormal_clamp"), (2, 4, "ties"), (2, 5, "near_b"), (3, 2, "zero"),
    ]
    for t, g, kind in plan:
        _fill_group(X[t], g, P[kind], rng)
    X[4] = 0.0
    X[5] = -0.0
    Xb = oracle.round_bf16_bits(X)
    for t, g, kind in plan:        # planted values are exact bf16 numbers
        bf(oracle.bf16_bits_to_f64(Xb[t, 64 * g:64 * g + 64]))
    return Xb, plan


def _assert_w4_ranges(xhat, s_x, codes, plan):
    """The planted groups reach the ranges they are meant to reach."""
    for t, g, kind in plan:
        v = xhat[t, 64 * g:64 * g + 64]
        s = float(s_x[g, t])
        m = float(np.max(np.abs(v)))
        c = codes[t, 64 * g:64 * g + 64]
        if kind == "zero":
            assert m == 0.0 and s == 0.0
            continue
        if kind == "underflow":
            assert m > 0.0 and s == 0.0 and not c.any()
            continue
        assert s > 0.0
        q = [_fr(x) / _fr(s) for x in v if x != 0.0]
        d = [abs(abs(x) - (int(abs(x)) + Fraction(1, 2))) for x in q]
        if kind == "ties":
            assert s == 2.0 ** -3 and sum(x == 0 for x in d) >= 14
        elif kind.startswith("near"):
            assert any(0 < x <= Fraction(1, 2 ** 20) for x in d)
        elif kind == "tiny":
            assert s < 2.0 ** -64
        elif kind == "subnormal_clamp":
            assert s < 2.0 ** -126 and max(abs(x) for x in q) >= Fraction(15, 2)
            assert 7 in c and -8 in c


def test_w4a4_activation_pass_edges():
    rng = np.random.default_rng(11)
    spec = synth.layer_spec("edge_w4", 64, K, 128, 16, 501, tiny=True)
    L = synth.make_layer(spec)
    a = _absmax_for(L.W)
    Xb, plan = _w4_X(64, rng)
    w = S.svdq_pack_weights(L.W, a, 16, bias_bits=L.b)
    p = oracle.pack_weights(L.W, a.astype(np.float64), 16, bias_bits=L.b)
    e = w.export()
    inv = e["inv_lambda"].astype(np.float64)
    assert np.array_equal(inv, p["inv_lambda"])
    assert np.all(inv[:384] == 1.0) and np.all(inv[384:] == 2.0 ** -16)
    xc, sxo, Zo, xhat = oracle.quantize_act(Xb, p["inv_lambda"], p["L1b"])
    _assert_w4_ranges(xhat, sxo, xc, plan)
    lin = S.SVDQLinear(w)
    xq, s_x, Z, Y = lin.buffers(64)
    lin.forward(_to_dev(Xb), out=Y)
    torch.cuda.synchronize()
    S.svdq_get_device_error(w)
    assert np.array_equal(xq.cpu().numpy(), oracle.pack_nibbles(xc)), "codes"
    assert np.array_equal(s_x.cpu().numpy().astype(np.float64), sxo), "scales"
    w.free()


# ------------------------------------------------------------------ W8A8
def _w8_X(M, rng):
    X = rng.standard_normal((M, K)) * 0.1
    X[:, 384:] = 0.0
    rows = {}
    r = np.zeros(K)                                  # ties: s = 2^-7 exactly
    r[rng.permutation(384)[:40]] = [127 * 2.0 ** -7] + \
        [sg * (k + 0.5) * 2.0 ** -7 for k in (0, 1, 2, 5, 17, 31, 62, 63, 64, 100, 125, 126,
                                              3, 9, 40, 77, 90, 111, 120, 124)
         for sg in (1, -1)][:39]
    X[0], rows["ties"] = r, 0
    r = np.zeros(K)                                  # near 63.5: s = fl32(1/127) inexact
    r[rng.permutation(384)[:5]] = [1.0, 0.5, -0.5, 0.5, -0.25]
    X[1], rows["near"] = r, 1
    r = np.zeros(K)                                  # tiny: s < 2^-64
    r[rng.permutation(384)[:6]] = [2.0 ** -70, -(2.0 ** -72), 3 * 2.0 ** -75, 2.0 ** -80,
                                   -(2.0 ** -71), 5 * 2.0 ** -78]
    X[2], rows["tiny"] = r, 2
    r = np.zeros(K)                                  # subnormal s, x / s = +-128
    r[384 + rng.permutation(128)[:4]] = [2.0 ** -126, -(2.0 ** -126), 2.0 ** -133, 3 * 2.0 ** -130]
    X[3], rows["subnormal_clamp"] = r, 3
    r = np.zeros(K)                                  # underflow: max 2^-149 after smoothing
    r[384 + rng.permutation(128)[:3]] = [2.0 ** -133, -(2.0 ** -133), 2.0 ** -133]
    X[4], rows["underflow"] = r, 4
    X[5] = 0.0
    X[6] = -0.0
    rows["zero"] = 5
    Xb = oracle.round_bf16_bits(X)
    for t in range(7):
        bf(oracle.bf16_bits_to_f64(Xb[t]))
    return Xb, rows


def test_w8a8_activation_pass_edges():
    rng = np.random.default_rng(12)
    spec = synth.layer_spec("edge_w8", 64, K, 128, 16, 502, tiny=True)
    L = synth.make_layer(spec)
    a = _absmax_for(L.W)
    Xb, rows = _w8_X(64, rng)
    w = S.svdq_pack_weights_w8a8(L.W, a, 16, bias_bits=L.b)
    p = oracle.pack_weights_w8a8(L.W, a.astype(np.float64), 16, bias_bits=L.b)
    xc, sxo, Zo, xhat = oracle.quantize_act_w8a8(Xb, p["inv_lambda"], p["L1b"])
    # ranges
    s = float(sxo[rows["ties"]])
    assert s == 2.0 ** -7
    q = [_fr(x) / _fr(s) for x in xhat[rows["ties"]] if x != 0]
    assert sum(abs(x) - int(abs(x)) == Fraction(1, 2) for x in q) >= 30
    s = float(sxo[rows["near"]])
    d = [abs(abs(_fr(x) / _fr(s)) - Fraction(127, 2)) for x in xhat[rows["near"]] if abs(x) == 0.5]
    assert d and all(0 < x <= Fraction(1, 2 ** 15) for x in d)
    assert 0 < float(sxo[rows["tiny"]]) < 2.0 ** -64
    s = float(sxo[rows["subnormal_clamp"]])
    assert 0 < s < 2.0 ** -126
    assert 127 in xc[rows["subnormal_clamp"]] and -128 in xc[rows["subnormal_clamp"]]
    assert float(sxo[rows["underflow"]]) == 0.0 and np.max(np.abs(xhat[rows["underflow"]])) > 0
    assert float(sxo[rows["zero"]]) == 0.0
    lin = S.W8A8Linear(w)
    xq, s_x, Z, Y = lin.buffers(64)
    lin.forward(_to_dev(Xb), out=Y)
    torch.cuda.synchronize()
    S.svdq_get_device_error(w)
    assert np.array_equal(xq.cpu().numpy().astype(np.int64), xc), "codes"
    assert np.array_equal(s_x.cpu().numpy().astype(np.float64), sxo), "scales"
    w.free()


# ------------------------------------------------------------------ NVFP4
def test_nvfp4_activation_pass_edges():
    from test_gpu_nvfp4 import atom_to_rows
    rng = np.random.default_rng(13)
    spec = synth.layer_spec("edge_f4", 64, K, 128, 16, 503, tiny=True)
    L = synth.make_layer(spec)
    a = _absmax_for(L.W)
    X = rng.standard_normal((64, K)) * 0.1
    X[:, 384:] = 0.0
    # row 0: row scale exactly 2^-10 (max 2688 2^-10), one group of 16 with
    # group scale 1 (max 6 2^-10) holding every E2M1 midpoint exactly
    X[0] = 0.0
    X[0, 0] = 2688 * 2.0 ** -10
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    X[0, 16:32] = [6.0 * 2.0 ** -10] + [sg * m * 2.0 ** -10 for m in mids for sg in (1, -1)] + [0.0]
    X[1] = 0.0                       # tiny row scale: 2^-60 / 2688 < 2^-64
    X[1, rng.permutation(384)[:5]] = [2.0 ** -60, -(2.0 ** -62), 2.0 ** -61, 3 * 2.0 ** -64, 2.0 ** -66]
    X[2] = 0.0
    X[3] = -0.0
    Xb = oracle.round_bf16_bits(X)
    for t in range(4):
        bf(oracle.bf16_bits_to_f64(Xb[t]))
    w = S.svdq_pack_weights_nvfp4(L.W, a, 16, bias_bits=L.b)
    e = w.export()
    inv = e["inv_lambda"].astype(np.float64)
    assert np.all(inv[:384] == 1.0)
    xc, xb, xs, Zo, xhat = oracle.quantize_act_nvfp4(Xb, inv, oracle.bf16_bits_to_f64(e["L1"]))
    assert float(xs[0]) == 2.0 ** -10 and float(xb[0, 1]) == 1.0
    d = xhat[0, 16:32] / (xb[0, 1] * xs[0])
    assert sorted(set(np.abs(d[1:15]))) == mids                     # exact midpoints
    assert 0 < float(xs[1]) < 2.0 ** -64
    assert float(xs[2]) == 0.0 and float(xs[3]) == 0.0
    lin = S.NVFP4Linear(w)
    xq, sfa, s_x, Z, Y = lin.buffers(64)
    lin.forward(_to_dev(Xb), out=Y)
    torch.cuda.synchronize()
    S.svdq_get_device_error(w)
    assert np.array_equal(xq.cpu().numpy(), oracle.pack_nibbles(xc)), "codes"
    sf_rows = atom_to_rows(sfa.cpu().numpy(), 128, K)
    assert np.array_equal(sf_rows[:64], oracle.e4m3_bits(xb)), "group scales"
    assert np.array_equal(s_x.cpu().numpy().astype(np.float64), xs), "row scales"
    w.free()


# ------------------------------------------------------------------ fusion epilogue
def test_fused_epilogue_quantiser_edges():
    """svdq_linear_quantize_next with an all-zero input: the first layer's
    output is exactly its bias, so the planted values reach the next
    layer's quantiser (smoothed with power-of-two factors) in every row."""
    rng = np.random.default_rng(14)
    M, K1, N1, N2 = 96, 256, K, 128
    L1 = synth.make_layer(synth.layer_spec("edge_f1", M, K1, N1, 8, 504, tiny=True))
    L2 = synth.make_layer(synth.layer_spec("edge_f2", M, N1, N2, 8, 505, tiny=True))
    P = _w4_group_patterns()
    kinds = ["ties", "near_a", "near_b", "tiny", "zero", "near_c", "subnormal_clamp", "underflow"]
    bias = rng.standard_normal(N1) * 0.1
    for g, kind in enumerate(kinds):
        vals = np.zeros(64)
        vals[rng.permutation(64)[:len(P[kind])]] = P[kind]
        bias[64 * g:64 * g + 64] = vals
    bias_bits = oracle.round_bf16_bits(bias)
    bf(oracle.bf16_bits_to_f64(bias_bits))
    w1 = S.svdq_pack_weights(L1.W, S.svdq_calib_absmax(L1.X), 8, bias_bits=bias_bits)
    a2 = _absmax_for(L2.W, sub_groups=(6, 7))
    w2 = S.svdq_pack_weights(L2.W, a2, 8, bias_bits=L2.b)
    e2 = w2.export()
    inv2 = e2["inv_lambda"].astype(np.float64)
    assert np.all(inv2[:384] == 1.0) and np.all(inv2[384:] == 2.0 ** -16)
    X = torch.zeros((M, K1), dtype=torch.bfloat16, device="cuda")
    lin1 = S.SVDQLinear(w1)
    H = lin1(X).clone()
    torch.cuda.synchronize()
    Hb = _bits(H)
    # H = bf16(0 + b): b itself, except that 0 + (-0) is +0 in round-to-nearest
    expect = np.where(bias_bits == 0x8000, 0, bias_bits).astype(np.uint16)
    bad = np.argwhere(Hb != np.broadcast_to(expect, (M, N1)))
    assert bad.size == 0, f"H differs from the bias at {bad[:8].tolist()}"
    xq2 = torch.full((M, N1 // 2), 0xAB, dtype=torch.uint8, device="cuda")
    s_x2 = torch.full((N1 // 64, M), -1.0, dtype=torch.float32, device="cuda")
    Z2 = torch.empty((M, 8), dtype=torch.bfloat16, device="cuda")
    nws = S.svdq_linear_quantize_next_workspace(w1, w2, M)
    ws = torch.empty((max(nws // 4, 1),), dtype=torch.float32, device="cuda")
    S.svdq_linear_quantize_next(w1, w2, lin1.xq, lin1.s_x, lin1.Z, xq2, s_x2, Z2, ws, S.EPI_NONE)
    torch.cuda.synchronize()
    S.svdq_get_device_error(w1)
    codes, s_o, Z_o, xhat = oracle.quantize_act(Hb, inv2, oracle.bf16_bits_to_f64(e2["L1"]))
    plan = [(t, g, kind) for t in (0, M - 1) for g, kind in enumerate(kinds)]
    _assert_w4_ranges(xhat, s_o, codes, plan)
    assert np.array_equal(xq2.cpu().numpy(), oracle.pack_nibbles(codes)), "codes"
    assert np.array_equal(s_x2.cpu().numpy().astype(np.float64), s_o), "scales"
    w1.free()
    w2.free()
