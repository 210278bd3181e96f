"""The library's W8A8 comparator pack (svdq_pack_weights_w8a8, host only)
against the oracle's pack_weights_w8a8: smoothing, factors (up to sign) and
the int8 residual codes and per-channel scales bit for bit; format checks
between the W4A4 and W8A8 calls."""
import ctypes
import os
import tempfile

import numpy as np
import pytest

import oracle
import synth
import w4a4_quantized_gemm_smooth_b200 as S
from helpers import column_signs


@pytest.mark.parametrize("case", ["tiny", "tall", "rank0"])
def test_w8a8_host_pack_matches_oracle(case):
    if case == "tiny":
        spec = synth.WORKLOADS["tiny"]
    elif case == "tall":
        spec = synth.layer_spec("w8_tall", 96, 640, 192, 24, 52)
    else:
        spec = synth.layer_spec("w8_r0", 64, 256, 136, 0, 53, tiny=True)
    L = synth.make_layer(spec)
    a = S.svdq_calib_absmax(L.X)
    w = S.svdq_pack_weights_w8a8(L.W, a, spec.rank, bias_bits=L.b, to_device=False)
    assert w.format == S.FORMAT_W8A8
    e = w.export()
    p = oracle.pack_weights_w8a8(L.W, a.astype(np.float64), spec.rank, bias_bits=L.b)
    assert np.array_equal(e["inv_lambda"].astype(np.float64), p["inv_lambda"])
    if spec.rank:
        sg = column_signs(e["L1"], p["L1b"])
        assert np.array_equal(oracle.bf16_bits_to_f64(e["L1"]) * sg[None, :], p["L1b"])
        assert np.array_equal(oracle.bf16_bits_to_f64(e["L2"]) * sg[:, None], p["L2b"])
    assert np.array_equal(e["wq8"].astype(np.int64), p["wcodes8"])
    assert np.array_equal(e["s_w8"].astype(np.float64), p["s_w8"])
    assert np.array_equal(e["bias"], L.b)
    w.free()


def test_formats_are_not_interchangeable():
    L = synth.make_layer(synth.WORKLOADS["tiny"])
    a = S.svdq_calib_absmax(L.X)
    w8 = S.svdq_pack_weights_w8a8(L.W, a, 16, to_device=False)
    w4 = S.svdq_pack_weights_host(L.W, a, 16)
    assert w4.format == S.FORMAT_W4A4 and w8.format == S.FORMAT_W8A8
    lib = S.lib()
    vp = ctypes.c_void_p
    buf = np.zeros(1 << 16, np.uint8)
    p = buf.ctypes.data_as(vp)
    # hot-path calls check the handle's format before touching any device
    assert lib.svdq_quantize_act(w8.handle, 16, p, 512, p, p, p, None) == 1
    assert lib.svdq_linear(w8.handle, 16, p, p, p, p, 512, 0, None) == 1
    assert lib.svdq_quantize_act_w8a8(w4.handle, 16, p, 512, p, p, p, None) == 1
    assert lib.svdq_linear_w8a8(w4.handle, 16, p, p, p, p, 512, 0, None) == 1
    assert lib.svdq_quantize_act_w8a8(w8.handle, 16, p, 512, p, p, p, None) == 1  # host-only
    assert lib.svdq_weights_export_w8a8(w4.handle, p, p) == 1
    assert lib.svdq_weights_format(None) == -1
    with tempfile.TemporaryDirectory() as d, pytest.raises(S.SVDQError):
        w8.save(os.path.join(d, "w8.svdq"))                    # save/load are W4A4 only
    w8.free()
    w4.free()


def test_w8a8_pack_argument_errors():
    L = synth.make_layer(synth.WORKLOADS["tiny"])
    a = S.svdq_calib_absmax(L.X)
    with pytest.raises(S.SVDQError):
        S.svdq_pack_weights_w8a8(L.W[:, :500], a[:500], 16, to_device=False)   # K % 64
    with pytest.raises(S.SVDQError):
        S.svdq_pack_weights_w8a8(L.W, a, 12, to_device=False)                  # rank % 8
    with pytest.raises(S.SVDQError):
        S.svdq_pack_weights_w8a8(L.W, a, 16, alpha=1.0, to_device=False)
