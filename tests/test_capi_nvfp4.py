"""The library's NVFP4 pack (svdq_pack_weights_nvfp4, host only) against the
oracle's pack_weights_nvfp4: packed E2M1 codes, E4M3 group-scale bits and
row scales bit for bit; the scale-atom size; format checks."""
import ctypes

import numpy as np
import pytest

import oracle
import synth
import w4a4_quantized_gemm_smooth_b200 as S


@pytest.mark.parametrize("case", ["tiny", "tall", "rank0"])
def test_nvfp4_host_pack_matches_oracle(case):
    if case == "tiny":
        spec = synth.WORKLOADS["tiny"]
    elif case == "tall":
        spec = synth.layer_spec("f4_tall", 96, 640, 192, 24, 62)
    else:
        spec = synth.layer_spec("f4_r0", 64, 320, 136, 0, 63, tiny=True)
    L = synth.make_layer(spec)
    a = S.svdq_calib_absmax(L.X)
    w = S.svdq_pack_weights_nvfp4(L.W, a, spec.rank, bias_bits=L.b, to_device=False)
    assert w.format == S.FORMAT_NVFP4
    e = w.export()
    p = oracle.pack_weights_nvfp4(L.W, a.astype(np.float64), spec.rank, bias_bits=L.b)
    assert np.array_equal(e["inv_lambda"].astype(np.float64), p["inv_lambda"])
    assert np.array_equal(e["wq4"], oracle.pack_nibbles(p["wcodes4"]))
    assert np.array_equal(e["sf4"], oracle.e4m3_bits(p["wb4"]))
    assert np.array_equal(e["s_w4"].astype(np.float64), p["ws4"])
    w.free()


def test_sf_bytes_and_format_checks():
    assert S.svdq_nvfp4_sf_bytes(1, 64) == 512
    assert S.svdq_nvfp4_sf_bytes(129, 320) == 2 * 5 * 512
    assert S.svdq_nvfp4_sf_bytes(128, 100) == 0
    L = synth.make_layer(synth.WORKLOADS["tiny"])
    a = S.svdq_calib_absmax(L.X)
    w4 = S.svdq_pack_weights_host(L.W, a, 16)
    f4 = S.svdq_pack_weights_nvfp4(L.W, a, 16, to_device=False)
    lib = S.lib()
    vp = ctypes.c_void_p
    buf = np.zeros(1 << 16, np.uint8)
    p = buf.ctypes.data_as(vp)
    assert lib.svdq_quantize_act_nvfp4(w4.handle, 16, p, 512, p, p, p, p, None) == 1
    assert lib.svdq_linear_nvfp4(w4.handle, 16, p, p, p, p, p, 512, 0, None) == 1
    assert lib.svdq_linear(f4.handle, 16, p, p, p, p, 512, 0, None) == 1
    assert lib.svdq_linear_w8a8(f4.handle, 16, p, p, p, p, 512, 0, None) == 1
    assert lib.svdq_weights_export_nvfp4(w4.handle, p, p, p) == 1
    w4.free()
    f4.free()
