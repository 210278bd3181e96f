"""CPU checks of the C-ABI library: it loads, exports every declared symbol,
validates arguments without touching a GPU, and its host pack (lambda, SVD,
residual quantisation, LoRA concat) agrees with the oracle."""
import os
import re
import tempfile

import numpy as np
import pytest

import oracle
import synth
import w4a4_quantized_gemm_smooth_b200 as S
from helpers import column_signs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    with open(os.path.join(ROOT, "include", "svdq.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(svdq_[a-z_0-9]+)\s*\(", text)))


def test_library_loads_and_exports_every_declared_symbol():
    L = S.lib()
    names = _declared_symbols()
    assert len(names) >= 14
    for n in names:
        assert hasattr(L, n), n
    assert L.svdq_version() >= 100
    assert L.svdq_status_string(3) == b"pointer or row not 16-byte aligned"


def test_pack_argument_validation():
    L = S.lib()
    import ctypes
    W = np.zeros((64, 100), np.uint16)
    a = np.ones(100, np.float32)
    h = ctypes.c_void_p()
    p = lambda x: x.ctypes.data_as(ctypes.c_void_p)
    # K not a multiple of 64
    assert L.svdq_pack_weights_host(100, 64, 4, 64, p(W), p(a), 0.5, None, 0, None, None,
                                    1.0, ctypes.byref(h)) == 2
    W = np.zeros((64, 128), np.uint16)
    a = np.ones(128, np.float32)
    assert L.svdq_pack_weights_host(128, 64, 4, 32, p(W), p(a), 0.5, None, 0, None, None,
                                    1.0, ctypes.byref(h)) == 4       # group != 64
    assert L.svdq_pack_weights_host(128, 64, 65, 64, p(W), p(a), 0.5, None, 0, None, None,
                                    1.0, ctypes.byref(h)) == 1       # rank > min(K, N)
    assert L.svdq_pack_weights_host(128, 64, 12, 64, p(W), p(a), 0.5, None, 0, None, None,
                                    1.0, ctypes.byref(h)) == 4       # branch rank % 8 != 0
    assert L.svdq_pack_weights_host(128, 64, 8, 64, None, p(a), 0.5, None, 0, None, None,
                                    1.0, ctypes.byref(h)) == 1       # null weight
    a_bad = a.copy()
    a_bad[3] = np.inf
    assert L.svdq_pack_weights_host(128, 64, 8, 64, p(W), p(a_bad), 0.5, None, 0, None,
                                    None, 1.0, ctypes.byref(h)) == 5
    assert not h.value


def test_host_only_handle_is_rejected_by_hot_path_calls():
    spec = synth.layer_spec("v", 16, 128, 64, 8, 5, tiny=True)
    L = synth.make_layer(spec)
    a = S.svdq_calib_absmax(L.X)
    w = S.svdq_pack_weights_host(L.W, a, 8, bias_bits=L.b)
    lib = S.lib()
    assert lib.svdq_quantize_act(w.handle, 16, None, 128, None, None, None, None) == 1
    assert lib.svdq_linear(w.handle, 16, None, None, None, None, 64, 0, None) == 1
    assert lib.svdq_debug_partials(w.handle, 16, None, 0, 1, 0, 1, None, None) == 1
    assert lib.svdq_linear_host(w.handle, 16, None, 128, None, 64, 0, None, 0, None) == 1
    assert lib.svdq_linear_host_workspace(w.handle, 16) == 0
    w.free()


def test_calib_absmax_matches_oracle():
    L = synth.make_layer(synth.WORKLOADS["tiny"])
    a = S.svdq_calib_absmax(L.X[:100])
    a = S.svdq_calib_absmax(L.X[100:], a)          # running max over two batches
    assert np.array_equal(a.astype(np.float64), oracle.calib_absmax(oracle.bf16_bits_to_f64(L.X)))


@pytest.mark.parametrize("case", ["tiny", "lora", "tall", "rank0"])
def test_host_pack_matches_oracle(case):
    if case == "tiny":
        spec = synth.WORKLOADS["tiny"]
    elif case == "lora":
        spec = synth.layer_spec("lora", 128, 384, 256, 16, 21, lora_rank=8)
    elif case == "tall":       # K > N: Gram of the columns
        spec = synth.layer_spec("tall", 128, 640, 192, 24, 22)
    else:
        spec = synth.layer_spec("r0", 64, 256, 128, 0, 23, tiny=True)
    L = synth.make_layer(spec)
    a = S.svdq_calib_absmax(L.X)
    w = S.svdq_pack_weights_host(L.W, a, spec.rank, bias_bits=L.b,
                                 lora_A_bits=L.A, lora_B_bits=L.B)
    e = w.export()
    p = oracle.pack_weights(L.W, a.astype(np.float64), spec.rank, bias_bits=L.b,
                            lora_A_bits=L.A, lora_B_bits=L.B)
    r = spec.rank
    assert np.array_equal(e["inv_lambda"].astype(np.float64), p["inv_lambda"])
    assert np.max(np.abs(e["sigma"] - p["sigma"]) / p["sigma"]) < 1e-10
    sg = column_signs(e["L1"], p["L1b"])
    L1 = oracle.bf16_bits_to_f64(e["L1"]) * sg[None, :]
    L2 = oracle.bf16_bits_to_f64(e["L2"]) * sg[:, None]
    assert np.array_equal(L1, p["L1b"]) and np.array_equal(L2, p["L2b"])
    assert np.array_equal(e["wq"], p["wq"])
    assert np.array_equal(e["s_w"].astype(np.float64), p["s_w"])
    assert np.array_equal(e["bias"], L.b)
    if r:
        # the unrounded product is the rank-r truncation: compare with fp64
        prod = L1[:, :r] @ L2[:r]
        assert np.linalg.norm(prod - p["L1"] @ p["L2"]) / np.linalg.norm(p["Wt"]) < 1e-2
    w.free()


def test_save_writes_a_versioned_file():
    spec = synth.layer_spec("s", 16, 128, 64, 8, 6, tiny=True)
    L = synth.make_layer(spec)
    w = S.svdq_pack_weights_host(L.W, S.svdq_calib_absmax(L.X), 8, bias_bits=L.b)
    with tempfile.TemporaryDirectory() as d:
        path = os.path.join(d, "layer.svdq")
        w.save(path)
        with open(path, "rb") as f:
            blob = f.read()
    assert blob[:8] == b"SVDQW001"
    hdr = np.frombuffer(blob[8:32], np.int32)
    assert list(hdr[:5]) == [128, 64, 8, 0, 64]
    expect = 32 + 128 * 4 + 64 * 64 + 2 * 64 * 4 + 128 * 8 * 2 + 8 * 64 * 2 + 64 * 2 + 9 * 8
    assert len(blob) == expect
