"""CPU checks of the cross-layer fusion's host side: argument validation of
svdq_linear_quantize_next and its workspace query on handles that were never
uploaded to a GPU (both return before any CUDA call), and the SVDQMLP
binding's shape check."""
import numpy as np
import pytest

import synth
import w4a4_quantized_gemm_smooth_b200 as S


def _host_pair():
    L1 = synth.make_layer(synth.layer_spec("hf1", 64, 128, 192, 8, 61, tiny=True))
    L2 = synth.make_layer(synth.layer_spec("hf2", 64, 192, 64, 8, 62, tiny=True))
    w1 = S.svdq_pack_weights_host(L1.W, S.svdq_calib_absmax(L1.X), 8, bias_bits=L1.b)
    w2 = S.svdq_pack_weights_host(L2.W, S.svdq_calib_absmax(L2.X), 8, bias_bits=L2.b)
    return w1, w2


def test_workspace_query_needs_device_handles():
    w1, w2 = _host_pair()
    assert S.svdq_linear_quantize_next_workspace(w1, w2, 64) == 0
    L = S.lib()
    assert L.svdq_linear_quantize_next_workspace(None, w2.handle, 64) == 0
    assert L.svdq_linear_quantize_next_workspace(w1.handle, None, 64) == 0
    w1.free()
    w2.free()


def test_call_rejects_host_only_handles_without_touching_a_gpu():
    w1, w2 = _host_pair()
    L = S.lib()
    # handles without device copies: SVDQ_ERR_INVALID_ARG before any CUDA call
    st = L.svdq_linear_quantize_next(w1.handle, w2.handle, 64, None, None, None, 0, None, None,
                                     None, None, 0, None)
    assert st == 1
    st = L.svdq_linear_quantize_next(None, w2.handle, 64, None, None, None, 0, None, None,
                                     None, None, 0, None)
    assert st == 1
    w1.free()
    w2.free()


def test_mlp_binding_checks_the_chained_shapes():
    w1, w2 = _host_pair()
    S.SVDQMLP(w1, w2)                        # fc2's K (192) equals fc1's N
    with pytest.raises(ValueError):
        S.SVDQMLP(w2, w1)                    # fc1's K (128) is not fc2's N (64)
    w1.free()
    w2.free()
