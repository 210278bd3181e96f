"""A bounded device wait that runs out, on the GPU, without a fault.

svdq_debug_linear_stall runs the W4A4 product with every device wait
bounded by a short limit while the first CTA's TMA producer withholds its
first stage: the warps waiting for that stage give up after the bound,
raise the handle's sticky error word and leave the kernel.  The host then
reads SVDQ_ERR_DEVICE_TIMEOUT, and the same handle and context keep
working: a normal call afterwards reproduces the earlier output bit for
bit and reports no error.  Nothing here faults, traps or hangs the GPU.
"""
import numpy as np
import pytest
import torch

import synth
import w4a4_quantized_gemm_smooth_b200 as S

pytestmark = pytest.mark.gpu

SVDQ_ERR_DEVICE_TIMEOUT = 7


def _bits(t):
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("M,K,N,r", [
    (128, 256, 128, 16),      # one tile, one CTA
    (256, 512, 512, 16),      # several CTAs: only the first one stalls
])
def test_stalled_stage_times_out_and_handle_recovers(M, K, N, r):
    assert torch.cuda.is_available()
    spec = synth.layer_spec(f"stall_{M}_{K}_{N}", M, K, N, r, 61 + M, tiny=True)
    L = synth.make_layer(spec)
    w = S.svdq_pack_weights(L.W, S.svdq_calib_absmax(L.X), r, bias_bits=L.b)
    lin = S.SVDQLinear(w)
    xq, s_x, Z, Y = lin.buffers(M)
    X = torch.from_numpy(L.X.view(np.int16)).view(torch.bfloat16).cuda()
    S.svdq_quantize_act(w, X, xq, s_x, Z)
    S.svdq_linear(w, xq, s_x, Z, Y)
    S.svdq_get_device_error(w)                      # raises on any error: none expected
    ref = _bits(Y).copy()

    Y2 = torch.zeros_like(Y)
    S.svdq_debug_linear_stall(w, xq, s_x, Z, Y2, limit_us=200)
    rc = S.lib().svdq_get_device_error(w.handle, None)
    assert rc == SVDQ_ERR_DEVICE_TIMEOUT
    assert S.lib().svdq_get_device_error(w.handle, None) == 0      # read and cleared
    assert not np.array_equal(_bits(Y2), ref)       # the stalled CTA left its tile unwritten

    Y3 = torch.zeros_like(Y)
    S.svdq_linear(w, xq, s_x, Z, Y3)
    S.svdq_get_device_error(w)
    assert np.array_equal(_bits(Y3), ref)
    w.free()


def test_stall_limit_checked_on_host():
    spec = synth.layer_spec("stall_args", 128, 256, 128, 16, 62, tiny=True)
    L = synth.make_layer(spec)
    w = S.svdq_pack_weights(L.W, S.svdq_calib_absmax(L.X), 16, bias_bits=L.b)
    xq, s_x, Z, Y = S.SVDQLinear(w).buffers(128)
    with pytest.raises(S.SVDQError):
        S.svdq_debug_linear_stall(w, xq, s_x, Z, Y, limit_us=0)
    with pytest.raises(S.SVDQError):
        S.svdq_debug_linear_stall(w, xq, s_x, Z, Y, limit_us=3000000)
    torch.cuda.synchronize()
    S.svdq_get_device_error(w)
    w.free()
