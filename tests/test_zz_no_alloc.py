"""svdq_linear_splitk_noalloc: the split-K GEMM on the library's fixed device
scratch.  Collected last on purpose (the scratch is shared process-wide);
it also passes alone.  Two calls in a row must each reproduce the existing
entry point (svdq_linear_splitk with a caller workspace) bit for bit, the
calls must not change the device's free memory, and oversize requests are
rejected."""
import ctypes

import numpy as np
import pytest
import torch

import synth
import w4a4_quantized_gemm_smooth_b200 as S

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _layer(M, K, N, r, seed):
    spec = synth.layer_spec(f"na_{M}_{K}_{N}_{r}", M, K, N, r, seed)
    L = synth.make_layer(spec)
    w = S.svdq_pack_weights(L.W, S.svdq_calib_absmax(L.X), r, bias_bits=L.b)
    lin = S.SVDQLinear(w)
    xq, s_x, Z, Y = lin.buffers(M)
    X = torch.from_numpy(L.X.view(np.int16)).view(torch.bfloat16).cuda()
    S.svdq_quantize_act(w, X, xq, s_x, Z)
    return w, xq, s_x, Z, Y


SCRATCH = 16 << 20


def _noalloc_split(w, M, splits):
    """The split count svdq_linear_splitk_noalloc runs: an explicit one as
    given; the automatic one lowered until its workspace fits the scratch."""
    if splits:
        return splits
    ws_auto = S.svdq_linear_splitk_workspace(w, M, 0)
    sp = next(s for s in range(1, 17) if S.svdq_linear_splitk_workspace(w, M, s) == ws_auto)
    while sp > 1 and S.svdq_linear_splitk_workspace(w, M, sp) > SCRATCH:
        sp -= 1
    return sp


@pytest.mark.parametrize("M,K,N,r,splits", [
    (256, 4608, 1152, 32, 0),     # automatic split (8 ranges), 9.4 MB of scratch
    (130, 320, 136, 24, 2),       # ragged, two ranges
    (1024, 1152, 4608, 32, 0),    # tiles fill the GPU: one split, no scratch
    (256, 15360, 3072, 32, 0),    # 256-column tiles: the automatic 6 ranges need 18.9 MB; 5 fit
    (128, 12288, 9216, 32, 0),    # 36 tiles x 4 ranges need 18.9 MB; 3 fit
])
def test_noalloc_matches_splitk_twice(M, K, N, r, splits):
    assert torch.cuda.is_available()
    w, xq, s_x, Z, Y = _layer(M, K, N, r, 900 + M + r)
    sp = _noalloc_split(w, M, splits)
    if splits == 0 and S.svdq_linear_splitk_workspace(w, M, 0) > SCRATCH:
        # a single split is the plain kernel and needs no scratch
        assert sp == 1 or S.svdq_linear_splitk_workspace(w, M, sp) <= SCRATCH
    ws = torch.empty(S.svdq_linear_splitk_workspace(w, M, sp), dtype=torch.uint8, device="cuda")
    S.svdq_linear_splitk(w, xq, s_x, Z, Y, ws, sp)
    torch.cuda.synchronize()
    ref = _bits(Y).copy()
    Yn = torch.empty_like(Y)
    S.svdq_linear_splitk_noalloc(w, xq, s_x, Z, Yn, splits)     # first call: per-device set-up
    torch.cuda.synchronize()
    assert np.array_equal(_bits(Yn), ref)
    Yn.zero_()                     # load torch's own kernels before measuring free memory
    _bits(Yn)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(2):
        Yn.zero_()
        S.svdq_linear_splitk_noalloc(w, xq, s_x, Z, Yn, splits)
        torch.cuda.synchronize()
        assert np.array_equal(_bits(Yn), ref)
    assert torch.cuda.mem_get_info()[0] == free0
    S.svdq_get_device_error(w)
    w.free()


def test_noalloc_rejects_oversize_requests():
    w, xq, s_x, Z, Y = _layer(256, 1152, 21504, 32, 31)
    need = S.svdq_linear_splitk_workspace(w, 256, 4)
    assert need > (16 << 20)
    vp = ctypes.c_void_p
    st = vp(torch.cuda.current_stream().cuda_stream)
    rc = S.lib().svdq_linear_splitk_noalloc(w.handle, 256, vp(xq.data_ptr()), vp(s_x.data_ptr()),
                                            vp(Z.data_ptr()), vp(Y.data_ptr()), Y.stride(0), 0, 4,
                                            st)
    assert rc == 2
    torch.cuda.synchronize()
    S.svdq_get_device_error(w)
    w.free()
