"""GPU parity of svdq_linear_splitk (split-K form for small batches): the
same operation as svdq_linear up to fp32 summation order, checked against
the oracle's bf16 Y (relative Frobenius <= 2e-3), against svdq_linear, and
for repeatability (two calls in a row give identical bits: the arrival
counters are left at zero)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
import w4a4_quantized_gemm_smooth_b200 as S
from helpers import Y_REL_FRO, rel_fro

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


def _layer(M, K, N, r, seed, lora=0):
    spec = synth.layer_spec(f"sk_{M}_{K}_{N}_{r}", M, K, N, r, seed, lora_rank=lora)
    L = synth.make_layer(spec)
    w = S.svdq_pack_weights(L.W, S.svdq_calib_absmax(L.X), r, bias_bits=L.b,
                            lora_A_bits=L.A, lora_B_bits=L.B)
    lin = S.SVDQLinear(w)
    xq, s_x, Z, Y = lin.buffers(M)
    S.svdq_quantize_act(w, _to_dev(L.X), xq, s_x, Z)
    return w, xq, s_x, Z, Y


@pytest.mark.parametrize("M,K,N,r,splits", [
    (256, 1152, 1152, 16, 0),     # PixArt, smallest batch; 128-column tiles; automatic split
    (256, 1152, 1152, 16, 5),     # uneven group ranges (18 groups / 5)
    (130, 320, 136, 24, 2),       # ragged M and N, 5 groups
    (256, 4608, 1152, 64, 0),     # long K, rank 64
    (384, 3072, 3072, 32, 3),     # 256-column tiles
])
def test_splitk_matches_oracle_and_linear(M, K, N, r, splits):
    w, xq, s_x, Z, Y = _layer(M, K, N, r, 500 + M + K + r)
    S.svdq_linear(w, xq, s_x, Z, Y)
    ws = torch.empty(S.svdq_linear_splitk_workspace(w, M, splits), dtype=torch.uint8, device="cuda")
    Ys = torch.empty_like(Y)
    S.svdq_linear_splitk(w, xq, s_x, Z, Ys, ws, splits)
    first = _bits(Ys).copy()
    Ys.zero_()
    S.svdq_linear_splitk(w, xq, s_x, Z, Ys, ws, splits)      # counters reset by the first call
    torch.cuda.synchronize()
    S.svdq_get_device_error(w)
    assert np.array_equal(first, _bits(Ys)), "second call differs"
    e = w.export()
    xc = oracle.unpack_nibbles(xq.cpu().numpy())
    Zg = oracle.bf16_bits_to_f64(_bits(Z)) if r else np.zeros((M, 0))
    _, Yo = oracle.linear(xc, s_x.cpu().numpy().astype(np.float64), Zg,
                          oracle.unpack_nibbles(e["wq"]), e["s_w"].astype(np.float64),
                          oracle.bf16_bits_to_f64(e["L2"]), oracle.bf16_bits_to_f64(e["bias"]))
    Yk = oracle.bf16_bits_to_f64(_bits(Ys))
    assert rel_fro(Yk, Yo) <= Y_REL_FRO
    assert rel_fro(Yk, oracle.bf16_bits_to_f64(_bits(Y))) <= 1e-3
    w.free()


def test_splitk_argument_errors():
    w, xq, s_x, Z, Y = _layer(128, 256, 128, 8, 77)
    lib = S.lib()
    vp = ctypes.c_void_p
    need = S.svdq_linear_splitk_workspace(w, 128, 2)
    assert need > 0
    assert S.svdq_linear_splitk_workspace(w, 128, 5) == 0          # more splits than groups
    ws = torch.empty(need + 512, dtype=torch.uint8, device="cuda")
    st = vp(torch.cuda.current_stream().cuda_stream)
    args = (w.handle, 128, vp(xq.data_ptr()), vp(s_x.data_ptr()), vp(Z.data_ptr()),
            vp(Y.data_ptr()), 128, 0)
    assert lib.svdq_linear_splitk(*args, 2, vp(ws.data_ptr()), need - 1, st) == 2     # too small
    assert lib.svdq_linear_splitk(*args, 2, vp(ws.data_ptr() + 16), need, st) == 3    # misaligned
    assert lib.svdq_linear_splitk(*args, 17, vp(ws.data_ptr()), need, st) == 1       # bad splits
    assert lib.svdq_linear_splitk(*args, 2, None, need, st) == 1                      # no workspace
    torch.cuda.synchronize()
    S.svdq_get_device_error(w)
    w.free()


def test_single_split_is_the_plain_kernel():
    w, xq, s_x, Z, Y = _layer(1024, 1152, 4608, 32, 91)     # tiles fill the GPU: automatic = 1
    S.svdq_linear(w, xq, s_x, Z, Y)
    ws = torch.empty(S.svdq_linear_splitk_workspace(w, 1024, 0), dtype=torch.uint8, device="cuda")
    Ys = torch.empty_like(Y)
    S.svdq_linear_splitk(w, xq, s_x, Z, Ys, ws, 0)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(Y), _bits(Ys))
    w.free()
