"""Python binding of the SVDQuant W4A4 linear-layer library (libsvdq.so).

Argument marshalling only: every step of the layer runs in the C-ABI
library (host pack code and sm_100a kernels).  PyTorch supplies device
memory and the current CUDA stream.  The binding never falls back to another
implementation: if the library is missing it raises.

The call names follow include/svdq.h:
    svdq_calib_absmax, svdq_pack_weights, svdq_pack_weights_host,
    svdq_weights_export, svdq_weights_save, svdq_weights_load,
    svdq_quantize_act, svdq_linear, svdq_get_device_error,
    svdq_debug_partials, svdq_linear_splitk*, svdq_pack_weights_calibrated,
    the W8A8 comparator svdq_pack_weights_w8a8, svdq_quantize_act_w8a8,
    svdq_linear_w8a8, and the NVFP4 variant svdq_pack_weights_nvfp4,
    svdq_quantize_act_nvfp4, svdq_linear_nvfp4, and the cross-layer fusion
    svdq_linear_quantize_next
and SVDQLinear / W8A8Linear / NVFP4Linear bundle one packed layer with its
two hot-path calls; SVDQMLP chains two layers (fc1, GELU, fc2) with or
without the fusion.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

__all__ = [
    "lib", "SVDQError", "Weights", "SVDQLinear", "svdq_calib_absmax",
    "svdq_pack_weights", "svdq_pack_weights_host", "svdq_weights_load",
    "svdq_quantize_act", "svdq_linear", "svdq_get_device_error",
    "svdq_debug_partials", "EPI_NONE", "EPI_GELU", "LIB_PATH",
    "svdq_pack_weights_w8a8", "svdq_quantize_act_w8a8", "svdq_linear_w8a8", "W8A8Linear",
    "FORMAT_W4A4", "FORMAT_W8A8", "FORMAT_NVFP4", "svdq_pack_weights_nvfp4",
    "svdq_quantize_act_nvfp4", "svdq_linear_nvfp4", "svdq_nvfp4_sf_bytes", "NVFP4Linear",
    "svdq_linear_quantize_next", "svdq_linear_quantize_next_workspace", "SVDQMLP",
    "svdq_linear_host", "svdq_linear_host_workspace",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_lib", "libsvdq.so")
EPI_NONE = 0
EPI_GELU = 1
FORMAT_W4A4 = 0
FORMAT_W8A8 = 1
FORMAT_NVFP4 = 2

_STATUS = {
    0: "SVDQ_OK", 1: "SVDQ_ERR_INVALID_ARG", 2: "SVDQ_ERR_SHAPE",
    3: "SVDQ_ERR_ALIGNMENT", 4: "SVDQ_ERR_UNSUPPORTED", 5: "SVDQ_ERR_NUMERIC",
    6: "SVDQ_ERR_CUDA", 7: "SVDQ_ERR_DEVICE_TIMEOUT", 8: "SVDQ_ERR_OOM",
    9: "SVDQ_ERR_IO",
}


class SVDQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_STATUS.get(status, status)}")


_lib = None
_vp = ctypes.c_void_p
_i = ctypes.c_int


def lib() -> ctypes.CDLL:
    """Load libsvdq.so (built in-tree by `python -m
    w4a4_quantized_gemm_smooth_b200.build`).  Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m w4a4_quantized_gemm_smooth_b200.build` (no fallback exists)")
    L = ctypes.CDLL(LIB_PATH)
    sig = {
        "svdq_status_string": (ctypes.c_char_p, [_i]),
        "svdq_version": (_i, []),
        "svdq_calib_absmax": (_i, [_i, _i, _vp, _i, _vp]),
        "svdq_pack_weights": (_i, [_i, _i, _i, _i, _vp, _vp, ctypes.c_double, _vp, _i,
                                   _vp, _vp, ctypes.c_float, _vp, _vp]),
        "svdq_pack_weights_host": (_i, [_i, _i, _i, _i, _vp, _vp, ctypes.c_double, _vp,
                                        _i, _vp, _vp, ctypes.c_float, _vp]),
        "svdq_weights_info": (_i, [_vp, _vp, _vp, _vp, _vp, _vp]),
        "svdq_pack_weights_calibrated": (_i, [_i, _i, _i, _i, _vp, _vp, _i, _i, _i, _vp, _i,
                                              _i, _vp, _i, _vp, _vp, ctypes.c_float, _i, _vp,
                                              _vp, _vp]),
        "svdq_weights_export": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
        "svdq_weights_save": (_i, [_vp, ctypes.c_char_p]),
        "svdq_weights_load": (_i, [ctypes.c_char_p, _vp, _vp]),
        "svdq_weights_free": (None, [_vp]),
        "svdq_quantize_act": (_i, [_vp, _i, _vp, _i, _vp, _vp, _vp, _vp]),
        "svdq_linear": (_i, [_vp, _i, _vp, _vp, _vp, _vp, _i, _i, _vp]),
        "svdq_get_device_error": (_i, [_vp, _vp]),
        "svdq_debug_partials": (_i, [_vp, _i, _vp, _i, _i, _i, _i, _vp, _vp]),
        "svdq_debug_linear_stall": (_i, [_vp, _i, _vp, _vp, _vp, _vp, _i, ctypes.c_uint, _vp]),
        "svdq_linear_splitk_workspace": (ctypes.c_size_t, [_vp, _i, _i]),
        "svdq_linear_splitk": (_i, [_vp, _i, _vp, _vp, _vp, _vp, _i, _i, _i, _vp,
                                    ctypes.c_size_t, _vp]),
        "svdq_linear_splitk_noalloc": (_i, [_vp, _i, _vp, _vp, _vp, _vp, _i, _i, _i, _vp]),
        "svdq_pack_weights_w8a8": (_i, [_i, _i, _i, _vp, _vp, ctypes.c_double, _vp, _i, _vp,
                                        _vp]),
        "svdq_weights_export_w8a8": (_i, [_vp, _vp, _vp]),
        "svdq_weights_format": (_i, [_vp]),
        "svdq_quantize_act_w8a8": (_i, [_vp, _i, _vp, _i, _vp, _vp, _vp, _vp]),
        "svdq_linear_w8a8": (_i, [_vp, _i, _vp, _vp, _vp, _vp, _i, _i, _vp]),
        "svdq_pack_weights_nvfp4": (_i, [_i, _i, _i, _vp, _vp, ctypes.c_double, _vp, _i, _vp,
                                         _vp]),
        "svdq_weights_export_nvfp4": (_i, [_vp, _vp, _vp, _vp]),
        "svdq_nvfp4_sf_bytes": (ctypes.c_size_t, [_i, _i]),
        "svdq_quantize_act_nvfp4": (_i, [_vp, _i, _vp, _i, _vp, _vp, _vp, _vp, _vp]),
        "svdq_linear_nvfp4": (_i, [_vp, _i, _vp, _vp, _vp, _vp, _vp, _i, _i, _vp]),
        "svdq_linear_host_workspace": (ctypes.c_size_t, [_vp, _i]),
        "svdq_linear_host": (_i, [_vp, _i, _vp, _i, _vp, _i, _i, _vp, ctypes.c_size_t, _vp]),
        "svdq_linear_quantize_next_workspace": (ctypes.c_size_t, [_vp, _vp, _i]),
        "svdq_linear_quantize_next": (_i, [_vp, _vp, _i, _vp, _vp, _vp, _i, _vp, _vp, _vp, _vp,
                                           ctypes.c_size_t, _vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _check(status: int, where: str):
    if status != 0:
        raise SVDQError(status, where)


def _np_ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(_vp)


def _stream_ptr(stream=None):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return _vp(stream.cuda_stream)


def _dev_ptr(t):
    return None if t is None else _vp(t.data_ptr())


class Weights:
    """Owns one packed layer handle (svdq_weights*)."""

    def __init__(self, handle: ctypes.c_void_p):
        self._h = handle
        K, N, r, sr, lr = (ctypes.c_int() for _ in range(5))
        _check(lib().svdq_weights_info(handle, ctypes.byref(K), ctypes.byref(N),
                                       ctypes.byref(r), ctypes.byref(sr),
                                       ctypes.byref(lr)), "svdq_weights_info")
        self.K, self.N, self.rank = K.value, N.value, r.value
        self.svd_rank, self.lora_rank = sr.value, lr.value
        self.format = int(lib().svdq_weights_format(handle))

    @property
    def handle(self):
        return self._h

    def export(self) -> dict:
        K, N, r = self.K, self.N, self.rank
        out = dict(
            inv_lambda=np.empty(K, np.float32), wq=np.empty((N, K // 2), np.uint8),
            s_w=np.empty((K // 64, N), np.float32), L1=np.empty((K, r), np.uint16),
            L2=np.empty((r, N), np.uint16), bias=np.empty(N, np.uint16),
            sigma=np.empty(self.svd_rank + 1, np.float64))
        _check(lib().svdq_weights_export(
            self._h, _np_ptr(out["inv_lambda"]), _np_ptr(out["wq"]), _np_ptr(out["s_w"]),
            _np_ptr(out["L1"]), _np_ptr(out["L2"]), _np_ptr(out["bias"]),
            _np_ptr(out["sigma"])), "svdq_weights_export")
        if self.format == FORMAT_W8A8:
            out["wq8"] = np.empty((N, K), np.int8)
            out["s_w8"] = np.empty(N, np.float32)
            _check(lib().svdq_weights_export_w8a8(self._h, _np_ptr(out["wq8"]),
                                                  _np_ptr(out["s_w8"])), "svdq_weights_export_w8a8")
        if self.format == FORMAT_NVFP4:
            out["wq4"] = np.empty((N, K // 2), np.uint8)
            out["sf4"] = np.empty((N, K // 16), np.uint8)
            out["s_w4"] = np.empty(N, np.float32)
            _check(lib().svdq_weights_export_nvfp4(self._h, _np_ptr(out["wq4"]), _np_ptr(out["sf4"]),
                                                   _np_ptr(out["s_w4"])), "svdq_weights_export_nvfp4")
        return out

    def save(self, path: str):
        _check(lib().svdq_weights_save(self._h, path.encode()), "svdq_weights_save")

    def free(self):
        if self._h:
            lib().svdq_weights_free(self._h)
            self._h = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def svdq_calib_absmax(X_bits: np.ndarray, absmax: np.ndarray | None = None) -> np.ndarray:
    """Running per-channel max|X| of a host bf16 matrix (uint16 bits [M, K])."""
    X_bits = np.ascontiguousarray(X_bits, dtype=np.uint16)
    M, K = X_bits.shape
    if absmax is None:
        absmax = np.zeros(K, np.float32)
    _check(lib().svdq_calib_absmax(M, K, _np_ptr(X_bits), K, _np_ptr(absmax)),
           "svdq_calib_absmax")
    return absmax


def _pack_args(W_bits, act_absmax, bias_bits, lora_A_bits, lora_B_bits):
    W_bits = np.ascontiguousarray(W_bits, dtype=np.uint16)
    act_absmax = np.ascontiguousarray(act_absmax, dtype=np.float32)
    bias_bits = None if bias_bits is None else np.ascontiguousarray(bias_bits, dtype=np.uint16)
    A = None if lora_A_bits is None else np.ascontiguousarray(lora_A_bits, dtype=np.uint16)
    B = None if lora_B_bits is None else np.ascontiguousarray(lora_B_bits, dtype=np.uint16)
    lr = 0 if A is None else A.shape[1]
    return W_bits, act_absmax, bias_bits, A, B, lr


def svdq_pack_weights(W_bits, act_absmax, rank, alpha=0.5, bias_bits=None,
                      lora_A_bits=None, lora_B_bits=None, lora_scale=1.0,
                      stream=None) -> Weights:
    """Offline pack onto the current CUDA device (see include/svdq.h)."""
    W_bits, act_absmax, bias_bits, A, B, lr = _pack_args(
        W_bits, act_absmax, bias_bits, lora_A_bits, lora_B_bits)
    N, K = W_bits.shape
    h = _vp()
    _check(lib().svdq_pack_weights(K, N, int(rank), 64, _np_ptr(W_bits), _np_ptr(act_absmax),
                                   float(alpha), _np_ptr(bias_bits), lr, _np_ptr(A),
                                   _np_ptr(B), float(lora_scale), _stream_ptr(stream),
                                   ctypes.byref(h)), "svdq_pack_weights")
    return Weights(h)


def svdq_pack_weights_host(W_bits, act_absmax, rank, alpha=0.5, bias_bits=None,
                           lora_A_bits=None, lora_B_bits=None, lora_scale=1.0) -> Weights:
    """Same transform without a GPU (host copies only)."""
    W_bits, act_absmax, bias_bits, A, B, lr = _pack_args(
        W_bits, act_absmax, bias_bits, lora_A_bits, lora_B_bits)
    N, K = W_bits.shape
    h = _vp()
    _check(lib().svdq_pack_weights_host(K, N, int(rank), 64, _np_ptr(W_bits),
                                        _np_ptr(act_absmax), float(alpha), _np_ptr(bias_bits),
                                        lr, _np_ptr(A), _np_ptr(B), float(lora_scale),
                                        ctypes.byref(h)), "svdq_pack_weights_host")
    return Weights(h)


def svdq_pack_weights_calibrated(W_bits, X_cal_bits, rank, alphas=(0.3, 0.4, 0.5, 0.6, 0.7),
                                 refine_iters=1, bias_bits=None, lora_A_bits=None,
                                 lora_B_bits=None, lora_scale=1.0, to_device=True, stream=None,
                                 gptq=False):
    """Pack with the calibrated alpha search, the alternating factor
    refinement and, with gptq=True, GPTQ rounding of the residual.
    X_cal_bits: host bf16 bits [M_cal, K] (calibration tokens).
    Returns (Weights, errors per alpha)."""
    X_cal_bits = np.ascontiguousarray(X_cal_bits, dtype=np.uint16)
    W_bits, _, bias_bits, A, B, lr = _pack_args(
        W_bits, np.zeros(X_cal_bits.shape[1], np.float32), bias_bits, lora_A_bits, lora_B_bits)
    N, K = W_bits.shape
    al = np.ascontiguousarray(alphas, dtype=np.float64)
    errs = np.zeros(len(al), np.float64)
    h = _vp()
    _check(lib().svdq_pack_weights_calibrated(
        K, N, int(rank), 64, _np_ptr(W_bits), _np_ptr(X_cal_bits), X_cal_bits.shape[0], K,
        len(al), _np_ptr(al), int(refine_iters), 1 if gptq else 0, _np_ptr(bias_bits), lr,
        _np_ptr(A), _np_ptr(B),
        float(lora_scale), 1 if to_device else 0, _stream_ptr(stream) if to_device else None,
        _np_ptr(errs), ctypes.byref(h)), "svdq_pack_weights_calibrated")
    return Weights(h), errs


def svdq_weights_load(path: str, stream=None) -> Weights:
    h = _vp()
    _check(lib().svdq_weights_load(path.encode(), _stream_ptr(stream), ctypes.byref(h)),
           "svdq_weights_load")
    return Weights(h)


def svdq_quantize_act(w: Weights, X, xq, s_x, Z=None, stream=None):
    """X: cuda bf16 [M, K] (row stride X.stride(0)); xq uint8 [M, K/2];
    s_x float32 [K/64, M]; Z bf16 [M, rank] or None when rank == 0."""
    M = X.shape[0]
    _check(lib().svdq_quantize_act(w.handle, M, _dev_ptr(X), X.stride(0), _dev_ptr(xq),
                                   _dev_ptr(s_x), _dev_ptr(Z), _stream_ptr(stream)),
           "svdq_quantize_act")


def svdq_linear(w: Weights, xq, s_x, Z, Y, epilogue=EPI_NONE, stream=None):
    """Y: cuda bf16 [M, N] (row stride Y.stride(0))."""
    M = Y.shape[0]
    _check(lib().svdq_linear(w.handle, M, _dev_ptr(xq), _dev_ptr(s_x), _dev_ptr(Z),
                             _dev_ptr(Y), Y.stride(0), int(epilogue), _stream_ptr(stream)),
           "svdq_linear")


def svdq_linear_host_workspace(w: Weights, M: int) -> int:
    """Device workspace bytes of svdq_linear_host (0 for invalid arguments)."""
    return int(lib().svdq_linear_host_workspace(w.handle, int(M)))


def svdq_linear_host(w: Weights, X, Y, workspace, epilogue=EPI_NONE, stream=None):
    """The layer from host memory: X CPU bf16 [M, K] (row stride X.stride(0)),
    Y CPU bf16 [M, N] (row stride Y.stride(0)), both ideally pinned;
    workspace: cuda tensor of at least svdq_linear_host_workspace(w, M)
    bytes.  Enqueues the copies and both kernels on the stream; Y is valid
    after it has been synchronised."""
    M = X.shape[0]
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().svdq_linear_host(w.handle, M, _vp(X.data_ptr()), X.stride(0), _vp(Y.data_ptr()),
                                  Y.stride(0), int(epilogue), _dev_ptr(workspace), nbytes,
                                  _stream_ptr(stream)),
           "svdq_linear_host")


def svdq_linear_quantize_next_workspace(w: Weights, w_next: Weights, M: int) -> int:
    """Workspace bytes of svdq_linear_quantize_next (the column tiles'
    partial Z_next, fp32; 0 when rank_next == 0 or for invalid arguments)."""
    return int(lib().svdq_linear_quantize_next_workspace(w.handle, w_next.handle, int(M)))


def svdq_linear_quantize_next(w: Weights, w_next: Weights, xq, s_x, Z, xq_next, s_x_next,
                              Z_next, workspace, epilogue=EPI_NONE, stream=None):
    """The layer of w with the next layer's activation pass in its epilogue:
    writes xq_next uint8 [M, N/2], s_x_next float32 [N/64, M] and Z_next bf16
    [M, rank_next] (None when rank_next == 0) instead of Y.  workspace: cuda
    tensor of at least svdq_linear_quantize_next_workspace(w, w_next, M)
    bytes (None when rank_next == 0)."""
    M = xq.shape[0]
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().svdq_linear_quantize_next(w.handle, w_next.handle, M, _dev_ptr(xq),
                                           _dev_ptr(s_x), _dev_ptr(Z), int(epilogue),
                                           _dev_ptr(xq_next), _dev_ptr(s_x_next),
                                           _dev_ptr(Z_next), _dev_ptr(workspace), nbytes,
                                           _stream_ptr(stream)),
           "svdq_linear_quantize_next")


def svdq_linear_splitk_workspace(w: Weights, M: int, splits: int = 0) -> int:
    """Workspace bytes of svdq_linear_splitk (0 for invalid arguments)."""
    return int(lib().svdq_linear_splitk_workspace(w.handle, int(M), int(splits)))


def svdq_linear_splitk(w: Weights, xq, s_x, Z, Y, workspace, splits=0, epilogue=EPI_NONE,
                       stream=None):
    """Split-K svdq_linear.  workspace: cuda tensor of at least
    svdq_linear_splitk_workspace(w, M, splits) bytes (256-byte aligned)."""
    M = Y.shape[0]
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().svdq_linear_splitk(w.handle, M, _dev_ptr(xq), _dev_ptr(s_x), _dev_ptr(Z),
                                    _dev_ptr(Y), Y.stride(0), int(epilogue), int(splits),
                                    _dev_ptr(workspace), nbytes, _stream_ptr(stream)),
           "svdq_linear_splitk")


def svdq_linear_splitk_noalloc(w: Weights, xq, s_x, Z, Y, splits=0, epilogue=EPI_NONE,
                               stream=None):
    """svdq_linear_splitk with the library's fixed device scratch (no allocation)."""
    M = Y.shape[0]
    _check(lib().svdq_linear_splitk_noalloc(w.handle, M, _dev_ptr(xq), _dev_ptr(s_x),
                                            _dev_ptr(Z), _dev_ptr(Y), Y.stride(0),
                                            int(epilogue), int(splits), _stream_ptr(stream)),
           "svdq_linear_splitk_noalloc")


def svdq_pack_weights_w8a8(W_bits, act_absmax, rank, alpha=0.5, bias_bits=None, to_device=True,
                           stream=None) -> Weights:
    """Offline pack of the W8A8 comparator (int8 residual per output channel)."""
    W_bits, act_absmax, bias_bits, _, _, _ = _pack_args(W_bits, act_absmax, bias_bits, None, None)
    N, K = W_bits.shape
    h = _vp()
    _check(lib().svdq_pack_weights_w8a8(K, N, int(rank), _np_ptr(W_bits), _np_ptr(act_absmax),
                                        float(alpha), _np_ptr(bias_bits), 1 if to_device else 0,
                                        _stream_ptr(stream) if to_device else None,
                                        ctypes.byref(h)), "svdq_pack_weights_w8a8")
    return Weights(h)


def svdq_quantize_act_w8a8(w: Weights, X, xq, s_x, Z=None, stream=None):
    """X: cuda bf16 [M, K]; xq int8 [M, K]; s_x float32 [M]; Z bf16 [M, rank]."""
    M = X.shape[0]
    _check(lib().svdq_quantize_act_w8a8(w.handle, M, _dev_ptr(X), X.stride(0), _dev_ptr(xq),
                                        _dev_ptr(s_x), _dev_ptr(Z), _stream_ptr(stream)),
           "svdq_quantize_act_w8a8")


def svdq_linear_w8a8(w: Weights, xq, s_x, Z, Y, epilogue=EPI_NONE, stream=None):
    """Y: cuda bf16 [M, N] (row stride Y.stride(0))."""
    M = Y.shape[0]
    _check(lib().svdq_linear_w8a8(w.handle, M, _dev_ptr(xq), _dev_ptr(s_x), _dev_ptr(Z),
                                  _dev_ptr(Y), Y.stride(0), int(epilogue), _stream_ptr(stream)),
           "svdq_linear_w8a8")


def svdq_pack_weights_nvfp4(W_bits, act_absmax, rank, alpha=0.5, bias_bits=None, to_device=True,
                            stream=None) -> Weights:
    """Offline pack of the NVFP4 variant (E2M1 residual, E4M3 group scales)."""
    W_bits, act_absmax, bias_bits, _, _, _ = _pack_args(W_bits, act_absmax, bias_bits, None, None)
    N, K = W_bits.shape
    h = _vp()
    _check(lib().svdq_pack_weights_nvfp4(K, N, int(rank), _np_ptr(W_bits), _np_ptr(act_absmax),
                                         float(alpha), _np_ptr(bias_bits), 1 if to_device else 0,
                                         _stream_ptr(stream) if to_device else None,
                                         ctypes.byref(h)), "svdq_pack_weights_nvfp4")
    return Weights(h)


def svdq_nvfp4_sf_bytes(rows: int, K: int) -> int:
    return int(lib().svdq_nvfp4_sf_bytes(int(rows), int(K)))


def svdq_quantize_act_nvfp4(w: Weights, X, xq, sfa, s_x, Z=None, stream=None):
    """X: cuda bf16 [M, K]; xq uint8 [M, K/2]; sfa uint8 [svdq_nvfp4_sf_bytes(M, K)];
    s_x float32 [M]; Z bf16 [M, rank] (stored divided by s_x)."""
    M = X.shape[0]
    _check(lib().svdq_quantize_act_nvfp4(w.handle, M, _dev_ptr(X), X.stride(0), _dev_ptr(xq),
                                         _dev_ptr(sfa), _dev_ptr(s_x), _dev_ptr(Z),
                                         _stream_ptr(stream)), "svdq_quantize_act_nvfp4")


def svdq_linear_nvfp4(w: Weights, xq, sfa, s_x, Z, Y, epilogue=EPI_NONE, stream=None):
    """Y: cuda bf16 [M, N] (row stride Y.stride(0))."""
    M = Y.shape[0]
    _check(lib().svdq_linear_nvfp4(w.handle, M, _dev_ptr(xq), _dev_ptr(sfa), _dev_ptr(s_x),
                                   _dev_ptr(Z), _dev_ptr(Y), Y.stride(0), int(epilogue),
                                   _stream_ptr(stream)), "svdq_linear_nvfp4")


def svdq_get_device_error(w: Weights, stream=None):
    _check(lib().svdq_get_device_error(w.handle, _stream_ptr(stream)), "device")


def svdq_debug_linear_stall(w: Weights, xq, s_x, Z, Y, limit_us=200, stream=None):
    """Test hook: svdq_linear with every device wait bounded by limit_us and
    the first CTA's first stage withheld (see include/svdq.h)."""
    M = Y.shape[0]
    _check(lib().svdq_debug_linear_stall(w.handle, M, _dev_ptr(xq), _dev_ptr(s_x), _dev_ptr(Z),
                                         _dev_ptr(Y), Y.stride(0), ctypes.c_uint(int(limit_us)),
                                         _stream_ptr(stream)), "svdq_debug_linear_stall")


def svdq_debug_partials(w: Weights, M, xq, row0, nrows, col0, ncols, P, stream=None):
    """P: cuda int32 [K/64, nrows, ncols]."""
    _check(lib().svdq_debug_partials(w.handle, int(M), _dev_ptr(xq), int(row0), int(nrows),
                                     int(col0), int(ncols), _dev_ptr(P), _stream_ptr(stream)),
           "svdq_debug_partials")


class SVDQLinear:
    """One packed layer plus the buffers of its two hot-path calls.

    forward(X) runs svdq_quantize_act then svdq_linear on the current stream
    and returns Y (bf16 [M, N]).  Buffers are reallocated only when M grows.
    """

    def __init__(self, weights: Weights, epilogue: int = EPI_NONE):
        self.w = weights
        self.epilogue = epilogue
        self._M = -1
        self.xq = self.s_x = self.Z = self.Y = None

    def buffers(self, M: int, device="cuda"):
        import torch
        if M != self._M:
            K, N, r = self.w.K, self.w.N, self.w.rank
            self.xq = torch.empty((M, K // 2), dtype=torch.uint8, device=device)
            self.s_x = torch.empty((K // 64, M), dtype=torch.float32, device=device)
            self.Z = torch.empty((M, max(r, 1)), dtype=torch.bfloat16, device=device) if r else None
            self.Y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
            self._M = M
        return self.xq, self.s_x, self.Z, self.Y

    def forward(self, X, out=None):
        M = X.shape[0]
        xq, s_x, Z, Y = self.buffers(M, X.device)
        if out is not None:
            Y = out
        svdq_quantize_act(self.w, X, xq, s_x, Z)
        svdq_linear(self.w, xq, s_x, Z, Y, self.epilogue)
        return Y

    __call__ = forward


class W8A8Linear(SVDQLinear):
    """The W8A8 comparator layer: svdq_quantize_act_w8a8 then svdq_linear_w8a8."""

    def buffers(self, M: int, device="cuda"):
        import torch
        if M != self._M:
            K, N, r = self.w.K, self.w.N, self.w.rank
            self.xq = torch.empty((M, K), dtype=torch.int8, device=device)
            self.s_x = torch.empty((M,), dtype=torch.float32, device=device)
            self.Z = torch.empty((M, max(r, 1)), dtype=torch.bfloat16, device=device) if r else None
            self.Y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
            self._M = M
        return self.xq, self.s_x, self.Z, self.Y

    def forward(self, X, out=None):
        M = X.shape[0]
        xq, s_x, Z, Y = self.buffers(M, X.device)
        if out is not None:
            Y = out
        svdq_quantize_act_w8a8(self.w, X, xq, s_x, Z)
        svdq_linear_w8a8(self.w, xq, s_x, Z, Y, self.epilogue)
        return Y

    __call__ = forward


class NVFP4Linear(SVDQLinear):
    """The NVFP4 layer: svdq_quantize_act_nvfp4 then svdq_linear_nvfp4."""

    def buffers(self, M: int, device="cuda"):
        import torch
        if M != self._M:
            K, N, r = self.w.K, self.w.N, self.w.rank
            self.xq = torch.empty((M, K // 2), dtype=torch.uint8, device=device)
            self.sfa = torch.empty((svdq_nvfp4_sf_bytes(M, K),), dtype=torch.uint8, device=device)
            self.s_x = torch.empty((M,), dtype=torch.float32, device=device)
            self.Z = torch.empty((M, max(r, 1)), dtype=torch.bfloat16, device=device) if r else None
            self.Y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
            self._M = M
        return self.xq, self.sfa, self.s_x, self.Z, self.Y

    def forward(self, X, out=None):
        M = X.shape[0]
        xq, sfa, s_x, Z, Y = self.buffers(M, X.device)
        if out is not None:
            Y = out
        svdq_quantize_act_nvfp4(self.w, X, xq, sfa, s_x, Z)
        svdq_linear_nvfp4(self.w, xq, sfa, s_x, Z, Y, self.epilogue)
        return Y

    __call__ = forward


class SVDQMLP:
    """Two packed layers applied in sequence, fc2(GELU(fc1(X))), as in a
    transformer block's feed-forward part.

    forward(X) runs the four plain calls, storing the bf16 hidden activation
    H in between (the faster chain on B200).  forward(X, fused=True) runs
    svdq_quantize_act(fc1), then svdq_linear_quantize_next (fc1 with GELU,
    emitting fc2's codes, scales and Z), then svdq_linear(fc2): H never
    reaches device memory, and fc2's codes and scales are the same bits.
    Buffers are reallocated only when M changes.
    """

    def __init__(self, fc1: Weights, fc2: Weights):
        if fc2.K != fc1.N:
            raise ValueError("fc2's K must equal fc1's N")
        self.fc1 = SVDQLinear(fc1, EPI_GELU)
        self.fc2 = SVDQLinear(fc2)
        self._M = -1
        self.H = self.ws = None

    def buffers(self, M: int, device="cuda"):
        import torch
        self.fc1.buffers(M, device)
        self.fc2.buffers(M, device)
        if M != self._M:
            self.H = torch.empty((M, self.fc1.w.N), dtype=torch.bfloat16, device=device)
            n = svdq_linear_quantize_next_workspace(self.fc1.w, self.fc2.w, M)
            self.ws = torch.empty((n,), dtype=torch.uint8, device=device) if n else None
            self._M = M
        return self.H, self.ws

    def forward(self, X, fused: bool = False, out=None):
        M = X.shape[0]
        H, ws = self.buffers(M, X.device)
        a, b = self.fc1, self.fc2
        Y = b.Y if out is None else out
        svdq_quantize_act(a.w, X, a.xq, a.s_x, a.Z)
        if fused:
            svdq_linear_quantize_next(a.w, b.w, a.xq, a.s_x, a.Z, b.xq, b.s_x, b.Z, ws, EPI_GELU)
        else:
            svdq_linear(a.w, a.xq, a.s_x, a.Z, H, EPI_GELU)
            svdq_quantize_act(b.w, H, b.xq, b.s_x, b.Z)
        svdq_linear(b.w, b.xq, b.s_x, b.Z, Y)
        return Y

    __call__ = forward
