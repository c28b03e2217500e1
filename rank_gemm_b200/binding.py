"""ctypes binding of libsvdq.so (include/svdq.h): argument marshalling only.

Each function has the C entry point's name and argument order.  Device
buffers are passed as torch CUDA tensors (their data pointers are handed to
the library), the stream defaults to torch's current stream, and a non-OK
status raises SvdqError.  No arithmetic of the layer happens here: every step
runs in the library's CUDA kernels.  If the library is missing this module
raises at import time; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsvdq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        "libsvdq.so is not built (expected at %s); run `python -m rank_gemm_b200.build` "
        "(needs nvcc); there is no CPU fallback" % LIB_PATH)

lib = ctypes.CDLL(LIB_PATH)

SVDQ_NVFP4, SVDQ_INT4 = 0, 1
SVDQ_EPI_NONE, SVDQ_EPI_GELU_TANH = 0, 1
STATUS = {0: "SVDQ_OK", 1: "SVDQ_ERR_INVALID_ARG", 2: "SVDQ_ERR_SHAPE", 3: "SVDQ_ERR_ALIGNMENT",
          4: "SVDQ_ERR_UNSUPPORTED_DEVICE", 5: "SVDQ_ERR_WORKSPACE", 6: "SVDQ_ERR_CUDA",
          7: "SVDQ_ERR_TIMEOUT", 8: "SVDQ_ERR_DEVICE_FAULT", 9: "SVDQ_ERR_NO_MEMORY"}
FORMATS = {"nvfp4": SVDQ_NVFP4, "int4": SVDQ_INT4}


class SvdqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib.svdq_status_string(status).decode()
        super().__init__("%s: %s (%s)" % (where, STATUS.get(status, status), msg))


class WeightsInfo(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int), ("K", ctypes.c_int), ("N", ctypes.c_int), ("rank", ctypes.c_int),
                ("lora_rank", ctypes.c_int), ("r_tot", ctypes.c_int), ("K_pad", ctypes.c_int),
                ("N_pad", ctypes.c_int), ("r_pad", ctypes.c_int), ("qR", ctypes.c_void_p),
                ("sR", ctypes.c_void_p), ("L1t", ctypes.c_void_p), ("L2a", ctypes.c_void_p),
                ("bias", ctypes.c_void_p), ("lambda_inv", ctypes.c_void_p), ("s_tR", ctypes.c_float),
                ("s_tX", ctypes.c_float), ("alpha", ctypes.c_float)]


class AwqInfo(ctypes.Structure):
    _fields_ = [("K", ctypes.c_int), ("N", ctypes.c_int), ("N_pad", ctypes.c_int), ("code", ctypes.c_void_p),
                ("scale", ctypes.c_void_p), ("zero", ctypes.c_void_p), ("inv_s", ctypes.c_void_p),
                ("bias", ctypes.c_void_p)]


_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_SIGS = {
    "svdq_status_string": (ctypes.c_char_p, [_i]),
    "svdq_calibrate_workspace_bytes": (_sz, [_i]),
    "svdq_calibrate": (_i, [_i, _i, _i, _vp, _vp, _f, _vp, _vp, _vp, _sz, _vp]),
    "svdq_prepare_weights": (_i, [_i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _f, _vp,
                                  ctypes.POINTER(_vp)]),
    "svdq_free_weights": (_i, [_vp]),
    "svdq_lowrank_factors": (_i, [_i, _i, _i, _vp, _vp, ctypes.c_ulonglong, _vp, _vp, _vp, _vp]),
    "svdq_weights_view": (_i, [_vp, ctypes.POINTER(WeightsInfo)]),
    "svdq_act_buffer_sizes": (_i, [_vp, _i, ctypes.POINTER(_sz), ctypes.POINTER(_sz), ctypes.POINTER(_sz)]),
    "svdq_quantize_act_lowrank_down": (_i, [_vp, _i, _vp, _vp, _vp, _vp, _vp]),
    "svdq_w4a4_gemm_lowrank_up": (_i, [_vp, _i, _vp, _vp, _vp, _i, _vp, _vp]),
    "svdq_linear_workspace_bytes": (_sz, [_vp, _i]),
    "svdq_linear": (_i, [_vp, _i, _vp, _i, _vp, _vp, _sz, _vp]),
    "svdq_linear_dynamic_workspace_bytes": (_sz, [_vp, _i]),
    "svdq_linear_dynamic": (_i, [_vp, _i, _vp, _i, _vp, _vp, _sz, _vp]),
    "svdq_linear_emit_next_workspace_bytes": (_sz, [_vp, _vp, _i]),
    "svdq_linear_emit_next": (_i, [_vp, _vp, _i, _vp, _i, _vp, _vp, _vp, _vp, _sz, _vp]),
    "svdq_mlp_workspace_bytes": (_sz, [_vp, _vp, _i]),
    "svdq_mlp": (_i, [_vp, _vp, _i, _vp, _i, _i, _vp, _vp, _sz, _vp]),
    "svdq_quantize_act": (_i, [_vp, _i, _vp, _vp, _vp, _vp]),
    "svdq_lowrank_down": (_i, [_vp, _i, _vp, _vp, _vp]),
    "svdq_w4a4_gemm": (_i, [_vp, _i, _vp, _vp, _vp, _vp]),
    "svdq_lowrank_up": (_i, [_vp, _i, _vp, _i, _vp, _vp]),
    "svdq_linear_unfused": (_i, [_vp, _i, _vp, _i, _vp, _vp, _sz, _vp]),
    "svdq_linear_noalloc": (_i, [_vp, _i, _vp, _i, _vp, _vp]),
    "svdq_awq_prepare": (_i, [_i, _i, _vp, _vp, _vp, _vp, ctypes.POINTER(_vp)]),
    "svdq_awq_free": (_i, [_vp]),
    "svdq_awq_view": (_i, [_vp, ctypes.POINTER(AwqInfo)]),
    "svdq_awq_linear": (_i, [_vp, _i, _vp, _vp, _vp]),
    "svdq_awq_gemm": (_i, [_vp, _i, _vp, _vp, _vp]),
    "svdq_linear_host_workspace_bytes": (ctypes.c_size_t, [_vp, _i]),
    "svdq_linear_host": (_i, [_vp, _i, _vp, _i, _vp, _vp, ctypes.c_size_t, _vp]),
    "svdq_poll_device_error": (_i, [_vp]),
    "svdq_selftest_wait_timeout": (_i, [ctypes.c_uint, _vp]),
    "svdq_debug_override_cc": (None, [_i, _i]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTED = tuple(_SIGS)


def _ptr(t) -> Optional[int]:
    """Device address of a tensor argument (every tensor the ABI takes is
    device memory read as a packed array): a host tensor or a strided view
    is refused here, before the call, instead of being read as raw memory."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if isinstance(t, torch.Tensor):
        if not t.is_cuda:
            raise ValueError("svdq: a tensor argument is in host memory; the library takes device memory")
        if not t.is_contiguous():
            raise ValueError("svdq: a tensor argument is not contiguous; the library reads packed arrays")
    return t.data_ptr()


def _stream(s) -> Optional[int]:
    if s is None:
        return torch.cuda.current_stream().cuda_stream
    return s.cuda_stream if hasattr(s, "cuda_stream") else int(s)


def _check(status: int, where: str):
    if status != 0:
        raise SvdqError(status, where)


# ------------------------------------------------------------------ entry points
def svdq_status_string(status: int) -> str:
    return lib.svdq_status_string(status).decode()


def svdq_calibrate_workspace_bytes(K: int) -> int:
    return lib.svdq_calibrate_workspace_bytes(K)


def svdq_calibrate(M, K, N, X, W_t, alpha, lambda_out, act_scale_out, workspace, ws_bytes=None, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    _check(lib.svdq_calibrate(M, K, N, _ptr(X), _ptr(W_t), alpha, _ptr(lambda_out), _ptr(act_scale_out),
                              _ptr(workspace), ws_bytes, _stream(stream)), "svdq_calibrate")


def svdq_prepare_weights(fmt, K, N, rank, W_t, lam, L1f, L2, bias=None, lora_A=None, lora_B=None,
                         lora_rank=0, act_scale=1.0, stream=None) -> int:
    """Returns the opaque handle (an int); release it with svdq_free_weights."""
    h = _vp()
    fmt = FORMATS.get(fmt, fmt)
    _check(lib.svdq_prepare_weights(fmt, K, N, rank, _ptr(W_t), _ptr(lam), _ptr(L1f), _ptr(L2), _ptr(bias),
                                    _ptr(lora_A), _ptr(lora_B), lora_rank, float(act_scale), _stream(stream),
                                    ctypes.byref(h)), "svdq_prepare_weights")
    return h.value


SVDQ_SPLIT_SEED = 0x5EED


def svdq_lowrank_factors(K, N, rank, W_t, lam, L1f, L2, seed=SVDQ_SPLIT_SEED, stream=None):
    """The device's randomized split of diag(lam) W; fills L1f / L2 and returns
    the estimated singular values (a list of min(rank + 8, K, N) floats)."""
    n_sig = min(rank + 8, K, N)
    sig = (ctypes.c_double * n_sig)()
    _check(lib.svdq_lowrank_factors(K, N, rank, _ptr(W_t), _ptr(lam), seed, _ptr(L1f), _ptr(L2), sig,
                                    _stream(stream)), "svdq_lowrank_factors")
    return list(sig)


def svdq_free_weights(w):
    _check(lib.svdq_free_weights(w), "svdq_free_weights")


def svdq_weights_view(w) -> WeightsInfo:
    info = WeightsInfo()
    _check(lib.svdq_weights_view(w, ctypes.byref(info)), "svdq_weights_view")
    return info


def svdq_act_buffer_sizes(w, M):
    q, s, l = _sz(), _sz(), _sz()
    _check(lib.svdq_act_buffer_sizes(w, M, ctypes.byref(q), ctypes.byref(s), ctypes.byref(l)),
           "svdq_act_buffer_sizes")
    return q.value, s.value, l.value


def svdq_quantize_act_lowrank_down(w, M, X, qX, sX, LR, stream=None):
    _check(lib.svdq_quantize_act_lowrank_down(w, M, _ptr(X), _ptr(qX), _ptr(sX), _ptr(LR), _stream(stream)),
           "svdq_quantize_act_lowrank_down")


def svdq_w4a4_gemm_lowrank_up(w, M, qX, sX, LR, epi, Y, stream=None):
    _check(lib.svdq_w4a4_gemm_lowrank_up(w, M, _ptr(qX), _ptr(sX), _ptr(LR), epi, _ptr(Y), _stream(stream)),
           "svdq_w4a4_gemm_lowrank_up")


def svdq_linear_workspace_bytes(w, M) -> int:
    return lib.svdq_linear_workspace_bytes(w, M)


def svdq_linear(w, M, X, epi, Y, workspace, ws_bytes=None, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    _check(lib.svdq_linear(w, M, _ptr(X), epi, _ptr(Y), _ptr(workspace), ws_bytes, _stream(stream)),
           "svdq_linear")


def _host_ptr(t) -> Optional[int]:
    """Address of a host tensor argument (svdq_linear_host's X and Y)."""
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        if t.is_cuda:
            raise ValueError("svdq: this argument is host memory; a device tensor was given")
        if not t.is_contiguous():
            raise ValueError("svdq: a tensor argument is not contiguous; the library reads packed arrays")
    return t.data_ptr()


def svdq_linear_host_workspace_bytes(w, M) -> int:
    return lib.svdq_linear_host_workspace_bytes(w, M)


def svdq_linear_host(w, M, X_host, epi, Y_host, workspace, ws_bytes=None, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    _check(lib.svdq_linear_host(w, M, _host_ptr(X_host), epi, _host_ptr(Y_host), _ptr(workspace), ws_bytes,
                                _stream(stream)), "svdq_linear_host")


def svdq_linear_dynamic_workspace_bytes(w, M) -> int:
    return lib.svdq_linear_dynamic_workspace_bytes(w, M)


def svdq_linear_dynamic(w, M, X, epi, Y, workspace, ws_bytes=None, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    _check(lib.svdq_linear_dynamic(w, M, _ptr(X), epi, _ptr(Y), _ptr(workspace), ws_bytes, _stream(stream)),
           "svdq_linear_dynamic")


def svdq_linear_emit_next_workspace_bytes(w1, w2, M) -> int:
    return lib.svdq_linear_emit_next_workspace_bytes(w1, w2, M)


def svdq_linear_emit_next(w1, w2, M, X, epi, qX2, sX2, LR2, workspace, ws_bytes=None, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    _check(lib.svdq_linear_emit_next(w1, w2, M, _ptr(X), epi, _ptr(qX2), _ptr(sX2), _ptr(LR2), _ptr(workspace),
                                     ws_bytes, _stream(stream)), "svdq_linear_emit_next")


def svdq_mlp_workspace_bytes(w1, w2, M) -> int:
    return lib.svdq_mlp_workspace_bytes(w1, w2, M)


def svdq_mlp(w1, w2, M, X, epi1, epi2, Y, workspace, ws_bytes=None, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    _check(lib.svdq_mlp(w1, w2, M, _ptr(X), epi1, epi2, _ptr(Y), _ptr(workspace), ws_bytes, _stream(stream)),
           "svdq_mlp")


def svdq_quantize_act(w, M, X, qX, sX, stream=None):
    _check(lib.svdq_quantize_act(w, M, _ptr(X), _ptr(qX), _ptr(sX), _stream(stream)), "svdq_quantize_act")


def svdq_lowrank_down(w, M, X, LR, stream=None):
    _check(lib.svdq_lowrank_down(w, M, _ptr(X), _ptr(LR), _stream(stream)), "svdq_lowrank_down")


def svdq_w4a4_gemm(w, M, qX, sX, Y, stream=None):
    _check(lib.svdq_w4a4_gemm(w, M, _ptr(qX), _ptr(sX), _ptr(Y), _stream(stream)), "svdq_w4a4_gemm")


def svdq_lowrank_up(w, M, LR, epi, Y, stream=None):
    _check(lib.svdq_lowrank_up(w, M, _ptr(LR), epi, _ptr(Y), _stream(stream)), "svdq_lowrank_up")


def svdq_linear_unfused(w, M, X, epi, Y, workspace, ws_bytes=None, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    _check(lib.svdq_linear_unfused(w, M, _ptr(X), epi, _ptr(Y), _ptr(workspace), ws_bytes, _stream(stream)),
           "svdq_linear_unfused")


def svdq_linear_noalloc(w, M, X, epi, Y, stream=None):
    """svdq_linear with the intermediates in the library's own scratch array
    (no workspace, no allocation); see include/svdq.h for its size limit and
    the rule that calls overlapping on the GPU race."""
    _check(lib.svdq_linear_noalloc(w, M, _ptr(X), epi, _ptr(Y), _stream(stream)), "svdq_linear_noalloc")


SVDQ_NOALLOC_SCRATCH_BYTES = 32 << 20


def svdq_awq_prepare(K, N, W_t, s=None, bias=None, stream=None) -> int:
    """Returns the opaque AWQ W4A16 handle (an int); release it with svdq_awq_free."""
    h = _vp()
    _check(lib.svdq_awq_prepare(K, N, _ptr(W_t), _ptr(s), _ptr(bias), _stream(stream), ctypes.byref(h)),
           "svdq_awq_prepare")
    return h.value


def svdq_awq_free(w):
    _check(lib.svdq_awq_free(w), "svdq_awq_free")


def svdq_awq_view(w) -> AwqInfo:
    info = AwqInfo()
    _check(lib.svdq_awq_view(w, ctypes.byref(info)), "svdq_awq_view")
    return info


def svdq_awq_linear(w, M, X, Y, stream=None):
    _check(lib.svdq_awq_linear(w, M, _ptr(X), _ptr(Y), _stream(stream)), "svdq_awq_linear")


def svdq_awq_gemm(w, M, X, Y, stream=None):
    _check(lib.svdq_awq_gemm(w, M, _ptr(X), _ptr(Y), _stream(stream)), "svdq_awq_gemm")


def svdq_poll_device_error(stream=None) -> int:
    """Returns the status code (does not raise): 0, SVDQ_ERR_TIMEOUT, ..."""
    return lib.svdq_poll_device_error(_stream(stream))


def svdq_selftest_wait_timeout(limit_us, stream=None):
    _check(lib.svdq_selftest_wait_timeout(limit_us, _stream(stream)), "svdq_selftest_wait_timeout")


def svdq_debug_override_cc(major, minor):
    lib.svdq_debug_override_cc(major, minor)
