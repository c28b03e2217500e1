"""Host-only checks of the C ABI (no GPU needed): the library loads, exports
every function include/svdq.h declares, and rejects bad arguments with a
status code before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "svdq.h")


@pytest.fixture(scope="module")
def B():
    from rank_gemm_b200 import build
    build.build()
    from rank_gemm_b200 import binding
    return binding


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_]+\s*\*?\s*(svdq_[a-z0-9_]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary_calls():
    names = declared_functions()
    for required in ("svdq_prepare_weights", "svdq_quantize_act_lowrank_down", "svdq_w4a4_gemm_lowrank_up",
                     "svdq_linear"):
        assert required in names


def test_library_exports_every_declared_symbol(B):
    for name in declared_functions():
        assert hasattr(B.lib, name), name
        assert name in B.EXPORTED, name


def test_status_strings(B):
    for s in range(10):
        assert B.svdq_status_string(s)
    assert "10.0" in B.svdq_status_string(4)
    assert B.svdq_status_string(999) == "unknown status"


def test_argument_errors_before_device(B):
    L = B.lib
    # prepare: null output handle / null inputs / bad format -> invalid argument
    assert L.svdq_prepare_weights(0, 64, 16, 16, 16, 16, 16, 16, None, None, None, 0, 1.0, None, None) == 1
    h = ctypes.c_void_p()
    assert L.svdq_prepare_weights(0, 64, 16, 16, None, 16, 16, 16, None, None, None, 0, 1.0, None,
                                  ctypes.byref(h)) == 1
    assert L.svdq_prepare_weights(7, 64, 16, 16, 16, 16, 16, 16, None, None, None, 0, 1.0, None,
                                  ctypes.byref(h)) == 1
    # NVFP4 needs a positive finite activation scale
    assert L.svdq_prepare_weights(0, 64, 16, 16, 16, 16, 16, 16, None, None, None, 0, 0.0, None,
                                  ctypes.byref(h)) == 1
    # LoRA pointers and rank must agree
    assert L.svdq_prepare_weights(0, 64, 16, 16, 16, 16, 16, 16, None, 16, None, 16, 1.0, None,
                                  ctypes.byref(h)) == 1
    # shapes: K % 64, N % 16, rank, r_tot % 16, r_tot <= 256
    for K, N, r, lr in [(65, 16, 16, 0), (64, 17, 16, 0), (64, 16, 0, 0), (64, 16, 20, 0), (64, 16, 256, 16)]:
        args = (16, 16) if lr else (None, None)
        assert L.svdq_prepare_weights(0, K, N, r, 16, 16, 16, 16, None, args[0], args[1], lr, 1.0, None,
                                      ctypes.byref(h)) == 2, (K, N, r, lr)
    # alignment
    assert L.svdq_prepare_weights(0, 64, 16, 16, 18, 16, 16, 16, None, None, None, 0, 1.0, None,
                                  ctypes.byref(h)) == 3
    assert h.value is None
    # calls on a null handle
    assert L.svdq_linear(None, 4, 16, 0, 16, 16, 1 << 20, None) == 1
    assert L.svdq_weights_view(None, None) == 1
    assert L.svdq_free_weights(None) == 0
    # calibrate: alpha outside [0, 1], bad shape, misaligned, small workspace
    assert L.svdq_calibrate(4, 64, 16, 16, 16, ctypes.c_float(1.5), 16, 16, 16, 1 << 20, None) == 1
    assert L.svdq_calibrate(4, 60, 16, 16, 16, ctypes.c_float(0.5), 16, 16, 16, 1 << 20, None) == 2
    assert L.svdq_calibrate(4, 64, 16, 8, 16, ctypes.c_float(0.5), 16, 16, 16, 1 << 20, None) == 3
    assert L.svdq_calibrate(4, 64, 16, 16, 16, ctypes.c_float(0.5), 16, 16, 16, 8, None) == 5
    assert L.svdq_selftest_wait_timeout(0, None) == 1



def test_argument_errors_of_the_wider_calls(B):
    """The per-call-scale, cross-layer, W4A16 and device-split entries also
    reject bad arguments with a status before touching the device."""
    L = B.lib
    # per-call tensor scale: null handle
    assert L.svdq_linear_dynamic(None, 4, 16, 0, 32, 16, 1 << 20, None) == 1
    # cross-layer fusion: null handles; sizes of an invalid pair are 0
    assert L.svdq_linear_emit_next(None, None, 4, 16, 0, 32, 16, 16, 16, 1 << 20, None) == 1
    assert L.svdq_mlp(None, None, 4, 16, 0, 0, 32, 16, 1 << 20, None) == 1
    assert L.svdq_linear_emit_next_workspace_bytes(None, None, 64) == 0
    assert L.svdq_mlp_workspace_bytes(None, None, 64) == 0
    # AWQ W4A16: null output / weight, K % 64, alignment; null handle
    h = ctypes.c_void_p()
    assert L.svdq_awq_prepare(64, 16, 16, None, None, None, None) == 1
    assert L.svdq_awq_prepare(64, 16, None, None, None, None, ctypes.byref(h)) == 1
    assert L.svdq_awq_prepare(96, 16, 16, None, None, None, ctypes.byref(h)) == 2
    assert L.svdq_awq_prepare(64, 0, 16, None, None, None, ctypes.byref(h)) == 2
    assert L.svdq_awq_prepare(64, 16, 24, None, None, None, ctypes.byref(h)) == 3
    assert h.value is None
    assert L.svdq_awq_linear(None, 1, 16, 16, None) == 1
    # device split: null pointers, rank outside [1, min(K, N)], alignment
    assert L.svdq_lowrank_factors(64, 32, 8, None, 16, 5, 16, 16, None, None) == 1
    assert L.svdq_lowrank_factors(64, 32, 0, 16, 16, 5, 16, 16, None, None) == 2
    assert L.svdq_lowrank_factors(64, 32, 33, 16, 16, 5, 16, 16, None, None) == 2
    assert L.svdq_lowrank_factors(64, 32, 8, 16, 24, 5, 16, 16, None, None) == 3


def test_no_gpu_means_unsupported_device(B):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    h = ctypes.c_void_p()
    assert B.lib.svdq_prepare_weights(0, 64, 16, 16, 16, 16, 16, 16, None, None, None, 0, 1.0, None,
                                      ctypes.byref(h)) == 4
    assert B.lib.svdq_poll_device_error(None) == 4
    assert B.lib.svdq_calibrate(4, 64, 16, 16, 16, ctypes.c_float(0.5), 16, 16, 16, 1 << 20, None) == 4


def test_binding_refuses_host_and_strided_tensors(B):
    """Tensor arguments are device memory read as packed arrays: the binding
    refuses a host tensor before the call (a host address given to a kernel
    as device memory would fault), and passes None and integers through."""
    import torch
    assert B._ptr(None) is None and B._ptr(16) == 16
    with pytest.raises(ValueError, match="host memory"):
        B._ptr(torch.zeros(4))
    with pytest.raises(ValueError, match="host memory"):
        B.svdq_linear(None, 4, torch.zeros(4, 64, dtype=torch.bfloat16), 0,
                      torch.zeros(4, 16, dtype=torch.bfloat16), torch.zeros(1024, dtype=torch.uint8))
