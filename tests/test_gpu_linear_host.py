"""svdq_linear_host: the layer from host X to host Y with the copies
overlapped with the kernels (slabs of rows on two copy streams).  Each row of
Y depends on its row of X only, so the result must be bit-identical to
svdq_linear on the whole batch in device memory; checked for NVFP4 and INT4,
with and without GELU, with one slab, with several and a ragged last one."""
import numpy as np
import pytest
import torch

import workloads
from svdq_harness import GpuLayer, dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from rank_gemm_b200 import binding
    return binding


@pytest.mark.parametrize("fmt,M,gelu", [("nvfp4", 1000, False), ("nvfp4", 100, True), ("int4", 777, True)])
def test_linear_host_matches_linear(B, fmt, M, gelu):
    L = workloads.draw_layer("host", fmt, M, 512, 384, 32, seed=90 + M, n_out=4)
    g = GpuLayer(L.fmt, L.X, L.W, L.bias, L.rank)
    try:
        epi = B.SVDQ_EPI_GELU_TANH if gelu else B.SVDQ_EPI_NONE
        Xd = dev_bf16(L.X)
        ref = g.linear(Xd, M, gelu=gelu).cpu()
        Xh = Xd.cpu().pin_memory()
        ws = torch.empty(B.svdq_linear_host_workspace_bytes(g.h, M), dtype=torch.uint8, device="cuda")
        for _ in range(2):
            Yh = torch.full((M, L.N), float("nan"), dtype=torch.bfloat16).pin_memory()
            B.svdq_linear_host(g.h, M, Xh, epi, Yh, ws)
            torch.cuda.synchronize()
            assert torch.equal(Yh, ref)
        assert B.svdq_poll_device_error() == 0
    finally:
        g.close()


def test_linear_host_orders_on_the_callers_stream_and_checks_its_workspace(B):
    L = workloads.draw_layer("host_order", "nvfp4", 640, 256, 256, 16, seed=99, n_out=4)
    g = GpuLayer(L.fmt, L.X, L.W, L.bias, L.rank)
    try:
        M = L.M
        Xh = dev_bf16(L.X).cpu().pin_memory()
        Yh = torch.zeros(M, L.N, dtype=torch.bfloat16).pin_memory()
        ws = torch.empty(B.svdq_linear_host_workspace_bytes(g.h, M), dtype=torch.uint8, device="cuda")
        s = torch.cuda.Stream()
        with torch.cuda.stream(s):
            B.svdq_linear_host(g.h, M, Xh, B.SVDQ_EPI_NONE, Yh, ws, stream=s)
            done = torch.cuda.Event()
            done.record(s)
        done.synchronize()            # the caller's stream covers the last copy to the host
        ref = g.linear(dev_bf16(L.X), M).cpu()
        assert torch.equal(Yh, ref)
        with pytest.raises(B.SvdqError) as e:
            B.svdq_linear_host(g.h, M, Xh, B.SVDQ_EPI_NONE, Yh, ws[:1024], 1024)
        assert e.value.status == 5
        B.svdq_linear_host(g.h, 0, Xh, B.SVDQ_EPI_NONE, Yh, ws)   # M = 0: nothing to do
    finally:
        g.close()
