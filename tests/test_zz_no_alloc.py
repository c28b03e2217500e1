"""svdq_linear_noalloc: the layer for callers that cannot allocate device
memory while they run it (a latency-critical loop where cudaMalloc's device
synchronisation is not affordable, or a plug-in inside an application that
owns all device memory and hands out no allocator).  The intermediates live
in a scratch array inside the library, so the call runs the very kernels
svdq_linear runs and its output must be bit-identical to svdq_linear's with a
caller workspace: on two calls in a row, for both formats and both
epilogues, at the largest M the array holds and at a smaller M right after
it.  Requests larger than the array are refused before anything runs.  This
file is named to be collected last."""
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


def _pair(B, g, Xd, M, epi):
    """(svdq_linear's Y, svdq_linear_noalloc's Y) for the first M rows of Xd."""
    ref = torch.empty(M, g.N, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(B.svdq_linear_workspace_bytes(g.h, M), dtype=torch.uint8, device="cuda")
    B.svdq_linear(g.h, M, Xd, epi, ref, ws)
    Y = torch.full((M, g.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    B.svdq_linear_noalloc(g.h, M, Xd, epi, Y)
    torch.cuda.synchronize()
    return ref, Y


def _max_rows(B, h):
    """The largest M whose workspace fits the scratch array (the workspace
    size grows with M)."""
    lo, hi = 1, 1 << 20
    while lo < hi:
        mid = (lo + hi + 1) // 2
        if B.svdq_linear_workspace_bytes(h, mid) <= B.SVDQ_NOALLOC_SCRATCH_BYTES:
            lo = mid
        else:
            hi = mid - 1
    return lo


@pytest.mark.parametrize("fmt", ["nvfp4", "int4"])
@pytest.mark.parametrize("gelu", [False, True])
def test_linear_noalloc_matches_linear_on_two_calls(B, fmt, gelu):
    L = workloads.draw_layer("noalloc", fmt, 300, 1024, 768, 32, seed=61, n_out=4)
    g = GpuLayer(L.fmt, L.X, L.W, L.bias, L.rank)
    try:
        Xd = dev_bf16(L.X)
        epi = B.SVDQ_EPI_GELU_TANH if gelu else B.SVDQ_EPI_NONE
        for _ in range(2):
            ref, Y = _pair(B, g, Xd, L.M, epi)
            assert torch.equal(Y, ref)
        assert B.svdq_poll_device_error() == 0
    finally:
        g.close()


def test_linear_noalloc_takes_no_device_memory(B):
    """After a first call (which may load the library's module and with it
    the scratch array), a call changes neither the device's free memory nor
    the caching allocator's count: nothing is allocated behind the caller."""
    L = workloads.draw_layer("noalloc_mem", "nvfp4", 300, 1024, 768, 32, seed=65, n_out=4)
    g = GpuLayer(L.fmt, L.X, L.W, L.bias, L.rank)
    try:
        Xd = dev_bf16(L.X)
        Y = torch.empty(L.M, L.N, dtype=torch.bfloat16, device="cuda")
        B.svdq_linear_noalloc(g.h, L.M, Xd, B.SVDQ_EPI_NONE, Y)
        torch.cuda.synchronize()
        free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
        for _ in range(3):
            B.svdq_linear_noalloc(g.h, L.M, Xd, B.SVDQ_EPI_NONE, Y)
        torch.cuda.synchronize()
        assert torch.cuda.mem_get_info()[0] == free0
        assert torch.cuda.memory_allocated() == alloc0
        assert B.svdq_poll_device_error() == 0
    finally:
        g.close()


def test_linear_noalloc_at_the_size_limit_then_smaller(B):
    """The largest M the array takes, then a smaller M: the second call reads
    nothing the first one left behind."""
    L = workloads.draw_layer("noalloc_big", "nvfp4", 128, 1024, 256, 32, seed=62, n_out=4)
    g = GpuLayer(L.fmt, L.X, L.W, L.bias, L.rank)
    try:
        M_max = _max_rows(B, g.h)
        assert B.svdq_linear_workspace_bytes(g.h, M_max) <= B.SVDQ_NOALLOC_SCRATCH_BYTES
        assert B.svdq_linear_workspace_bytes(g.h, M_max + 1) > B.SVDQ_NOALLOC_SCRATCH_BYTES
        gen = torch.Generator(device="cpu").manual_seed(63)
        Xd = (torch.randn(M_max, L.K, generator=gen) * 2).to(torch.bfloat16).cuda()
        for M in (M_max, 1000):
            ref, Y = _pair(B, g, Xd, M, B.SVDQ_EPI_NONE)
            assert torch.equal(Y, ref), M
        assert B.svdq_poll_device_error() == 0
        # a request one row over the limit is refused before any launch; X and
        # Y are sized for it, so even a launch would stay in bounds
        Xb = torch.zeros(M_max + 1, L.K, dtype=torch.bfloat16, device="cuda")
        Yb = torch.zeros(M_max + 1, L.N, dtype=torch.bfloat16, device="cuda")
        with pytest.raises(B.SvdqError) as e:
            B.svdq_linear_noalloc(g.h, M_max + 1, Xb, B.SVDQ_EPI_NONE, Yb)
        assert e.value.status == 5
        torch.cuda.synchronize()
        assert not torch.any(Yb != 0)
    finally:
        g.close()


@pytest.mark.parametrize("fmt,K,rows", [("nvfp4", 3072, 13784), ("nvfp4", 12288, 3584),
                                        ("int4", 3072, 9886), ("int4", 12288, 2544)])
def test_documented_row_limits(B, fmt, K, rows):
    """The limits include/svdq.h states (rank 32, so r_pad = 64) are the
    library's: that many rows fit the array, one more does not."""
    L = workloads.draw_layer("noalloc_lim", fmt, 64, K, 256, 32, seed=64, n_out=4)
    g = GpuLayer(L.fmt, L.X, L.W, L.bias, L.rank)
    try:
        assert B.svdq_linear_workspace_bytes(g.h, rows) <= B.SVDQ_NOALLOC_SCRATCH_BYTES
        assert B.svdq_linear_workspace_bytes(g.h, rows + 1) > B.SVDQ_NOALLOC_SCRATCH_BYTES
    finally:
        g.close()
