"""svdq_linear_noalloc: the layer for callers that cannot allocate device
memory while they run it (the intermediates live in a scratch array inside
the library).  Its output must match svdq_linear's, which gets a caller
workspace, on two calls in a row, and oversized requests must be refused
before anything runs.  This file is named to be collected last."""
import numpy as np
import pytest
import torch

import workloads
from svdq_harness import GpuLayer, assert_y, bf16_np, dev_bf16

pytestmark = pytest.mark.gpu


def test_linear_noalloc_matches_linear_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from rank_gemm_b200 import binding as B
    L = workloads.draw_layer("noalloc", "nvfp4", 300, 1024, 768, 32, seed=61, n_out=4)
    g = GpuLayer(L.fmt, L.X, L.W, L.bias, L.rank)
    try:
        Xd = dev_bf16(L.X)
        ref = bf16_np(g.linear(Xd, L.M))
        for _ in range(2):
            Y = torch.full((L.M, L.N), float("nan"), dtype=torch.bfloat16, device="cuda")
            B.svdq_linear_noalloc(g.h, L.M, Xd, B.SVDQ_EPI_NONE, Y)
            torch.cuda.synchronize()
            assert_y(bf16_np(Y), ref)
        assert B.svdq_poll_device_error() == 0
        # a request larger than the scratch array is refused up front
        M_big = B.SVDQ_NOALLOC_SCRATCH_BYTES // (L.K // 2) + 1
        assert B.svdq_linear_workspace_bytes(g.h, M_big) > B.SVDQ_NOALLOC_SCRATCH_BYTES
        with pytest.raises(B.SvdqError) as e:
            B.svdq_linear_noalloc(g.h, M_big, Xd, B.SVDQ_EPI_NONE, Y)
        assert e.value.status == 5
    finally:
        g.close()
