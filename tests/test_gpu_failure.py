"""Device-side failure detection, exercised without faulting a GPU (needs a B200).

Every pipeline wait in the grouped GEMM is bounded in global time.  The
diagnostic entry point runs that wait on a barrier nothing arrives on: it must
give up after the requested limit, record MOE_ERR_DEVICE_TIMEOUT in the status
word, and leave the CUDA context usable.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from routing_grouped_gemm_moe_b200 import _lib as L
from routing_grouped_gemm_moe_b200 import ops

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    elapsed = torch.zeros(1, dtype=torch.int64, device="cuda")
    limit = 50_000_000  # 50 ms
    L.call("moe_selftest_bounded_wait", ops._p(status), limit, ops._p(elapsed), ops._s())
    torch.cuda.synchronize()
    assert int(status.item()) == 1 << 4          # MOE_ERR_DEVICE_TIMEOUT
    waited = int(elapsed.item())
    assert limit <= waited < limit + 200_000_000
    # the context is still usable: a real kernel runs and is right
    lg = torch.randn(64, 8, device="cuda")
    idx, w = ops.router_topk(lg, 2)
    ref = torch.topk(lg, 2, dim=1).indices.to(torch.int32)
    assert torch.equal(idx, ref)


def test_status_read_back_and_clear():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.call("moe_selftest_bounded_wait", ops._p(status), 1_000_000, None, ops._s())
    out = C.c_int32(0)
    L.call("moe_read_device_status", ops._p(status), 1, C.byref(out), ops._s())
    assert out.value == 1 << 4
    assert int(status.item()) == 0                # cleared


def test_selftest_rejects_bad_limits():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(L.MoeError):
        L.call("moe_selftest_bounded_wait", ops._p(status), 10, None, ops._s())
