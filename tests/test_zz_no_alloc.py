"""The allocation-free dispatch entry point (moe_permute_rows_noalloc) against
the workspace-taking one (moe_permute_rows), through the C ABI, on two calls in
a row (needs a B200).

The variant exists for callers that cannot allocate device memory when they
call the library (a plugin inside a host that owns all device memory, a
runtime that forbids cudaMalloc after start-up).  Its scratch is a fixed array
inside the library shared by all calls, so the second call also checks that
nothing left over from the first call leaks into its results.  This file is
collected last so that a run stopping at the first failure has already run
every other test.
"""
import pytest
import torch

from routing_grouped_gemm_moe_b200 import inputs as I
from routing_grouped_gemm_moe_b200 import ops

pytestmark = pytest.mark.gpu


def _case(T, d, E, k, seed):
    lg = I.normal_f32(I.stream_key(seed, 1), (T, E)).cuda()
    idx, _ = ops.router_topk(lg, k)
    x = I.normal_bf16(I.stream_key(seed, 2), (T, d), 1.0).cuda()
    return x, idx


def _same(a, b):
    names = ("counts", "offsets", "dest_pos", "src_token", "x_perm")
    for n, u, v in zip(names, a, b):
        assert torch.equal(u.view(torch.uint8), v.view(torch.uint8)), n


def test_noalloc_matches_workspace_dispatch_on_two_calls():
    # first call: a larger problem; second call: a smaller one with more
    # experts, so stale scratch from the first call would show up
    for (T, d, E, k, seed) in [(3000, 256, 64, 8, 11), (700, 136, 96, 4, 12)]:
        x, idx = _case(T, d, E, k, seed)
        ref = ops.permute_rows(x, idx, E)[:5]
        got = ops.permute_rows_noalloc(x, idx, E)
        torch.cuda.synchronize()
        _same(got, ref)
        assert int(got[0].sum().item()) == T * k


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from routing_grouped_gemm_moe_b200 import _lib as L
    T, d, E, k = 128 * 300, 8, 1024, 1          # 300 tasks x 1024 experts > 262144
    x = torch.zeros(T, d, dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros(T, k, dtype=torch.int32, device="cuda")
    with pytest.raises(L.MoeError) as e:
        ops.permute_rows_noalloc(x, idx, E)
    assert e.value.status == 1


def test_noalloc_skips_out_of_range_experts():
    """An expert index outside [0, E) is skipped (dest_pos = -1) and left out
    of the counts; every valid pick is still dispatched exactly as the
    workspace dispatch does it."""
    T, d, E, k = 257, 64, 12, 3
    x, idx = _case(T, d, E, k, 13)
    bad = idx.clone()
    bad[5, 1] = E
    bad[100, 0] = -1
    bad[256, 2] = E + 7
    got = ops.permute_rows_noalloc(x, bad, E)
    ref = ops.permute_rows(x, bad, E)[:5]
    torch.cuda.synchronize()
    dest = got[2].cpu()
    assert dest[5, 1] == -1 and dest[100, 0] == -1 and dest[256, 2] == -1
    assert int(got[0].sum().item()) == T * k - 3
    for n, u, v in zip(("counts", "offsets", "dest_pos"), got[:3], ref[:3]):
        assert torch.equal(u, v), n
    valid = int(got[1][-1].item())
    assert torch.equal(got[3][:valid], ref[3][:valid])
    assert torch.equal(got[4][:valid].view(torch.int16), ref[4][:valid].view(torch.int16))


def test_noalloc_with_no_tokens():
    """T = 0: counts and offsets are all zero and nothing else is touched."""
    E, d, k = 16, 64, 2
    x = torch.empty(0, d, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(0, k, dtype=torch.int32, device="cuda")
    counts, offsets, _, _, _ = ops.permute_rows_noalloc(x, idx, E)
    torch.cuda.synchronize()
    assert torch.all(counts == 0) and torch.all(offsets == 0)
    assert counts.numel() == E and offsets.numel() == E + 1
