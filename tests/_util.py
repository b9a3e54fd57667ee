"""Helpers shared by the tests (conversions, routing resolution).

The parity rule for float outputs lives in ``tests/_parity.py``; ``assert_close``
here is its plain form for outputs with no storage rounding to account for
(fp32 results, logits): max|got - ref| / RMS(ref) <= rel, nothing excused.
"""
import numpy as np
import torch

from ._parity import TOL_BF16, TOL_MXFP8  # noqa: F401


def np64(t) -> np.ndarray:
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    t = t.detach().cpu()
    if t.dtype in (torch.bfloat16, torch.float16):
        t = t.float()
    return t.double().numpy()


def npi(t) -> np.ndarray:
    return t.detach().cpu().numpy().astype(np.int64)


def rel_err(got, ref) -> float:
    """max|got - ref| / RMS(ref), nothing excused."""
    got = np64(got)
    ref = np64(ref)
    if ref.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(ref * ref)))
    err = float(np.max(np.abs(got - ref)))
    if rms == 0.0:
        return 0.0 if err == 0.0 else float("inf")
    return err / rms


def assert_close(got, ref, rel, what=""):
    e = rel_err(got, ref)
    print(f"parity {what}: strict {e:.3e} tol {rel:.0e} (max|err| / RMS)")
    assert e <= rel, f"{what}: max|err| / RMS(ref) = {e:.3e} > {rel:.1e}"


def bf16_cuda(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).cuda()


def resolve_routing(ref_logits64, gpu_idx, k, delta=1e-4):
    """Routing decided on logits that the device computes in fp32 and the
    oracle in fp64 (router projection).  A token is ambiguous when two of its
    k+1 largest oracle logits lie within `delta` (far above the fp32
    accumulation error): several selections are then correct.  Unambiguous
    tokens must match the oracle exactly; for ambiguous ones the device's
    selection is checked to be one of the correct ones and then adopted.
    Returns (idx, ambiguous mask)."""
    from oracle import moe as om
    lg64 = np.asarray(ref_logits64, np.float64)
    T, E = lg64.shape
    ridx, _ = om.router_topk(lg64.astype(np.float32), k)
    top = -np.sort(-lg64, axis=1)[:, :k + 1]
    amb = np.any(np.abs(np.diff(top, axis=1)) <= delta, axis=1) if top.shape[1] > 1 \
        else np.zeros(T, bool)
    assert amb.mean() < 1e-2, f"{amb.sum()} ambiguous tokens"
    g = np.asarray(gpu_idx, np.int64)
    assert np.array_equal(g[~amb], ridx[~amb])
    for t in np.nonzero(amb)[0]:
        sel = g[t]
        lt = lg64[t]
        assert len(set(sel.tolist())) == k and np.all((sel >= 0) & (sel < E))
        assert np.all(np.diff(lt[sel]) <= delta)                     # descending within delta
        rest = np.setdiff1d(np.arange(E), sel)
        assert rest.size == 0 or lt[rest].max() <= lt[sel].min() + delta
    res = ridx.astype(np.int64)
    res[amb] = g[amb]
    return res.astype(np.int32), amb
