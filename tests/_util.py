"""Helpers shared by the tests (conversions and the tolerance rule).

Tolerance rule for float outputs: max|gpu - oracle| <= REL * RMS(oracle), with
REL = 2e-2 (BF16 path) or 6e-2 (MXFP8 path).  When the GPU stores a tensor in
bf16, the storage rounding itself is not counted: each element may differ from
the oracle by one bf16 spacing at that value (the two sides round values that
differ in the last fp32 bits, or the oracle value is unrounded) before the
remainder is charged to the budget.  Without this, a single half-unit rounding
at the largest element of a heavy-tailed tensor (an outer product, silu(g) u)
already exceeds 2e-2 RMS.
"""
import numpy as np
import torch

TOL_BF16 = 2e-2
TOL_MXFP8 = 6e-2


def np64(t) -> np.ndarray:
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    t = t.detach().cpu()
    if t.dtype in (torch.bfloat16, torch.float16):
        t = t.float()
    return t.double().numpy()


def npi(t) -> np.ndarray:
    return t.detach().cpu().numpy().astype(np.int64)


def bf16_spacing(ref: np.ndarray) -> np.ndarray:
    """Distance between adjacent bf16 numbers around |ref|."""
    _, e = np.frexp(np.abs(ref))
    return np.ldexp(1.0, np.maximum(e, -125) - 8)


def rel_err(got, ref, bf16_storage=None) -> float:
    is_bf16 = isinstance(got, torch.Tensor) and got.dtype == torch.bfloat16
    if bf16_storage is None:
        bf16_storage = is_bf16
    got = np64(got)
    ref = np64(ref)
    if ref.size == 0:
        return 0.0
    diff = np.abs(got - ref)
    if bf16_storage:
        diff = np.maximum(diff - bf16_spacing(ref), 0.0)
    rms = float(np.sqrt(np.mean(ref * ref)))
    err = float(np.max(diff))
    if rms == 0.0:
        return 0.0 if err == 0.0 else float("inf")
    return err / rms


def assert_close(got, ref, rel=TOL_BF16, what="", bf16_storage=None):
    e = rel_err(got, ref, bf16_storage)
    assert e <= rel, f"{what}: max|err| / RMS(ref) = {e:.3e} > {rel:.1e}"


def bf16_cuda(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).cuda()
