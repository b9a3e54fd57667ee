"""Helpers shared by the tests (conversions and the tolerance rule)."""
import numpy as np
import torch

# max |gpu - ref| <= REL * RMS(ref) per float tensor
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


def rel_err(got, ref) -> float:
    got = np64(got)
    ref = np64(ref)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    if rms == 0.0:
        return 0.0 if err == 0.0 else float("inf")
    return err / rms


def assert_close(got, ref, rel=TOL_BF16, what=""):
    e = rel_err(got, ref)
    assert e <= rel, f"{what}: max|err| / RMS(ref) = {e:.3e} > {rel:.1e}"


def bf16_cuda(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).cuda()
