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


def bf16_roundings(v64, rel_window=5e-2):
    """The bf16 values a correct implementation may store for the exact value
    v64: its nearest bf16 value, and also the other neighbour when v64 lies
    within `rel_window` of a bf16 spacing from the midpoint between the two
    (5e-2 of a spacing is 2e-4 relative: the reach of an fp32 accumulation
    over thousands of products, against fp64).
    Returns (nearest, alternative) with alternative == nearest when unique."""
    from oracle import numerics as nm
    v = np.asarray(v64, np.float64)
    near = nm.round_bf16(v)
    sp = bf16_spacing(near)
    other = np.where(v >= near, near + sp, near - sp)
    mid = 0.5 * (near + other)
    ambiguous = np.abs(v - mid) <= rel_window * sp
    return near, np.where(ambiguous, other, near)


def dh_reference_candidates(dA, gu_exact, got_dh, f):
    """Reference for dH = SwiGLU-backward(dA, G, U) with G, U the stored bf16
    values: per element, the oracle value for the rounding of G and U (either
    correct rounding where the exact value sits on a midpoint, see
    bf16_roundings) that lies closest to the device result."""
    from oracle import moe as om
    gn, ga = bf16_roundings(gu_exact[..., :f])
    un, ua = bf16_roundings(gu_exact[..., f:])
    got = np.asarray(got_dh, np.float64)
    cands = [om.swiglu_backward(dA, g_, u_) for g_ in (gn, ga) for u_ in (un, ua)]
    dg = np.stack([om.round_bf16(c[0]) for c in cands])
    du = np.stack([om.round_bf16(c[1]) for c in cands])
    ig = np.argmin(np.abs(dg - got[None, ..., :f]), axis=0)
    iu = np.argmin(np.abs(du - got[None, ..., f:]), axis=0)
    pg = np.take_along_axis(dg, ig[None], axis=0)[0]
    pu = np.take_along_axis(du, iu[None], axis=0)[0]
    return np.concatenate([pg, pu], axis=-1)


def resolve_mx_dy(w, dout, pre, got_dh, w2_decoded, f, rel_window=2e-4, max_units=8):
    """dY = bf16(w * dOut) with MXFP8 operands for dA (full-size check).

    The device forms w * dOut in fp32 from its fp32 routing weights, which
    differ from the oracle's exact ones in the last bits; where w * dOut lies
    that close to a bf16 rounding midpoint either rounding of dY is correct
    (bf16_roundings with a window of 2e-4 spacing: a relative reach of 8e-7,
    several fp32 ulps).  Rounding is scale and sign invariant, so all
    elements of a row whose dOut share a significand round the same way: one
    decision per (row, significand).  A decision can change E4M3 codes or a
    block scale of the row-wise MXFP8 dY, which moves the whole dA row --
    within the format's error, but beyond the tolerance at the heavy tail of
    dH.  Per row, every combination of the decisions is a correct dY row; the
    one whose dH (through the oracle: row-wise MXFP8 of the row, times the
    decoded column-wise W2, SwiGLU backward) lies closest to the device's dH
    row is adopted.  Returns dY [rows, d] (fp64)."""
    from oracle import moe as om
    w = np.asarray(w, np.float64)
    dout = np.asarray(dout, np.float64)
    near, alt = bf16_roundings(w[:, None] * dout, rel_window)
    sig = np.frexp(np.abs(dout))[0]
    dy = near.copy()
    got = np.asarray(got_dh, np.float64)
    for r in np.nonzero(np.any(near != alt, axis=1))[0]:
        amb = near[r] != alt[r]
        units = [sig[r] == m for m in np.unique(sig[r][amb])]
        # keep the decisions that change the quantised row at all
        one = np.repeat(near[r][None], len(units) + 1, axis=0)
        for j, sel in enumerate(units):
            one[j + 1, sel] = alt[r, sel]
        q = om.mx_rowwise_decoded(one)
        units = [u for j, u in enumerate(units) if np.any(q[j + 1] != q[0])]
        if not units:
            continue
        assert len(units) <= max_units, f"row {r}: {len(units)} rounding decisions"
        cands = np.repeat(near[r][None], 1 << len(units), axis=0)
        for m in range(1 << len(units)):
            for j, sel in enumerate(units):
                if (m >> j) & 1:
                    cands[m, sel] = alt[r, sel]
        dA = om.mx_rowwise_decoded(cands) @ w2_decoded
        pr = np.repeat(np.asarray(pre[r:r + 1], np.float64), len(cands), axis=0)
        g = np.repeat(got[r:r + 1], len(cands), axis=0)
        dh = dh_reference_candidates(dA, pr, g, f)
        dist = np.max(np.abs(dh - g), axis=1)
        dy[r] = cands[int(np.argmin(dist))]
    return dy
