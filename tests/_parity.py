"""The parity rule for floating-point outputs (test infrastructure; every
reference value here is computed by ``oracle`` calls).

Budget: max|err| <= 2e-2 RMS(ref) for the BF16 path, 6e-2 RMS(ref) for MXFP8.

Which stored values are correct.  The device stores a tensor in bf16 by
rounding a value it computed in fp32.  Where the exact value lies within fp32
reach of a bf16 rounding midpoint, either neighbour is a correct result.  For
every stored element the oracle gives its *candidates*:

    near = rnd(v),  and the other neighbour of v when |v - midpoint| <= WINDOW x spacing

where v is the oracle's exact (fp64) value of the element.  WINDOW = 5e-2 of a
bf16 spacing is a relative reach of 2e-4..4e-4: about fifty times the fp32
error of a sum of thousands of products (~4e-6 relative at K = 4096), and
twenty times less than a spacing, so an implementation that rounds the wrong
way (truncation, half-up everywhere) is charged.

Chains.  A later stage reads the stored values of earlier ones, and where an
earlier element had two correct values the later exact values depend on which
one an implementation stored.  The checks therefore go stage by stage: each
stored element of a stage is compared with its candidates, the candidate the
device stored is *picked* (the oracle's nearest where the device stored
neither, and that element is charged), and the next stage's exact values are
computed by the oracle from the picked candidates.  Every picked value is one
of the oracle's own candidates, bit for bit; a device value never enters a
reference unless the oracle produced exactly that value as correct.

Charged error of an element: its distance to the nearest candidate.  Nothing
else is excused.  Every check prints the charged maximum, the strict maximum
|got - near| (no second candidate), both / RMS, and the fraction of elements
with two candidates.

fp32 outputs (routing weights, dw, d_logits, logits) have no storage rounding:
their error is |got - v| / RMS(v), nothing excused.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from oracle import moe as om
from oracle import numerics as nm

TOL_BF16 = 2e-2
TOL_MXFP8 = 6e-2
WINDOW = 5e-2


def spacing(v) -> np.ndarray:
    """bf16 spacing at |v|: distance from a bf16 value of that binade to the
    next one away from zero (0 at v = 0)."""
    v = np.abs(np.asarray(v, np.float64))
    _, e = np.frexp(v)
    sp = np.ldexp(1.0, np.maximum(e, -125) - 8)
    return np.where(v == 0.0, 0.0, sp)


@dataclass
class Cand:
    """Candidates of a stored bf16 tensor: ``near`` everywhere, ``alt`` the
    other correct value (equal to ``near`` where there is none)."""
    near: np.ndarray
    alt: np.ndarray

    @property
    def two(self) -> float:
        """Fraction of elements with two correct values."""
        return float(np.mean(self.near != self.alt)) if self.near.size else 0.0


_CLIB = None


def _clib():
    """tests/_cand.c (candidates and tallies in one pass, OpenMP), built with
    gcc into the repository's _build/ folder when missing or stale."""
    global _CLIB
    if _CLIB is None:
        import ctypes as C
        import os
        import subprocess
        here = os.path.dirname(os.path.abspath(__file__))
        src = os.path.join(here, "_cand.c")
        out_dir = os.path.join(os.path.dirname(here), "_build")
        so = os.path.join(out_dir, "tests_cand.so")
        if not os.path.exists(so) or os.path.getmtime(so) < os.path.getmtime(src):
            os.makedirs(out_dir, exist_ok=True)
            tmp = f"{so}.{os.getpid()}"
            subprocess.run(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", tmp, src, "-lm"],
                           check=True)
            os.replace(tmp, so)
        lib = C.CDLL(so)
        lib.cand_tally.restype = None
        lib.cand_only.restype = None
        _CLIB = lib
    return _CLIB


def _ptr(a):
    import ctypes as C
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def candidates(v, window=None) -> Cand:
    """The correct stored bf16 values of exact values ``v`` (tests/_cand.c):
    near = round-to-nearest-even; the other neighbour of v also when the 45
    dropped fraction bits of v lie within window x 2^45 of the halfway
    pattern 2^44, i.e. |v - midpoint| <= window x spacing.  Below the bf16
    normal range (|v| < 2^-126): the subnormal grid and no second value."""
    import ctypes as C
    window = WINDOW if window is None else window
    v = np.ascontiguousarray(v, dtype=np.float64)
    near = np.empty_like(v)
    alt = np.empty_like(v)
    _clib().cand_only(_ptr(v), C.c_int64(v.size), C.c_double(window), _ptr(near), _ptr(alt))
    return Cand(near, alt)


def tally_piece(v, got, window=None):
    """One pass over exact values ``v`` and a device tensor ``got`` (bf16
    torch tensor or fp64 array): (picks, [max charged, max strict, sum
    near^2, number with two candidates])."""
    import ctypes as C
    window = WINDOW if window is None else window
    v = np.ascontiguousarray(v, dtype=np.float64)
    g16 = g64 = None
    if isinstance(got, np.ndarray):
        g64 = np.ascontiguousarray(got, dtype=np.float64)
    else:
        import torch
        t = got.detach().contiguous().cpu()
        if t.dtype == torch.bfloat16:
            g16 = t.view(torch.int16).numpy()
        else:
            g64 = t.double().numpy()
    shape = (g16 if g16 is not None else g64).shape
    if shape != v.shape:
        raise AssertionError(f"shape {shape} != {v.shape}")
    pick_ = np.empty_like(v)
    stats = np.zeros(4)
    _clib().cand_tally(_ptr(v), _ptr(g16), _ptr(g64), C.c_int64(v.size), C.c_double(window),
                       _ptr(pick_), _ptr(stats))
    return pick_, stats


def _f64(t) -> np.ndarray:
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    import torch
    t = t.detach().cpu()
    if t.dtype in (torch.bfloat16, torch.float16):
        t = t.float()
    return t.double().numpy()


def _rms(a) -> float:
    return float(np.sqrt(np.mean(np.square(a)))) if a.size else 0.0


def charged_error(got, c: Cand) -> tuple[float, float]:
    """(charged, strict) max error / RMS(near)."""
    g = _f64(got)
    if g.shape != c.near.shape:
        raise AssertionError(f"shape {g.shape} != {c.near.shape}")
    if c.near.size == 0:
        return 0.0, 0.0
    st = np.abs(g - c.near)
    ch = np.minimum(st, np.abs(g - c.alt))
    ch = np.where(np.isnan(g), np.inf, ch)
    rms = _rms(c.near)
    if rms == 0.0:
        return (0.0 if np.all(ch == 0) else np.inf), (0.0 if np.all(st == 0) else np.inf)
    return float(np.max(ch)) / rms, float(np.max(st)) / rms


def pick(got, c: Cand) -> np.ndarray:
    """Per element, the candidate the device stored, else the oracle's nearest."""
    g = _f64(got)
    return np.where(g == c.alt, c.alt, c.near)


def check(got, c: Cand, tol: float, what: str, oracle=None) -> np.ndarray:
    """Assert the charged error of a stored bf16 tensor is within ``tol``;
    returns the picked candidates.  ``oracle``: the oracle's own stored value
    of the tensor (no picks upstream), reported as a second strict figure."""
    g = _f64(got)
    ch, st = charged_error(g, c)
    extra = ""
    if oracle is not None:
        o = np.asarray(oracle, np.float64)
        r = _rms(o)
        extra = f" vs oracle {float(np.max(np.abs(g - o))) / r if r else 0.0:.3e}"
    print(f"parity {what}: charged {ch:.3e} strict {st:.3e}{extra} tol {tol:.0e} "
          f"(max|err| / RMS; {100 * c.two:.3f} % of elements with two correct values)")
    assert ch <= tol, f"{what}: charged max|err| / RMS(ref) = {ch:.3e} > {tol:.1e} (strict {st:.3e})"
    return pick(g, c)


def check_f32(got, v, tol: float, what: str) -> float:
    """Assert max|got - v| / RMS(v) <= tol for an fp32 output."""
    g = _f64(got)
    v = np.asarray(v, np.float64)
    if g.shape != v.shape:
        raise AssertionError(f"{what}: shape {g.shape} != {v.shape}")
    if v.size == 0:
        return 0.0
    d = np.where(np.isnan(g), np.inf, np.abs(g - v))
    r = _rms(v)
    e = float(np.max(d)) / r if r else (0.0 if np.all(d == 0) else np.inf)
    print(f"parity {what}: strict {e:.3e} tol {tol:.0e} (max|err| / RMS, fp32)")
    assert e <= tol, f"{what}: max|err| / RMS(ref) = {e:.3e} > {tol:.1e}"
    return e


class Tally:
    """Whole-tensor figures of a tensor checked in pieces (expert by expert):
    ``add`` checks one piece and returns its picks, ``finish`` asserts the
    charged maximum over all pieces against the RMS over all pieces (one
    pass of tests/_cand.c per piece: the pieces of the large workloads hold
    tens of millions of elements)."""

    def __init__(self, tol):
        self.tol = tol if callable(tol) else (lambda key: tol)
        self.s = {}

    def add(self, key, got, v) -> np.ndarray:
        """Check device piece ``got`` against the candidates of exact values
        ``v``; returns the picks."""
        pick_, (ch, st, ss, two) = tally_piece(v, got)
        r = self.s.setdefault(key, [0.0, 0.0, 0.0, 0, 0])
        r[0] = max(r[0], ch)
        r[1] = max(r[1], st)
        r[2] += ss
        r[3] += pick_.size
        r[4] += int(two)
        return pick_

    def finish(self):
        bad = []
        for key, (ch, st, ss, n, two) in self.s.items():
            rms = np.sqrt(ss / n) if n else 0.0
            c = ch / rms if rms else (0.0 if ch == 0 else np.inf)
            print(f"parity {key}: charged {c:.3e} strict {st / rms if rms else 0.0:.3e} "
                  f"tol {self.tol(key):.0e} (max|err| / RMS over {n} elements; "
                  f"{100 * two / max(n, 1):.3f} % with two correct values)")
            if c > self.tol(key):
                bad.append(f"{key}: {c:.3e}")
        assert not bad, "charged max|err| / RMS beyond the budget: " + ", ".join(bad)


# ---------------------------------------------------------------------------
# the layer, stage by stage
# ---------------------------------------------------------------------------

def _qr(a, mx):
    """Operand with its reduction axis last (row-wise MXFP8 when ``mx``)."""
    return om.mx_rowwise_decoded(a) if mx else np.asarray(a, np.float64)


def _qc(a, mx, offsets=None):
    """Operand with its reduction axis first (column-wise MXFP8 per group)."""
    if not mx:
        return np.asarray(a, np.float64)
    return om.mx_colwise_decoded(a, [0, np.asarray(a).shape[0]] if offsets is None else offsets)


class Stages:
    """Checks the stored tensors of one run of the expert part of the layer
    (GEMM1 + SwiGLU, GEMM2, combine backward's dY, dA + SwiGLU backward, dX,
    dW2, dW13) on routed rows in expert order, stage by stage.

    x_perm [M, d] (exact copies), w13 [E, 2f, d], w2 [E, d, f], offsets
    [E + 1]; ``mx`` as the oracle's selection (bool or GEMM names); ``tol`` a
    number or a function of the tensor name.  Each ``check_*`` method takes
    the device's tensor, checks it and keeps the picked candidates for the
    later stages; ``oracle`` arguments give the oracle's own values for the
    report."""

    def __init__(self, x_perm, w13, w2, offsets, mx=False, tol=TOL_BF16, sink=None):
        self.xp = np.asarray(x_perm, np.float64)
        self.w13 = np.asarray(w13, np.float64)
        self.w2 = np.asarray(w2, np.float64)
        self.off = np.asarray(offsets, np.int64)
        self.E, f2, self.d = self.w13.shape
        self.f = f2 // 2
        self.mx = lambda g: om._mx_on(mx, g)  # noqa: E731
        self.tol = tol if callable(tol) else (lambda key: tol)
        self.sink = sink     # a Tally: record instead of asserting per call
        self.p = {}

    def _w(self, name, w, gemm, cols):
        key = (name, gemm, cols)
        if key not in self.p:
            mx = self.mx(gemm)
            self.p[key] = w if not mx else np.stack(
                [_qc(w[e], mx) if cols else _qr(w[e], mx) for e in range(self.E)])
        return self.p[key]

    def _chk(self, key, got, v, oracle=None):
        if self.sink is not None:
            self.p[key] = self.sink.add(key, got, v)
        else:
            self.p[key] = check(got, candidates(v), self.tol(key), key, oracle)
        return self.p[key]

    def gu_exact(self):
        """[G | U] before rounding (fp64 from the exact routed rows)."""
        if "gu_exact" not in self.p:
            self.p["gu_exact"] = om.grouped_gemm_ragged_m(
                _qr(self.xp, self.mx("gemm1")), self._w("w13", self.w13, "gemm1", False), self.off)
        return self.p["gu_exact"]

    def check_gu(self, got, oracle=None):
        return self._chk("GU", got, self.gu_exact(), oracle)

    def check_a(self, got, oracle=None):
        gu, f = self.gu_exact(), self.f
        return self._chk("A", got, om.silu(gu[:, :f]) * gu[:, f:], oracle)

    def y_exact(self):
        return om.grouped_gemm_ragged_m(_qr(self.p["A"], self.mx("gemm2")),
                                        self._w("w2", self.w2, "gemm2", False), self.off)

    def check_y(self, got, oracle=None):
        return self._chk("Y_perm", got, self.y_exact(), oracle)

    def check_dy(self, got, w_rows, dout_rows, oracle=None):
        v = np.asarray(w_rows, np.float64)[:, None] * np.asarray(dout_rows, np.float64)
        return self._chk("dY_perm", got, v, oracle)

    def dh_exact(self):
        f = self.f
        dA = om.grouped_gemm_ragged_m(_qr(self.p["dY_perm"], self.mx("dA")),
                                      self._w("w2", self.w2, "dA", True), self.off, b_mn_major=True)
        gu = self.p["GU"]
        dG, dU = om.swiglu_backward(dA, gu[:, :f], gu[:, f:])
        return np.concatenate([dG, dU], axis=1)

    def check_dh(self, got, oracle=None):
        return self._chk("dH", got, self.dh_exact(), oracle)

    def check_dx_perm(self, got, oracle=None):
        v = om.grouped_gemm_ragged_m(_qr(self.p["dH"], self.mx("dX")),
                                     self._w("w13", self.w13, "dX", True), self.off, b_mn_major=True)
        return self._chk("dX_perm", got, v, oracle)

    def check_dw2(self, got, oracle=None):
        m = self.mx("dW2")
        v = om.grouped_gemm_ragged_k(_qc(self.p["dY_perm"], m, self.off), _qc(self.p["A"], m, self.off),
                                     self.off)
        return self._chk("dW2", got, v, oracle)

    def check_dw13(self, got, oracle=None):
        m = self.mx("dW13")
        v = om.grouped_gemm_ragged_k(_qc(self.p["dH"], m, self.off), _qc(self.xp, m, self.off), self.off)
        return self._chk("dW13", got, v, oracle)


def check_layer_outputs(st: Stages, got, idx, w, dest, dout=None, x=None, wr=None, oracle=None):
    """The token-side outputs after the expert stages: out from the picked
    Y_perm; dw and d_logits (fp32) from the picked Y_perm; dx from the picked
    dX_perm (+ the router term); dW_r.  ``got``: dict of device tensors with
    keys out, and for the backward dw, d_logits, dx (, dWr).  ``oracle``:
    the oracle's own outputs by the same names (reported only)."""
    o = oracle or {}
    E = st.E
    w = np.asarray(w, np.float64)
    st._chk("out", got["out"], om.combine(st.p["Y_perm"], dest, w, bf16=False), o.get("out"))
    if dout is None:
        return
    _, dw = om.combine_backward(dout, st.p["Y_perm"], dest, w, bf16=False)
    check_f32(got["dw"], dw, st.tol("dw"), "dw")
    dl = om.router_backward(w, dw, idx, E)
    check_f32(got["d_logits"], dl, st.tol("d_logits"), "d_logits")
    extra = None
    if wr is not None:
        extra, dwr = om.router_proj_backward(x, wr, dl)
        st._chk("dWr", got["dWr"], dwr, o.get("dWr"))
    st._chk("dx", got["dx"], om.unpermute_sum(st.p["dX_perm"], dest, extra, bf16=False), o.get("dx"))
