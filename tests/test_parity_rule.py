"""The parity rule of tests/_parity.py, on the CPU (no GPU involved).

* Fed the oracle's own stored tensors, the stage-by-stage checks pick the
  oracle's nearest value everywhere and charge nothing.
* A correct implementation that differs from the oracle only by computing in
  fp32 (a plain PyTorch CPU statement of the layer below: fp32 products and
  sums in library order, bf16 round-to-nearest-even stores) passes, and some
  of its elements do take the second correct value.
* The same implementation storing by truncation (round toward zero) instead
  of rounding to nearest is charged beyond the budget, and so is a single
  element one spacing off at the largest value of a tensor.
"""
import numpy as np
import pytest
import torch

from oracle import moe as om
from routing_grouped_gemm_moe_b200 import inputs as I

from . import _parity as P

CASES = {
    "ragged": I.LayerConfig("ragged", T=300, d=256, E=6, k=2, f=384, logits="zipf", n_empty=1,
                            zipf_s=0.8, seed=71),
    "wide": I.LayerConfig("wide", T=256, d=1024, E=4, k=2, f=512, seed=79),
    "mx_ragged": I.LayerConfig("mx_ragged", T=300, d=256, E=6, k=2, f=384, logits="zipf",
                               n_empty=1, zipf_s=0.8, dtype="mxfp8", seed=75),
}


def _f64(t):
    return t.float().double().numpy()


def _store(t, truncate=False):
    """fp32 -> bf16 bits -> fp64 values (nearest-even, or toward zero)."""
    t = t.float()
    if truncate:
        b = (t.view(torch.int32) & -65536).view(torch.float32)
        return b.double().numpy()
    return t.to(torch.bfloat16).double().numpy()


def fp32_layer(x, w13, w2, idx, w, dout, E, f, mx=False, truncate=False):
    """The layer as an fp32 implementation computes it: stores in bf16,
    MXFP8 operands encoded from the stored values (the oracle's encoder, a
    bit-exact definition), fp32 routing weights."""
    T, k = idx.shape
    _, off, dest, src = om.dispatch_plan(idx, E)
    t32 = lambda a: torch.tensor(np.asarray(a), dtype=torch.float32)  # noqa: E731
    qr = (lambda a: om.mx_rowwise_decoded(a)) if mx else (lambda a: a)          # noqa: E731
    qc = (lambda a, o=None: om.mx_colwise_decoded(a, [0, a.shape[0]] if o is None else o)) \
        if mx else (lambda a, o=None: a)
    st = lambda v: _store(v, truncate)  # noqa: E731
    M = T * k
    xp = x[src]
    r = {n: np.zeros(s) for n, s in (("GU", (M, 2 * f)), ("A", (M, f)), ("Y_perm", (M, x.shape[1])),
                                      ("dY_perm", (M, x.shape[1])), ("dH", (M, 2 * f)),
                                      ("dX_perm", (M, x.shape[1])), ("dW2", (E, x.shape[1], f)),
                                      ("dW13", (E, 2 * f, x.shape[1])))}
    xq = qr(xp)
    for e in range(E):
        a, b = off[e], off[e + 1]
        if a == b:
            continue
        gu = t32(xq[a:b]) @ t32(qr(w13[e])).T
        r["GU"][a:b] = st(gu)
        g, u = gu[:, :f], gu[:, f:]
        r["A"][a:b] = st(g * torch.sigmoid(g) * u)
    aq = qr(r["A"])
    for e in range(E):
        a, b = off[e], off[e + 1]
        if a < b:
            r["Y_perm"][a:b] = st(t32(aq[a:b]) @ t32(qr(w2[e])).T)
    w32 = t32(w)
    Y = t32(r["Y_perm"])
    r["out"] = st(sum(w32[:, i:i + 1] * Y[dest[:, i]] for i in range(k)))
    do = t32(dout)
    dw = torch.stack([(do * Y[dest[:, i]]).sum(1) for i in range(k)], 1)
    for i in range(k):
        r["dY_perm"][dest[:, i]] = st(w32[:, i:i + 1] * do)
    dyq = qr(r["dY_perm"])
    for e in range(E):
        a, b = off[e], off[e + 1]
        if a == b:
            continue
        dA = t32(dyq[a:b]) @ t32(qc(w2[e]))
        G, U = t32(r["GU"][a:b, :f]), t32(r["GU"][a:b, f:])
        s = torch.sigmoid(G)
        r["dH"][a:b] = np.concatenate([st(dA * U * s * (1 + G * (1 - s))), st(dA * G * s)], 1)
    dhq = qr(r["dH"])
    dyc, ac = qc(r["dY_perm"], off), qc(r["A"], off)
    dhc, xc = qc(r["dH"], off), qc(xp, off)
    for e in range(E):
        a, b = off[e], off[e + 1]
        if a == b:
            continue
        r["dX_perm"][a:b] = st(t32(dhq[a:b]) @ t32(qc(w13[e])))
        r["dW2"][e] = st(t32(dyc[a:b]).T @ t32(ac[a:b]))
        r["dW13"][e] = st(t32(dhc[a:b]).T @ t32(xc[a:b]))
    dX = t32(r["dX_perm"])
    r["dx"] = st(sum(dX[dest[:, i]] for i in range(k)))
    r["dw"] = dw.double().numpy()
    wd = (w32 * dw).sum(1, keepdim=True)
    dl = torch.zeros(T, E)
    dl.scatter_(1, torch.tensor(idx, dtype=torch.int64), w32 * (dw - wd))
    r["d_logits"] = dl.double().numpy()
    return r


def _case(name):
    cfg = CASES[name]
    inp = I.make_inputs(cfg)
    x, w13, w2, dout = (_f64(inp[n]) for n in ("x", "w13", "w2", "dout"))
    mx = cfg.dtype == "mxfp8"
    fwd = om.layer_forward(x, w13, w2, cfg.k, logits32=inp["logits"].numpy(), mx=mx)
    bwd = om.layer_backward(fwd, dout, x, w13, w2, mx=mx)
    return cfg, (x, w13, w2, dout), fwd, bwd, mx


def run_checks(cfg, arrays, fwd, bwd, mx, dev):
    """The stage-by-stage checks on a device result ``dev`` (dict of arrays);
    returns the Stages with the picks."""
    x, w13, w2, dout = arrays
    tol = P.TOL_MXFP8 if mx else P.TOL_BF16
    dest, src = fwd["dest_pos"], fwd["src_token"]
    S = P.Stages(fwd["x_perm"], w13, w2, fwd["offsets"], mx, tol)
    S.check_gu(dev["GU"], fwd["GU"])
    S.check_a(dev["A"], fwd["A"])
    S.check_y(dev["Y_perm"], fwd["Y_perm"])
    w_rows = np.zeros(dest.size)
    w_rows[dest.reshape(-1)] = fwd["topk_w"].reshape(-1)
    S.check_dy(dev["dY_perm"], w_rows, dout[src], bwd["dY_perm"])
    S.check_dh(dev["dH"], bwd["dH"])
    S.check_dx_perm(dev["dX_perm"], bwd["dX_perm"])
    S.check_dw2(dev["dW2"], bwd["dW2"])
    S.check_dw13(dev["dW13"], bwd["dW13"])
    P.check_layer_outputs(S, dev, fwd["topk_idx"], fwd["topk_w"], dest, dout,
                          oracle={"out": fwd["out"], "dx": bwd["dx"]})
    return S


@pytest.mark.parametrize("name", list(CASES))
def test_the_oracle_itself_is_charged_nothing(name):
    cfg, arrays, fwd, bwd, mx = _case(name)
    dev = dict(fwd, **bwd)
    S = run_checks(cfg, arrays, fwd, bwd, mx, dev)
    for key in ("GU", "A", "Y_perm", "out"):
        assert np.array_equal(S.p[key], fwd[key]), key
    for key in ("dY_perm", "dH", "dX_perm", "dW2", "dW13", "dx"):
        assert np.array_equal(S.p[key], bwd[key]), key


@pytest.mark.parametrize("name", list(CASES))
def test_a_correct_fp32_implementation_passes(name):
    cfg, arrays, fwd, bwd, mx = _case(name)
    x, w13, w2, dout = arrays
    dev = fp32_layer(x, w13, w2, fwd["topk_idx"], fwd["topk_w"], dout, cfg.E, cfg.f, mx)
    S = run_checks(cfg, arrays, fwd, bwd, mx, dev)
    # it does differ from the oracle's nearest values somewhere, and each of
    # those elements is the oracle's second correct value
    assert any(np.any(S.p[k] != bwd.get(k, fwd.get(k))) for k in ("GU", "A", "Y_perm", "dH", "dX_perm"))


@pytest.mark.parametrize("name", ["ragged", "wide"])
def test_a_truncating_implementation_is_charged(name):
    cfg, arrays, fwd, bwd, mx = _case(name)
    x, w13, w2, dout = arrays
    dev = fp32_layer(x, w13, w2, fwd["topk_idx"], fwd["topk_w"], dout, cfg.E, cfg.f, mx,
                     truncate=True)
    with pytest.raises(AssertionError, match="charged"):
        run_checks(cfg, arrays, fwd, bwd, mx, dev)


def test_one_spacing_off_at_the_largest_element_is_charged():
    cfg, arrays, fwd, bwd, mx = _case("ragged")
    c = P.candidates(om.grouped_gemm_ragged_k(bwd["dH"], fwd["x_perm"], fwd["offsets"]))
    assert np.array_equal(c.near, bwd["dW13"])
    got = c.near.copy()
    i = np.unravel_index(np.argmax(np.abs(got)), got.shape)
    got[i] += np.copysign(P.spacing(got[i]), got[i])
    ch, strict = P.charged_error(got, c)
    assert ch == strict > P.TOL_BF16


def test_candidates_round_like_the_oracle():
    """candidates' nearest value is the oracle's bf16 rounding (ties to even,
    binade edges, signs, zeros, the subnormal range), and the second value
    is the neighbour on the other side of v, present exactly when v lies
    within the window of the halfway point between the two."""
    from oracle import numerics as nm
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.standard_normal(100000) * 10.0 ** rng.integers(-30, 30, 100000),
                        [0.0, -0.0, 1.0, -1.0, 2.0 ** -126, 2.0 ** -130, -3e-39, 1e30]])
    c = P.candidates(v)
    assert np.array_equal(c.near, nm.round_bf16(v))
    # consecutive bf16 values a < b (binade edges included), their midpoint,
    # and points just inside and just outside the window
    a32 = nm.round_bf16(rng.standard_normal(5000) * 4.0).astype(np.float32)
    a32[:8] = [1.0, 2.0, 0.5, -1.0, -2.0, 4.0, -0.25, 8.0]
    bits = a32.view(np.uint32)
    b32 = np.where(a32 >= 0, bits + (1 << 16), bits - (1 << 16)).astype(np.uint32).view(np.float32)
    a, b = np.minimum(a32, b32).astype(np.float64), np.maximum(a32, b32).astype(np.float64)
    m, w = 0.5 * (a + b), b - a
    for off, two in ((0.0, True), (0.04, True), (-0.04, True), (0.06, False), (-0.06, False)):
        c = P.candidates(m + off * w)
        assert np.array_equal(c.near, nm.round_bf16(m + off * w))
        got = np.sort(np.stack([c.near, c.alt]), axis=0)
        if two:
            assert np.array_equal(got[0], a) and np.array_equal(got[1], b), off
        else:
            assert np.array_equal(c.near, c.alt), off
