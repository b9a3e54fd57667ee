"""Whole-layer parity (forward + backward) against the CPU oracle (needs a B200).

Small layers are compared element by element; they span several GEMM tiles
and ragged expert tails, an expert with no tokens and both router modes.
"""
import numpy as np
import pytest
import torch

from oracle import moe as om
from oracle import ref_c as rc
from routing_grouped_gemm_moe_b200 import inputs as I
from routing_grouped_gemm_moe_b200 import ops

from . import _parity as P
from ._parity import TOL_BF16, TOL_MXFP8
from ._util import assert_close, np64, npi, resolve_routing

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": I.CONFIGS["tiny"],
    "ragged": I.LayerConfig("ragged", T=300, d=256, E=6, k=2, f=384, logits="zipf", n_empty=1,
                            zipf_s=0.8, seed=71),
    "proj_wide": I.LayerConfig("proj_wide", T=520, d=136, E=12, k=3, f=200, router="proj", seed=72),
    "one_token": I.LayerConfig("one_token", T=1, d=64, E=4, k=2, f=64, seed=73),
    "all_one_expert": I.LayerConfig("all_one_expert", T=200, d=128, E=5, k=1, f=128,
                                    logits="zipf", n_empty=4, seed=74),
    "mx_ragged": I.LayerConfig("mx_ragged", T=300, d=256, E=6, k=2, f=384, logits="zipf",
                               n_empty=1, zipf_s=0.8, dtype="mxfp8", seed=75),
    "mx_proj": I.LayerConfig("mx_proj", T=200, d=128, E=8, k=2, f=256, router="proj",
                             dtype="mxfp8", seed=76),
}


def _forward_with_routing(x, w13, w2, cfg, idx, logits64, mx=None):
    """The oracle forward for a given (validated) selection, step by step."""
    if mx is None:
        mx = cfg.dtype == "mxfp8"
    w = om.router_weights(logits64.astype(np.float32), idx)
    counts, offsets, dest, src = om.dispatch_plan(idx, cfg.E)
    x_perm = om.dispatch_rows(x, src)
    GU, A, Y = om.expert_forward(x_perm, w13, w2, offsets, mx=mx)
    out = om.combine(Y, dest, w)
    return dict(logits=logits64, topk_idx=idx, topk_w=w, counts=counts, offsets=offsets,
                dest_pos=dest, src_token=src, x_perm=x_perm, GU=GU, A=A, Y_perm=Y, out=out)


def run_layer(cfg, inp, **opts):
    layer = ops.MoELayer(cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, router=cfg.router, dtype=cfg.dtype,
                         **opts)
    g = {n: t.cuda() for n, t in inp.items()}
    out = layer.forward(g["x"], g["w13"], g["w2"], logits=g.get("logits"), w_r=g.get("wr"))
    layer.backward(g["dout"], g["x"], g["w13"], g["w2"], logits=g.get("logits"), w_r=g.get("wr"))
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    return layer, out


def ws_views(layer):
    """Backward intermediates the layer leaves in its workspace (the layout
    documented for moe_layer_bwd: status word, dispatch scratch, dY_perm
    reused for dX_perm, dH, dw; recompute mode then [G | U] and A; all
    sub-buffers 256-byte aligned)."""
    al = lambda v: (v + 255) // 256 * 256  # noqa: E731
    T, d, E, k, f = layer.T, layer.d, layer.E, layer.k, layer.f
    M = T * k
    ws = layer.workspace
    off = 256 + al(ops.permute_workspace_bytes(T, E) - 256)
    views = {}

    def take(name, nbytes, dtype, shape):
        nonlocal off
        views[name] = ws[off:off + nbytes].view(dtype).view(*shape)
        off += al(nbytes)

    take("dX_perm", M * d * 2, torch.bfloat16, (M, d))
    take("dH", M * 2 * f * 2, torch.bfloat16, (M, 2 * f))
    take("dw", T * k * 4, torch.float32, (T, k))
    if layer.recompute:
        take("GU", M * 2 * f * 2, torch.bfloat16, (M, 2 * f))
        take("A", M * f * 2, torch.bfloat16, (M, f))
    return views


def check_layer(layer, out, inp, fwd, bwd, mx, tol, wr=None):
    """Every float output and intermediate of a layer run, stage by stage
    against the oracle (tests/_parity.py: the device's stored value must be
    one of the oracle's correct values of each element; later stages are
    computed by the oracle from those values).  ``tol``: a number, or a
    function of the tensor name (selective MXFP8)."""
    st = layer.state
    wsv = ws_views(layer)
    x, w13, w2, dout = (np64(inp[n]) for n in ("x", "w13", "w2", "dout"))
    dest, src, idx, w = fwd["dest_pos"], fwd["src_token"], fwd["topk_idx"], fwd["topk_w"]
    S = P.Stages(fwd["x_perm"], w13, w2, fwd["offsets"], mx, tol)
    S.check_gu(st.gu if st.gu is not None else wsv["GU"], fwd["GU"])
    S.check_a(st.a if st.a is not None else wsv["A"], fwd["A"])
    S.check_y(st.y_perm, fwd["Y_perm"])
    # dY_perm is overwritten by dX_perm inside the backward: it is taken from
    # the layer's combine-backward kernel called again on the layer's own
    # inputs (the dw that call writes must be the layer's, bit for bit)
    dy_dev, dw_dev = ops.unpermute_combine_bwd(inp["dout"].cuda(), st.y_perm, st.dest_pos,
                                               st.topk_w)
    assert torch.equal(dw_dev, wsv["dw"])
    w_rows = np.zeros(dest.size)
    w_rows[dest.reshape(-1)] = np.asarray(w, np.float64).reshape(-1)
    S.check_dy(dy_dev, w_rows, dout[src], bwd["dY_perm"])
    S.check_dh(wsv["dH"], bwd["dH"])
    S.check_dx_perm(wsv["dX_perm"], bwd["dX_perm"])
    S.check_dw2(layer.dw2, bwd["dW2"])
    S.check_dw13(layer.dw13, bwd["dW13"])
    got = {"out": out, "dw": wsv["dw"], "d_logits": layer.d_logits, "dx": layer.dx,
           "dWr": layer.dw_r}
    P.check_layer_outputs(S, got, idx, w, dest, dout, x, wr,
                          oracle={"out": fwd["out"], "dx": bwd["dx"], "dWr": bwd.get("dWr")})
    for e in np.nonzero(fwd["counts"] == 0)[0]:
        assert torch.all(layer.dw13[e] == 0) and torch.all(layer.dw2[e] == 0)


def oracle_layer(cfg, inp, layer, mx):
    """The oracle's layer (forward + backward) for the routing the oracle
    decides (router projection: validated against the device's fp32 logits,
    ambiguous near-ties resolved as resolve_routing documents)."""
    x, w13, w2, dout = (np64(inp[n]) for n in ("x", "w13", "w2", "dout"))
    wr = np64(inp["wr"]) if "wr" in inp else None
    st = layer.state
    if wr is not None:
        ref_lg = om.router_logits(x, wr)
        assert_close(st.logits, ref_lg, 1e-5, "logits")
        ridx, _ = resolve_routing(ref_lg, npi(st.topk_idx), cfg.k)
        fwd = _forward_with_routing(x, w13, w2, cfg, ridx, ref_lg, mx=mx)
    else:
        fwd = om.layer_forward(x, w13, w2, cfg.k, logits32=inp["logits"].numpy(), mx=mx)
    bwd = om.layer_backward(fwd, dout, x, w13, w2, wr=wr, mx=mx)
    return fwd, bwd, wr


def _check_routing(layer, inp, fwd):
    st = layer.state
    for key in ("topk_idx", "counts", "offsets", "dest_pos", "src_token"):
        assert np.array_equal(npi(getattr(st, key)), fwd[key]), key
    assert np.array_equal(st.x_perm.cpu().view(torch.int16).numpy(),
                          inp["x"].view(torch.int16).numpy()[fwd["src_token"]])
    assert_close(st.topk_w, fwd["topk_w"], 1e-5, "topk_w")


@pytest.mark.parametrize("name", list(SMALL))
def test_layer_matches_oracle(name):
    cfg = SMALL[name]
    inp = I.make_inputs(cfg)
    layer, out = run_layer(cfg, inp)
    mx = cfg.dtype == "mxfp8"
    fwd, bwd, wr = oracle_layer(cfg, inp, layer, mx)
    _check_routing(layer, inp, fwd)
    check_layer(layer, out, inp, fwd, bwd, mx, TOL_MXFP8 if mx else TOL_BF16, wr)


@pytest.mark.parametrize("name", ["ragged", "one_token", "all_one_expert", "mx_ragged"])
def test_layer_matches_c_oracle(name):
    """The same layer against the independent C oracle (plain fp64 loops per
    token and selected expert); layers routed on given fp32 logits, so the
    selection is fixed by the inputs.  Every stored tensor of the C oracle
    must equal the numpy oracle's bit for bit (the stage-by-stage checks are
    computed with the numpy oracle's steps); the device is then checked stage
    by stage, with the C oracle's values as the reported reference."""
    cfg = SMALL[name]
    inp = I.make_inputs(cfg)
    layer, out = run_layer(cfg, inp)
    x, w13, w2, dout = (np64(inp[n]) for n in ("x", "w13", "w2", "dout"))
    mx = cfg.dtype == "mxfp8"
    fwd = rc.layer_forward(x, w13, w2, cfg.k, logits32=inp["logits"].numpy(), mx=mx)
    bwd = rc.layer_backward(fwd, dout, x, w13, w2, mx=mx)
    nf = om.layer_forward(x, w13, w2, cfg.k, logits32=inp["logits"].numpy(), mx=mx)
    nb = om.layer_backward(nf, dout, x, w13, w2, mx=mx)
    for key in ("GU", "A", "Y_perm", "out"):
        assert np.array_equal(fwd[key], nf[key]), key
    for key in ("dY_perm", "dH", "dX_perm", "dW2", "dW13", "dx"):
        assert np.array_equal(bwd[key], nb[key]), key
    _check_routing(layer, inp, fwd)
    check_layer(layer, out, inp, fwd, bwd, mx, TOL_MXFP8 if mx else TOL_BF16)


def test_layer_is_deterministic():
    cfg = SMALL["ragged"]
    inp = I.make_inputs(cfg)
    l1, o1 = run_layer(cfg, inp)
    r1 = [t.clone() for t in (o1, l1.dx, l1.dw13, l1.dw2)]
    l2, o2 = run_layer(cfg, inp)
    for a, b in zip(r1, (o2, l2.dx, l2.dw13, l2.dw2)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_layer_captures_in_a_cuda_graph():
    """A forward + backward contains no synchronising call (capture would
    fail on one); the replayed graph reproduces the eager results bit for bit."""
    cfg = SMALL["ragged"]
    inp = I.make_inputs(cfg)
    g = {n: t.cuda() for n, t in inp.items()}
    layer = ops.MoELayer(cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, router=cfg.router)

    def step():
        layer.forward(g["x"], g["w13"], g["w2"], logits=g.get("logits"))
        layer.backward(g["dout"], g["x"], g["w13"], g["w2"], logits=g.get("logits"))

    step()
    torch.cuda.synchronize()
    ref = [t.clone() for t in (layer.out, layer.dx, layer.dw13, layer.dw2, layer.d_logits)]
    for t in (layer.out, layer.dx, layer.dw13, layer.dw2):
        t.zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    graph.replay()
    torch.cuda.synchronize()
    got = (layer.out, layer.dx, layer.dw13, layer.dw2, layer.d_logits)
    for a, b in zip(ref, got):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
    del graph


@pytest.mark.parametrize("name", ["ragged", "proj_wide", "mx_ragged", "mx_proj"])
def test_recompute_matches_oracle(name):
    """Recompute mode keeps [G | U] and A only in the workspace and runs GEMM1 +
    SwiGLU again in the backward.  Its outputs, and the recomputed [G | U] and
    A it leaves in the workspace, are checked against the oracle under the
    same rule as the stored-activation mode -- and are also that mode's results
    bit for bit (same kernels, same inputs)."""
    cfg = SMALL[name]
    inp = I.make_inputs(cfg)
    l2, o2 = run_layer(cfg, inp, recompute=True)
    assert l2.state.gu is None and l2.state.a is None
    mx = cfg.dtype == "mxfp8"
    fwd, bwd, wr = oracle_layer(cfg, inp, l2, mx)
    _check_routing(l2, inp, fwd)
    check_layer(l2, o2, inp, fwd, bwd, mx, TOL_MXFP8 if mx else TOL_BF16, wr)
    l1, o1 = run_layer(cfg, inp)
    ref = [o1, l1.dx, l1.dw13, l1.dw2, l1.d_logits, l1.state.gu, l1.state.a]
    wsv = ws_views(l2)
    for a, b in zip(ref, (o2, l2.dx, l2.dw13, l2.dw2, l2.d_logits, wsv["GU"], wsv["A"])):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))


SELECTIONS = [("gemm1", "gemm2"), ("dA", "dX"), ("dW2", "dW13"), ("gemm2", "dA", "dW13")]


@pytest.mark.parametrize("sel", SELECTIONS, ids=["+".join(s) for s in SELECTIONS])
def test_selective_mxfp8_matches_oracle(sel):
    """Only the named GEMMs take MXFP8 operands; the oracle applies the same
    selection.  An output that no selected GEMM feeds must stay within the
    BF16 budget, so a GEMM quantised by mistake fails the test."""
    cfg = SMALL["mx_ragged"]
    inp = I.make_inputs(cfg)
    layer, out = run_layer(cfg, inp, mx_gemms=sel)
    mx = set(sel)
    fwd, bwd, wr = oracle_layer(cfg, inp, layer, mx)
    _check_routing(layer, inp, fwd)
    # the grouped GEMMs each output depends on
    feeds = {"GU": {"gemm1"}, "A": {"gemm1"}, "Y_perm": {"gemm1", "gemm2"},
             "out": {"gemm1", "gemm2"}, "dw": {"gemm1", "gemm2"}, "d_logits": {"gemm1", "gemm2"},
             "dH": {"gemm1", "dA"}, "dX_perm": {"gemm1", "dA", "dX"},
             "dx": {"gemm1", "dA", "dX"}, "dW2": {"gemm1", "dW2"},
             "dW13": {"gemm1", "dA", "dW13"}, "dY_perm": {"gemm1", "gemm2"}, "dWr": set()}
    check_layer(layer, out, inp, fwd, bwd, mx,
                lambda key: TOL_MXFP8 if feeds[key] & mx else TOL_BF16, wr)


def test_host_streamed_steps_match_plain_calls():
    """Copies overlapped with the neighbouring steps' compute (two device
    buffer sets, two copy streams) give each step exactly the outputs of a
    plain forward + backward on that step's inputs."""
    cfg = SMALL["ragged"]
    steps = 5
    inps = [I.make_inputs(cfg.with_(seed=cfg.seed + 100 * i)) for i in range(3)]
    base = inps[0]
    w13, w2 = base["w13"].cuda(), base["w2"].cuda()
    layer = ops.MoELayer(cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, router=cfg.router)
    pipe = ops.HostStreamedSteps(layer)
    host_in = [{n: inp[n].pin_memory() for n in pipe.names} for inp in inps]
    host_out = [{"out": torch.zeros(cfg.T, cfg.d, dtype=torch.bfloat16).pin_memory(),
                 "dx": torch.zeros(cfg.T, cfg.d, dtype=torch.bfloat16).pin_memory()}
                for _ in range(steps)]
    pipe.run(w13, w2, host_in, host_out, steps)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    ref = ops.MoELayer(cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, router=cfg.router)
    for i in range(steps):
        src = host_in[i % len(host_in)]
        g = {n: t.cuda() for n, t in src.items()}
        out = ref.forward(g["x"], w13, w2, logits=g.get("logits")).clone()
        dx = ref.backward(g["dout"], g["x"], w13, w2, logits=g.get("logits")).clone()
        torch.cuda.synchronize()
        assert torch.equal(host_out[i]["out"].view(torch.int16), out.cpu().view(torch.int16)), i
        assert torch.equal(host_out[i]["dx"].view(torch.int16), dx.cpu().view(torch.int16)), i


@pytest.mark.parametrize("name,recompute", [("mx_ragged", False), ("mx_proj", False),
                                            ("mx_ragged", True)])
def test_mx_keep_weights_is_bit_identical(name, recompute):
    """Weights quantised once per step (row- and column-wise from one read in
    the forward, the second layout kept for the backward) give the same
    bytes as quantising them again in the backward."""
    cfg = SMALL[name]
    inp = I.make_inputs(cfg)
    l1, o1 = run_layer(cfg, inp)
    ref = [t.clone() for t in (o1, l1.dx, l1.dw13, l1.dw2, l1.d_logits)]
    l2, o2 = run_layer(cfg, inp, mx_keep_weights=True, recompute=recompute)
    for a, b in zip(ref, (o2, l2.dx, l2.dw13, l2.dw2, l2.d_logits)):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
