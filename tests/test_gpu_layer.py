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

from ._util import TOL_BF16, TOL_MXFP8, assert_close, np64, npi, resolve_routing

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


@pytest.mark.parametrize("name", list(SMALL))
def test_layer_matches_oracle(name):
    cfg = SMALL[name]
    inp = I.make_inputs(cfg)
    layer, out = run_layer(cfg, inp)
    x, w13, w2, dout = (np64(inp[n]) for n in ("x", "w13", "w2", "dout"))
    wr = np64(inp["wr"]) if "wr" in inp else None
    mx = cfg.dtype == "mxfp8"
    st = layer.state
    if wr is not None:
        # routing is decided on the kernel's fp32 logits and on the oracle's
        # fp64 ones: compare the logits, then the selection (ambiguous
        # near-ties resolved as resolve_routing documents)
        ref_lg = om.router_logits(x, wr)
        assert_close(st.logits, ref_lg, 1e-5, "logits")
        ridx, _ = resolve_routing(ref_lg, npi(st.topk_idx), cfg.k)
        fwd = _forward_with_routing(x, w13, w2, cfg, ridx, ref_lg)
    else:
        fwd = om.layer_forward(x, w13, w2, cfg.k, logits32=inp["logits"].numpy(), mx=mx)
    bwd = om.layer_backward(fwd, dout, x, w13, w2, wr=wr, mx=mx)
    tol = TOL_MXFP8 if mx else TOL_BF16

    for key in ("topk_idx", "counts", "offsets", "dest_pos", "src_token"):
        assert np.array_equal(npi(getattr(st, key)), fwd[key]), key
    assert np.array_equal(st.x_perm.cpu().view(torch.int16).numpy(),
                          inp["x"].view(torch.int16).numpy()[fwd["src_token"]])
    assert_close(st.topk_w, fwd["topk_w"], 1e-5, "topk_w")
    for key, got in (("GU", st.gu), ("A", st.a), ("Y_perm", st.y_perm), ("out", out)):
        assert_close(got, fwd[key], tol, what=key)
    for key, got in (("dx", layer.dx), ("dW13", layer.dw13), ("dW2", layer.dw2),
                     ("d_logits", layer.d_logits)):
        assert_close(got, bwd[key], tol, what=key)
    if wr is not None:
        assert_close(layer.dw_r, bwd["dWr"], tol, what="dW_r")
    empty = np.nonzero(fwd["counts"] == 0)[0]
    for e in empty:
        assert torch.all(layer.dw13[e] == 0) and torch.all(layer.dw2[e] == 0)


@pytest.mark.parametrize("name", ["ragged", "one_token", "all_one_expert", "mx_ragged"])
def test_layer_matches_c_oracle(name):
    """The same layer against the independent C oracle (plain fp64 loops per
    token and selected expert); layers routed on given fp32 logits, so the
    selection is fixed by the inputs."""
    cfg = SMALL[name]
    inp = I.make_inputs(cfg)
    layer, out = run_layer(cfg, inp)
    x, w13, w2, dout = (np64(inp[n]) for n in ("x", "w13", "w2", "dout"))
    mx = cfg.dtype == "mxfp8"
    fwd = rc.layer_forward(x, w13, w2, cfg.k, logits32=inp["logits"].numpy(), mx=mx)
    bwd = rc.layer_backward(fwd, dout, x, w13, w2, mx=mx)
    tol = TOL_MXFP8 if mx else TOL_BF16
    st = layer.state
    for key in ("topk_idx", "counts", "offsets", "dest_pos", "src_token"):
        assert np.array_equal(npi(getattr(st, key)), fwd[key]), key
    assert_close(st.topk_w, fwd["topk_w"], 1e-5, "topk_w")
    for key, got in (("GU", st.gu), ("A", st.a), ("Y_perm", st.y_perm), ("out", out)):
        assert_close(got, fwd[key], tol, what=key)
    for key, got in (("dx", layer.dx), ("dW13", layer.dw13), ("dW2", layer.dw2),
                     ("d_logits", layer.d_logits)):
        assert_close(got, bwd[key], tol, what=key)


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
def test_recompute_is_bit_identical(name):
    """Recompute mode runs the same GEMM1 + SwiGLU kernels on the same saved
    x_perm again, so every output equals the stored-activation mode's bit for
    bit (and the layer keeps no [G | U] or A of its own)."""
    cfg = SMALL[name]
    inp = I.make_inputs(cfg)
    l1, o1 = run_layer(cfg, inp)
    ref = [t.clone() for t in (o1, l1.dx, l1.dw13, l1.dw2, l1.d_logits)]
    l2, o2 = run_layer(cfg, inp, recompute=True)
    assert l2.state.gu is None and l2.state.a is None
    for a, b in zip(ref, (o2, l2.dx, l2.dw13, l2.dw2, l2.d_logits)):
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
    x, w13, w2, dout = (np64(inp[n]) for n in ("x", "w13", "w2", "dout"))
    mx = set(sel)
    fwd = om.layer_forward(x, w13, w2, cfg.k, logits32=inp["logits"].numpy(), mx=mx)
    bwd = om.layer_backward(fwd, dout, x, w13, w2, mx=mx)
    st = layer.state
    # the grouped GEMMs each output depends on
    feeds = {"GU": {"gemm1"}, "A": {"gemm1"}, "Y_perm": {"gemm1", "gemm2"},
             "out": {"gemm1", "gemm2"}, "d_logits": {"gemm1", "gemm2"},
             "dx": {"gemm1", "dA", "dX"}, "dW2": {"gemm1", "dW2"},
             "dW13": {"gemm1", "dA", "dW13"}}
    got = {"GU": st.gu, "A": st.a, "Y_perm": st.y_perm, "out": out, "d_logits": layer.d_logits,
           "dx": layer.dx, "dW2": layer.dw2, "dW13": layer.dw13}
    for key, t in got.items():
        ref = fwd[key] if key in fwd else bwd[key]
        tol = TOL_MXFP8 if feeds[key] & mx else TOL_BF16
        assert_close(t, ref, tol, what=key)


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
