"""Parity at the full workload sizes, in the launch configuration bench.py
times (needs a B200).

The layer runs forward + backward on each workload at its full size.  The
oracle then checks:
  * routing, counts, offsets, row positions of every token, bit for bit;
  * the permutation property x_perm[dest_pos[t, i]] == x[t] for every row;
  * every routed row of every expert -- [G | U], A, Y_perm, dY_perm, dH,
    dX_perm -- stage by stage under the rule of tests/_parity.py, the oracle
    evaluating one expert at a time over all of its rows;
  * every token's out, dx, dw and d_logits, summed by the oracle from those
    rows;
  * the whole weight gradients dW13_e, dW2_e of sampled experts (the busiest,
    the lightest non-empty one and two more), and exact zeros for every empty
    expert.
Inputs are drawn on the GPU by the seeded generator, which is device
independent (test_generator_is_device_independent); the rows the oracle needs
are the generator's bytes, never a kernel's output.
"""
import numpy as np
import pytest
import torch

from oracle import moe as om
from routing_grouped_gemm_moe_b200 import inputs as I
from routing_grouped_gemm_moe_b200 import ops

from . import _parity as P
from ._parity import TOL_BF16, TOL_MXFP8
from ._util import assert_close, npi, resolve_routing

pytestmark = pytest.mark.gpu

WORKLOADS = ["fine", "pool_e8", "pool_e32", "pool_e128", "skewed", "large_bf16"]


def _f64(t):
    return t.detach().float().cpu().double().numpy()


def _run(cfg, dtype="bf16"):
    dev = torch.device("cuda")
    inp = I.make_inputs(cfg, device=dev)
    layer = ops.MoELayer(cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, router=cfg.router, dtype=dtype,
                         device=dev)
    lg, wr = inp.get("logits"), inp.get("wr")
    layer.forward(inp["x"], inp["w13"], inp["w2"], logits=lg, w_r=wr)
    layer.backward(inp["dout"], inp["x"], inp["w13"], inp["w2"], logits=lg, w_r=wr)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    return inp, layer


def _routing(cfg, inp, layer):
    """Oracle routing (router projection: validated against the device's fp32
    logits, near-ties resolved as resolve_routing documents), checked bit for
    bit together with the dispatch plan and the permutation property."""
    st = layer.state
    lg, wr = inp.get("logits"), inp.get("wr")
    if cfg.router == "logits":
        lg32 = I.make_logits(cfg).numpy()          # the generator's bytes, drawn on the CPU
        assert np.array_equal(lg32.view(np.int32), lg.cpu().numpy().view(np.int32))
        ridx, rw = om.router_topk(lg32, cfg.k)
    else:
        wl = om.router_logits(_f64(inp["x"]), _f64(wr))
        assert_close(st.logits, wl, 1e-5, "logits")
        ridx, _ = resolve_routing(wl, npi(st.topk_idx), cfg.k)
        rw = om.router_weights(wl.astype(np.float32), ridx)
    assert np.array_equal(npi(st.topk_idx), ridx)
    counts, offsets, dest, src = om.dispatch_plan(ridx, cfg.E)
    assert np.array_equal(npi(st.counts), counts)
    assert np.array_equal(npi(st.offsets), offsets)
    assert np.array_equal(npi(st.dest_pos), dest)
    assert np.array_equal(npi(st.src_token), src)
    d_t = st.dest_pos.long()
    for i in range(cfg.k):
        assert torch.equal(st.x_perm[d_t[:, i]].view(torch.int16), inp["x"].view(torch.int16))
    assert_close(st.topk_w, rw, 1e-5, "topk_w")
    return ridx, rw, counts, offsets, dest, src


def _ws(layer, cfg):
    """dX_perm, dH and dw from the layer workspace (the layout documented for
    moe_layer_bwd: status word, dispatch scratch, dY_perm reused for dX_perm,
    dH, dw; sub-buffers 256-byte aligned)."""
    al = lambda v: (v + 255) // 256 * 256  # noqa: E731
    M = cfg.T * cfg.k
    ws = layer.workspace
    o = 256 + al(ops.permute_workspace_bytes(cfg.T, cfg.E) - 256)
    dX = ws[o:o + M * cfg.d * 2].view(torch.bfloat16).view(M, cfg.d)
    o += al(M * cfg.d * 2)
    dH = ws[o:o + M * 2 * cfg.f * 2].view(torch.bfloat16).view(M, 2 * cfg.f)
    o += al(M * 2 * cfg.f * 2)
    dw = ws[o:o + cfg.T * cfg.k * 4].view(torch.float32).view(cfg.T, cfg.k)
    return dX, dH, dw


def _sampled(counts, seed, n=2):
    nz = np.nonzero(counts > 0)[0]
    busy = int(np.argmax(counts))
    light = int(nz[np.argmin(counts[nz])])
    rng = np.random.default_rng(seed)
    return sorted(set([busy, light] + rng.choice(nz, n, replace=False).tolist()))


@pytest.mark.parametrize("name", WORKLOADS)
def test_fullsize_layer(name):
    cfg = I.CONFIGS[name]
    inp, layer = _run(cfg)
    st = layer.state
    ridx, rw, counts, offsets, dest, src = _routing(cfg, inp, layer)
    dX_dev, dH_dev, dw_ws = _ws(layer, cfg)
    # dY_perm is overwritten by dX_perm inside the backward: the layer's own
    # combine-backward kernel is called again on the layer's own inputs (its
    # dw must be the layer's, bit for bit)
    dY_dev, dw_dev = ops.unpermute_combine_bwd(inp["dout"], st.y_perm, st.dest_pos, st.topk_w)
    torch.cuda.synchronize()
    assert torch.equal(dw_dev, dw_ws)

    T, d, k = cfg.T, cfg.d, cfg.k
    slot_of_row = np.empty(T * k, np.int64)
    slot_of_row[dest.reshape(-1)] = np.tile(np.arange(k), T)
    w_rows = rw[src, slot_of_row]
    dout = _f64(inp["dout"])
    out_acc = np.zeros((T, d))
    dx_acc = np.zeros((T, d))
    dw_acc = np.zeros((T, k))
    tally = P.Tally(TOL_BF16)
    dw_experts = _sampled(counts, cfg.seed)
    for e in range(cfg.E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 == r0:
            assert torch.all(layer.dw13[e] == 0) and torch.all(layer.dw2[e] == 0)
            continue
        rows = slice(r0, r1)
        tok = src[r0:r1].astype(np.int64)
        xp = _f64(inp["x"][torch.from_numpy(tok).cuda()])
        S = P.Stages(xp, _f64(inp["w13"][e:e + 1]), _f64(inp["w2"][e:e + 1]), [0, r1 - r0],
                     sink=tally)
        S.check_gu(st.gu[rows])
        S.check_a(st.a[rows])
        Y = S.check_y(st.y_perm[rows])
        S.check_dy(dY_dev[rows], w_rows[rows], dout[tok])
        S.check_dh(dH_dev[rows])
        dX = S.check_dx_perm(dX_dev[rows])
        if e in dw_experts:
            S.check_dw2(layer.dw2[e:e + 1])
            S.check_dw13(layer.dw13[e:e + 1])
        sl = slot_of_row[rows]
        out_acc[tok] += rw[tok, sl][:, None] * Y
        dw_acc[tok, sl] = np.sum(dout[tok] * Y, axis=1)
        dx_acc[tok] += dX
    tally.finish()
    # every token
    P.check(layer.out, P.candidates(out_acc), TOL_BF16, "out")
    P.check_f32(dw_ws, dw_acc, TOL_BF16, "dw")
    dl = om.router_backward(rw, dw_acc, ridx, cfg.E)
    P.check_f32(layer.d_logits, dl, TOL_BF16, "d_logits")
    if cfg.router == "proj":
        dx_r, dwr = om.router_proj_backward(_f64(inp["x"]), _f64(inp["wr"]), dl)
        dx_acc += dx_r
        P.check(layer.dw_r, P.candidates(dwr), TOL_BF16, "dW_r")
    P.check(layer.dx, P.candidates(dx_acc), TOL_BF16, "dx")


def test_fullsize_mxfp8_large():
    """The large workload with MXFP8 grouped GEMMs, at full size.  Routing and
    dispatch are checked for every token; every routed row of sampled experts
    (the busiest, the lightest and two more) is checked stage by stage --
    [G | U], A, Y, dY, dH, dX -- together with their dW13 and dW2, against
    the oracle's MXFP8 statement of that expert alone (row-wise blocks are
    local to a row, and column-wise blocks restart at the expert's first row,
    so the sub-problem quantises exactly the same blocks)."""
    cfg = I.CONFIGS["large"]
    inp, layer = _run(cfg, "mxfp8")
    st = layer.state
    ridx, rw, counts, offsets, dest, src = _routing(cfg, inp, layer)
    dX_dev, dH_dev, dw_ws = _ws(layer, cfg)
    dY_dev, dw_dev = ops.unpermute_combine_bwd(inp["dout"], st.y_perm, st.dest_pos, st.topk_w)
    torch.cuda.synchronize()
    assert torch.equal(dw_dev, dw_ws)
    T, k = cfg.T, cfg.k
    slot_of_row = np.empty(T * k, np.int64)
    slot_of_row[dest.reshape(-1)] = np.tile(np.arange(k), T)
    w_rows = rw[src, slot_of_row]
    tally = P.Tally(TOL_MXFP8)
    for e in _sampled(counts, cfg.seed):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        rows = slice(r0, r1)
        tok_t = torch.from_numpy(src[r0:r1].astype(np.int64)).cuda()
        S = P.Stages(_f64(inp["x"][tok_t]), _f64(inp["w13"][e:e + 1]), _f64(inp["w2"][e:e + 1]),
                     [0, r1 - r0], mx=True, sink=tally)
        S.check_gu(st.gu[rows])
        S.check_a(st.a[rows])
        S.check_y(st.y_perm[rows])
        S.check_dy(dY_dev[rows], w_rows[rows], _f64(inp["dout"][tok_t]))
        S.check_dh(dH_dev[rows])
        S.check_dx_perm(dX_dev[rows])
        S.check_dw2(layer.dw2[e:e + 1])
        S.check_dw13(layer.dw13[e:e + 1])
    tally.finish()
