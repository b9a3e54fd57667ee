"""Parity at the full workload sizes, in the launch configuration bench.py
times (needs a B200).

The layer runs forward + backward on each workload at its full size.  The
oracle then checks:
  * routing, counts, offsets, row positions of every token, bit for bit;
  * the permutation property x_perm[dest_pos[t, i]] == x[t] for every row;
  * sampled tokens end to end (GU, A, Y rows, out, dH rows, dx, topk_w,
    d_logits) by per-token evaluation without any dispatch;
  * whole weight gradients dW13_e, dW2_e of sampled experts (the busiest, a
    light one, and every empty expert, which must be exactly zero).
Inputs are drawn on the GPU by the seeded generator, which is device
independent (test_generator_is_device_independent); the slices the oracle
needs are the generator's bytes, never a kernel's output.
"""
import numpy as np
import pytest
import torch

from oracle import moe as om
from routing_grouped_gemm_moe_b200 import inputs as I
from routing_grouped_gemm_moe_b200 import ops

from ._util import (assert_close, bf16_roundings, dh_reference_candidates, np64, npi,
                    resolve_mx_dy, resolve_routing)

pytestmark = pytest.mark.gpu

WORKLOADS = ["fine", "pool_e8", "pool_e32", "pool_e128", "skewed", "large_bf16"]
N_TOKENS = {"large_bf16": 3, "skewed": 4}


def _f64(t):
    return t.detach().float().cpu().double().numpy()


@pytest.mark.parametrize("name", WORKLOADS)
def test_fullsize_layer(name):
    cfg = I.CONFIGS[name]
    dev = torch.device("cuda")
    inp = I.make_inputs(cfg, device=dev)
    layer = ops.MoELayer(cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, router=cfg.router, device=dev)
    lg, wr = inp.get("logits"), inp.get("wr")
    layer.forward(inp["x"], inp["w13"], inp["w2"], logits=lg, w_r=wr)
    layer.backward(inp["dout"], inp["x"], inp["w13"], inp["w2"], logits=lg, w_r=wr)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    st = layer.state

    # ---------------------------------------------------------- routing
    if cfg.router == "logits":
        lg32 = I.make_logits(cfg).numpy()          # the generator's bytes, drawn on the CPU
        assert np.array_equal(lg32.view(np.int32), lg.cpu().numpy().view(np.int32))
        ridx, rw = om.router_topk(lg32, cfg.k)
        wl = None
    else:
        wl = om.router_logits(_f64(inp["x"]), _f64(wr))
        assert_close(st.logits, wl, 1e-5, "logits")
        ridx, amb = resolve_routing(wl, npi(st.topk_idx), cfg.k)
        rw = om.router_weights(wl.astype(np.float32), ridx)
    assert np.array_equal(npi(st.topk_idx), ridx)
    counts, offsets, dest, src = om.dispatch_plan(ridx, cfg.E)
    assert np.array_equal(npi(st.counts), counts)
    assert np.array_equal(npi(st.offsets), offsets)
    assert np.array_equal(npi(st.dest_pos), dest)
    assert np.array_equal(npi(st.src_token), src)
    # permutation property on the device, every routed row
    d_t = st.dest_pos.long()
    for i in range(cfg.k):
        assert torch.equal(st.x_perm[d_t[:, i]].view(torch.int16), inp["x"].view(torch.int16))
    assert_close(st.topk_w, rw, 1e-5, "topk_w")

    # ---------------------------------------------------------- sampled tokens
    rng = np.random.default_rng(cfg.seed)
    n_tok = N_TOKENS.get(name, 8)
    toks = sorted(set([0, cfg.T - 1] + rng.choice(cfg.T, n_tok, replace=False).tolist()))[:n_tok]
    cache = {}

    def expert(e):
        if e not in cache:
            cache[e] = (_f64(inp["w13"][e]), _f64(inp["w2"][e]))
        return cache[e]

    ref = {k: [] for k in ("gu", "a", "y", "out", "dh", "dx", "dl")}
    got = {k: [] for k in ref}
    for t in toks:
        sel = ridx[t]
        w13s = np.stack([expert(int(e))[0] for e in sel])
        w2s = np.stack([expert(int(e))[1] for e in sel])
        xt = _f64(inp["x"][t])
        ft = om.token_forward(xt, w13s, w2s, rw[t])
        dxe, dw_t, dH_t, _ = om.token_backward(_f64(inp["dout"][t]), xt, w13s, w2s, rw[t], ft)
        dl_t = om.router_backward(rw[t:t + 1], dw_t[None], ridx[t:t + 1], cfg.E)[0]
        extra = 0.0
        if wr is not None:
            extra = dl_t @ _f64(wr).T
        pos = dest[t]
        ref["gu"].append(ft[2]); got["gu"].append(_f64(st.gu[pos]))
        ref["a"].append(ft[3]); got["a"].append(_f64(st.a[pos]))
        ref["y"].append(ft[1]); got["y"].append(_f64(st.y_perm[pos]))
        ref["out"].append(ft[0]); got["out"].append(_f64(layer.out[t]))
        # dH is elementwise in the stored bf16 G, U: where the exact G or U
        # sits on a bf16 rounding midpoint both roundings are correct, so each
        # element is compared with the closest of the oracle's candidates
        gdh = _f64(_dh_rows(layer, cfg, pos))
        dY_t = om.round_bf16(rw[t][:, None] * _f64(inp["dout"][t])[None, :])
        best = []
        for i in range(cfg.k):
            gu64 = om.expert_preactivation(xt, w13s[i])
            gn, ga = bf16_roundings(gu64[:cfg.f])
            un, ua = bf16_roundings(gu64[cfg.f:])
            dA = w2s[i].T @ dY_t[i]
            cands = [om.swiglu_backward(dA, g_, u_) for g_ in (gn, ga) for u_ in (un, ua)]
            dg = np.stack([om.round_bf16(c[0]) for c in cands])
            du = np.stack([om.round_bf16(c[1]) for c in cands])
            pick_g = dg[np.argmin(np.abs(dg - gdh[i, :cfg.f]), axis=0), np.arange(cfg.f)]
            pick_u = du[np.argmin(np.abs(du - gdh[i, cfg.f:]), axis=0), np.arange(cfg.f)]
            best.append(np.concatenate([pick_g, pick_u]))
        ref["dh"].append(np.stack(best)); got["dh"].append(gdh)
        ref["dx"].append(om.round_bf16(dxe + extra)); got["dx"].append(_f64(layer.dx[t]))
        ref["dl"].append(dl_t); got["dl"].append(_f64(layer.d_logits[t]))
    for key in ref:
        assert_close(np.stack(got[key]), np.stack(ref[key]), what=key,
                     bf16_storage=(key != "dl"))

    # ---------------------------------------------------------- whole experts
    empty = np.nonzero(counts == 0)[0].tolist()
    busy = int(np.argmax(counts))
    light = int(np.argmin(np.where(counts > 0, counts, np.iinfo(np.int64).max)))
    for e in empty:
        assert torch.all(layer.dw13[e] == 0) and torch.all(layer.dw2[e] == 0)
    for e in sorted(set([busy, light])):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        rows = src[r0:r1]
        slot = np.argmax(ridx[rows] == e, axis=1)
        wrow = rw[rows, slot]
        xe = _f64(inp["x"][torch.from_numpy(rows.astype(np.int64)).cuda()])
        de = _f64(inp["dout"][torch.from_numpy(rows.astype(np.int64)).cuda()])
        w13e, w2e = expert(e)
        sub = [0, r1 - r0]
        GU, A, _ = om.expert_forward(xe, w13e[None], w2e[None], sub)
        dY = om.round_bf16(wrow[:, None] * de)
        _, dW2, _, dW13 = om.expert_backward(dY, GU, A, xe, w13e[None], w2e[None], sub)
        assert_close(layer.dw2[e], dW2[0], what=f"dW2[{e}]")
        assert_close(layer.dw13[e], dW13[0], what=f"dW13[{e}]")


def _dh_rows(layer, cfg, pos):
    """dH rows of the routed positions `pos`, read from the layer workspace
    (the layout documented for moe_layer_bwd: status, dispatch scratch, dY/dX,
    dH, dw; sub-buffers 256-byte aligned)."""
    al = lambda v: (v + 255) // 256 * 256  # noqa: E731
    M = cfg.T * cfg.k
    ntasks = (cfg.T + 127) // 128
    off = 256 + al(ntasks * cfg.E * 4) + al(M * cfg.d * 2)
    dh = layer.workspace[off:off + M * 2 * cfg.f * 2].view(torch.bfloat16).view(M, 2 * cfg.f)
    return dh[torch.from_numpy(np.asarray(pos, np.int64)).cuda()]


def test_fullsize_mxfp8_large():
    """The large workload with MXFP8 grouped GEMMs, at full size.  Routing and
    dispatch are checked for every token; GU, A, Y, dH, dX rows and dW13, dW2
    of sampled experts are checked against the oracle's MXFP8 emulation of
    that expert alone (row-wise blocks are local to a row, and column-wise
    blocks restart at the expert's first row, so the sub-problem quantises
    exactly the same blocks)."""
    from ._util import TOL_MXFP8
    cfg = I.CONFIGS["large"]
    dev = torch.device("cuda")
    inp = I.make_inputs(cfg, device=dev)
    layer = ops.MoELayer(cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, router=cfg.router, dtype="mxfp8",
                         device=dev)
    lg = inp["logits"]
    layer.forward(inp["x"], inp["w13"], inp["w2"], logits=lg)
    layer.backward(inp["dout"], inp["x"], inp["w13"], inp["w2"], logits=lg)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    st = layer.state
    lg32 = I.make_logits(cfg).numpy()
    ridx, rw = om.router_topk(lg32, cfg.k)
    assert np.array_equal(npi(st.topk_idx), ridx)
    counts, offsets, dest, src = om.dispatch_plan(ridx, cfg.E)
    assert np.array_equal(npi(st.offsets), offsets)
    assert np.array_equal(npi(st.dest_pos), dest)
    M = cfg.T * cfg.k
    al = lambda v: (v + 255) // 256 * 256  # noqa: E731
    off_dy = 256 + al(((cfg.T + 127) // 128) * cfg.E * 4)
    dX = layer.workspace[off_dy:off_dy + M * cfg.d * 2].view(torch.bfloat16).view(M, cfg.d)
    busy = int(np.argmax(counts))
    light = int(np.argmin(counts))
    for e in sorted(set([busy, light])):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        rows = src[r0:r1]
        rows_t = torch.from_numpy(rows.astype(np.int64)).cuda()
        slot = np.argmax(ridx[rows] == e, axis=1)
        wrow = rw[rows, slot]
        xe = _f64(inp["x"][rows_t])
        de = _f64(inp["dout"][rows_t])
        w13e, w2e = _f64(inp["w13"][e]), _f64(inp["w2"][e])
        sub = [0, r1 - r0]
        pre = np.zeros((r1 - r0, 2 * cfg.f))
        GU, A, Y = om.expert_forward(xe, w13e[None], w2e[None], sub, mx=True, preact=pre)
        gdh = _f64(_dh_rows(layer, cfg, np.arange(r0, r1)))
        # the correct bf16 roundings of w * dOut, resolved per row (see
        # resolve_mx_dy); W2_e decoded from its column-wise MXFP8 blocks
        w2q = om.mx_colwise_decoded(w2e, [0, cfg.d])
        dY = resolve_mx_dy(wrow, de, pre, gdh, w2q, cfg.f)
        dA = np.zeros((r1 - r0, cfg.f))
        dH, dW2, dXe, dW13 = om.expert_backward(dY, GU, A, xe, w13e[None], w2e[None], sub, mx=True,
                                                dA_out=dA)
        sl = slice(r0, r1)
        assert_close(st.gu[sl], GU, TOL_MXFP8, f"GU[{e}]")
        assert_close(st.a[sl], A, TOL_MXFP8, f"A[{e}]")
        assert_close(st.y_perm[sl], Y, TOL_MXFP8, f"Y[{e}]")
        # dH is elementwise in the stored bf16 G, U: accept either correct
        # rounding of a G or U that sits on a bf16 rounding midpoint
        assert_close(gdh, dh_reference_candidates(dA, pre, gdh, cfg.f), TOL_MXFP8, f"dH[{e}]",
                     bf16_storage=True)
        assert_close(dX[sl], dXe, TOL_MXFP8, f"dX[{e}]")
        assert_close(layer.dw2[e], dW2[0], TOL_MXFP8, f"dW2[{e}]")
        assert_close(layer.dw13[e], dW13[0], TOL_MXFP8, f"dW13[{e}]")
