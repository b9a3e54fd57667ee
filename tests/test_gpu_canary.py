"""Canary regions: every entry point writes its outputs and nothing next to
them (needs a B200).

Each output is carved out of a larger device buffer whose guard regions, in
front of and behind it, hold a byte pattern; after the call (ragged expert
groups, an empty expert, tails shorter than a tile) the guards must be
unchanged and the outputs must be right.  This stands in for a memory
checker, which is not available on the GPUs these tests run on.
"""
import numpy as np
import pytest
import torch

from oracle import moe as om
from routing_grouped_gemm_moe_b200 import _lib as L
from routing_grouped_gemm_moe_b200 import inputs as I
from routing_grouped_gemm_moe_b200 import ops

from ._parity import TOL_BF16, check
from ._parity import candidates
from ._util import np64, npi

pytestmark = pytest.mark.gpu

GUARD = 4096        # bytes on each side (keeps 16-byte alignment)
PATTERN = 0x5A


class Guarded:
    """A device tensor of `shape` / `dtype` with guard bytes on both sides."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.nbytes = n
        self.buf = torch.full((GUARD + n + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.t = self.buf[GUARD:GUARD + n].view(dtype).view(*shape)

    def intact(self) -> bool:
        head = self.buf[:GUARD]
        tail = self.buf[GUARD + self.nbytes:]
        return bool(torch.all(head == PATTERN)) and bool(torch.all(tail == PATTERN))


def _topk(T, E, k, seed, empty=0):
    lg = I.normal_f32(I.stream_key(seed, 3), (T, E))
    if empty:
        lg[:, E - empty:] = -1e4
    idx, _ = om.router_topk(lg.numpy(), k)
    return idx


def _offsets(counts):
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)


@pytest.mark.parametrize("mx", [False, True])
def test_dispatch_writes_only_its_outputs(mx):
    T, E, k = 1000, 32, 4
    d = 1056 if mx else 136
    idx = _topk(T, E, k, 41, empty=3)
    x = I.normal_bf16(I.stream_key(T, d), (T, d), 1.0)
    M = T * k
    counts, offsets = Guarded((E,), torch.int32), Guarded((E + 1,), torch.int32)
    dest, src = Guarded((T, k), torch.int32), Guarded((M,), torch.int32)
    xp = Guarded((M, d), torch.bfloat16)
    codes, scales = Guarded((M, d), torch.uint8), Guarded((M, d // 32), torch.uint8)
    ws = torch.zeros(ops.permute_workspace_bytes(T, E), dtype=torch.uint8, device="cuda")
    x_d, idx_d = x.cuda(), torch.from_numpy(idx.astype(np.int32)).cuda()  # alive until the sync
    args = [ops._p(x_d), ops._p(idx_d), T, d, E, k,
            ops._p(counts.t), ops._p(offsets.t), ops._p(dest.t), ops._p(src.t), ops._p(xp.t)]
    if mx:
        L.call("moe_permute_rows_mxfp8", *args, ops._p(codes.t), ops._p(scales.t), ops._p(ws),
               ws.numel(), ops._s())
    else:
        L.call("moe_permute_rows", *args, ops._p(ws), ws.numel(), ops._s())
    torch.cuda.synchronize()
    outs = [counts, offsets, dest, src, xp] + ([codes, scales] if mx else [])
    assert all(g.intact() for g in outs)
    rc, ro, rd, rs = om.dispatch_plan(idx, E)
    assert np.array_equal(npi(dest.t), rd) and np.array_equal(npi(offsets.t), ro)
    assert np.array_equal(xp.t.cpu().view(torch.int16).numpy(),
                          om.dispatch_rows(x.view(torch.int16).numpy(), rs))


@pytest.mark.parametrize("N,K,epi", [(320, 256, L.EPI_NONE), (256, 192, L.EPI_NONE),
                                     (384, 128, L.EPI_SWIGLU)])
def test_grouped_gemm_ragged_m_writes_only_its_outputs(N, K, epi):
    counts = [70, 0, 200, 1, 64, 129, 300]
    E, off = len(counts), _offsets(counts)
    Mt = int(off[-1])
    a = I.normal_bf16(I.stream_key(N, K), (Mt, K), 1.0)
    b = I.normal_bf16(I.stream_key(K, N), (E, N, K), 0.05)
    c = Guarded((Mt, N), torch.bfloat16)
    aux = Guarded((Mt, N // 2), torch.bfloat16)
    a_d, b_d, off_d = a.cuda(), b.cuda(), torch.from_numpy(off.astype(np.int32)).cuda()
    ops.grouped_gemm(L.GG_RAGGED_M, a_d, b_d, off_d, E, N=N, K=K, epilogue=epi, c=c.t,
                     aux=aux.t if epi == L.EPI_SWIGLU else None)
    torch.cuda.synchronize()
    assert c.intact() and aux.intact()
    ref = om.grouped_gemm_ragged_m(np64(a), np64(b), off)
    check(c.t, candidates(ref), TOL_BF16, "C")


@pytest.mark.parametrize("M,N", [(384, 320), (128, 136)])
def test_grouped_gemm_ragged_k_writes_only_its_outputs(M, N):
    counts = [70, 0, 200, 1, 64, 129, 48]
    E, off = len(counts), _offsets(counts)
    Mt = int(off[-1])
    a = I.normal_bf16(I.stream_key(M, N + 1), (Mt, M), 1.0)
    b = I.normal_bf16(I.stream_key(N, M + 1), (Mt, N), 1.0)
    c = Guarded((E, M, N), torch.bfloat16)
    a_d, b_d, off_d = a.cuda(), b.cuda(), torch.from_numpy(off.astype(np.int32)).cuda()
    ops.grouped_gemm(L.GG_RAGGED_K, a_d, b_d, off_d, E, M=M, N=N, c=c.t)
    torch.cuda.synchronize()
    assert c.intact()
    ref = om.grouped_gemm_ragged_k(np64(a), np64(b), off)
    assert torch.all(c.t[1] == 0)
    for e in (0, 2, 5):
        check(c.t[e], candidates(ref[e]), TOL_BF16, f"C[{e}]")


def test_combine_and_its_backward_write_only_their_outputs():
    T, E, k, d = 600, 16, 4, 200
    idx = _topk(T, E, k, 43)
    lg = I.normal_f32(I.stream_key(43, 3), (T, E))
    w = om.router_weights(lg.numpy(), idx).astype(np.float32)
    _, _, dest, _ = om.dispatch_plan(idx, E)
    y = I.normal_bf16(I.stream_key(43, 5), (T * k, d), 1.0).cuda()
    dout = I.normal_bf16(I.stream_key(43, 6), (T, d), 1.0).cuda()
    dest_t, w_t = torch.from_numpy(dest).cuda(), torch.from_numpy(w).cuda()
    out = Guarded((T, d), torch.bfloat16)
    dy, dw = Guarded((T * k, d), torch.bfloat16), Guarded((T, k), torch.float32)
    L.call("moe_unpermute_combine", ops._p(y), ops._p(dest_t), ops._p(w_t), T, d, k, ops._p(out.t),
           ops._s())
    L.call("moe_unpermute_combine_bwd", ops._p(dout), ops._p(y), ops._p(dest_t), ops._p(w_t), T, d, k,
           ops._p(dy.t), ops._p(dw.t), ops._s())
    torch.cuda.synchronize()
    assert out.intact() and dy.intact() and dw.intact()
    check(out.t, candidates(om.combine(np64(y), dest, w, bf16=False)), TOL_BF16, "out")


def test_mxfp8_quantisers_write_only_their_outputs():
    counts = [40, 0, 24, 1, 100, 33]
    off = _offsets(counts)
    rows, cols = int(off[-1]), 320
    x = I.normal_bf16(I.stream_key(rows, cols), (rows, cols), 1.0).cuda()
    ng = len(counts)
    rc, rs = Guarded((rows, cols), torch.uint8), Guarded((rows, cols // 32), torch.uint8)
    cc, cs = Guarded((rows, cols), torch.uint8), Guarded((rows // 32 + ng, cols), torch.uint8)
    offs = torch.from_numpy(off.astype(np.int32)).cuda()
    L.call("mxfp8_quantize_rowcol", ops._p(x), rows, cols, ops._p(offs), ng, ops._p(rc.t), ops._p(rs.t),
           ops._p(cc.t), ops._p(cs.t), ops._s())
    torch.cuda.synchronize()
    assert all(g.intact() for g in (rc, rs, cc, cs))
    ref_c, ref_s = om.mx_rowwise(np64(x))
    assert np.array_equal(rc.t.cpu().numpy(), ref_c) and np.array_equal(rs.t.cpu().numpy(), ref_s)


def test_mxfp8_quantisers_with_offsets_that_go_down():
    """Group offsets that go down ([0, R, 0, R]) would size more column-wise
    blocks than the scales buffer (rows/32 + ngroups rows) holds; the kernel
    takes the running maximum ([0, R, R, R]) instead, so the guards stay
    intact and the result is the oracle's for those offsets."""
    rows, cols = 160, 64
    bad = np.array([0, rows, 0, rows], np.int64)
    eff = np.maximum.accumulate(bad)
    ng = len(bad) - 1
    x = I.normal_bf16(I.stream_key(rows, 3 * cols), (rows, cols), 1.0).cuda()
    offs = torch.from_numpy(bad.astype(np.int32)).cuda()
    ref_c, ref_s, _ = om.mx_colwise_grouped(np64(x), eff)
    cc, cs = Guarded((rows, cols), torch.uint8), Guarded((rows // 32 + ng, cols), torch.uint8)
    L.call("mxfp8_quantize", ops._p(x), rows, cols, 0, ops._p(offs), ng, ops._p(cc.t),
           ops._p(cs.t), None, ops._s())
    torch.cuda.synchronize()
    assert cc.intact() and cs.intact()
    assert np.array_equal(cc.t.cpu().numpy(), ref_c)
    assert np.array_equal(cs.t.cpu().numpy()[:ref_s.shape[0]], ref_s)
    rc, rs = Guarded((rows, cols), torch.uint8), Guarded((rows, cols // 32), torch.uint8)
    cc2, cs2 = Guarded((rows, cols), torch.uint8), Guarded((rows // 32 + ng, cols), torch.uint8)
    L.call("mxfp8_quantize_rowcol", ops._p(x), rows, cols, ops._p(offs), ng, ops._p(rc.t),
           ops._p(rs.t), ops._p(cc2.t), ops._p(cs2.t), ops._s())
    torch.cuda.synchronize()
    assert all(g.intact() for g in (rc, rs, cc2, cs2))
    assert torch.equal(cc2.t, cc.t) and torch.equal(cs2.t, cs.t)


@pytest.mark.parametrize("dtype", ["bf16", "mxfp8"])
def test_layer_writes_only_its_outputs(dtype):
    cfg = I.LayerConfig("canary", T=300, d=256, E=6, k=2, f=384, logits="zipf", n_empty=1,
                        zipf_s=0.8, dtype=dtype, seed=77)
    inp = I.make_inputs(cfg)
    g = {n: t.cuda() for n, t in inp.items()}
    layer = ops.MoELayer(cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, router=cfg.router, dtype=dtype)
    out, dx = Guarded((cfg.T, cfg.d), torch.bfloat16), Guarded((cfg.T, cfg.d), torch.bfloat16)
    layer.forward(g["x"], g["w13"], g["w2"], logits=g["logits"], out=out.t)
    layer.backward(g["dout"], g["x"], g["w13"], g["w2"], logits=g["logits"], dx=dx.t)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    assert out.intact() and dx.intact()
    # the same results as the layer's own buffers
    ref = ops.MoELayer(cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, router=cfg.router, dtype=dtype)
    o2 = ref.forward(g["x"], g["w13"], g["w2"], logits=g["logits"])
    ref.backward(g["dout"], g["x"], g["w13"], g["w2"], logits=g["logits"])
    torch.cuda.synchronize()
    assert torch.equal(out.t.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(dx.t.view(torch.int16), ref.dx.view(torch.int16))
