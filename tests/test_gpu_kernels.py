"""Parity of each CUDA entry point against the CPU oracle (needs a B200).

Integer outputs (indices, counts, offsets, row positions, copied rows, MXFP8
codes and scales) must match bit for bit; float outputs must satisfy
max|gpu - oracle| <= 2e-2 * RMS(oracle).  Inputs come from the seeded
generator; nothing compared here is produced by the CUDA path on both sides.
"""
import numpy as np
import pytest
import torch

from oracle import moe as om
from oracle import numerics as nm
from routing_grouped_gemm_moe_b200 import _lib as L
from routing_grouped_gemm_moe_b200 import inputs as I
from routing_grouped_gemm_moe_b200 import ops

from ._parity import TOL_BF16, check
from ._parity import candidates
from ._util import assert_close, bf16_cuda, np64, npi

pytestmark = pytest.mark.gpu


def _bf16(key, shape, std=1.0):
    return I.normal_bf16(key, shape, std)


def _offsets(counts):
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)


# ------------------------------------------------------------------ router

@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (1000, 8, 2), (777, 32, 4), (513, 64, 8),
                                   (300, 128, 8), (64, 1024, 32), (100, 5, 5), (257, 256, 8),
                                   (333, 130, 6), (50, 200, 1), (129, 300, 8), (70, 64, 12),
                                   (4100, 128, 8)])
def test_router_topk_bit_exact(T, E, k):
    lg = I.normal_f32(I.stream_key(T + E, 11), (T, E))
    lg[::7, 1] = lg[::7, 0]                 # exact ties
    lg[::11, 2] = -0.0
    lg[::11, 3] = 0.0
    idx, w = ops.router_topk(lg.cuda(), k)
    ridx, rw = om.router_topk(lg.numpy(), k)
    assert np.array_equal(npi(idx), ridx)
    assert np.max(np.abs(np64(w) - rw)) < 2e-6


@pytest.mark.parametrize("E,k", [(32, 2), (32, 8), (64, 4), (128, 2), (128, 8)])
def test_router_topk_heavy_ties(E, k):
    """Many equal logits (values on a 0.5 grid, constant rows, -0 next to
    +0): the selection order is still (value descending, index ascending)."""
    T = 700
    lg = I.normal_f32(I.stream_key(E, k), (T, E))
    lg[::3] = torch.round(lg[::3] * 2) / 2
    lg[::17] = 1.0
    lg[::11, 5] = -0.0
    lg[::11, 6] = 0.0
    idx, w = ops.router_topk(lg.cuda(), k)
    ridx, rw = om.router_topk(lg.numpy(), k)
    assert np.array_equal(npi(idx), ridx)
    assert np.max(np.abs(np64(w) - rw)) < 2e-6


def test_router_proj_and_topk():
    cfg = I.CONFIGS["tiny"]
    x = I.make_x(cfg)
    wr = I.make_wr(cfg)
    lg, idx, w = ops.router_topk_proj(x.cuda(), wr.cuda(), cfg.k)
    ref = om.router_logits(np64(x), np64(wr))
    assert_close(lg, ref, 1e-5, "logits")
    # selection compared on the same fp32 values the kernel selected from
    ridx, rw = om.router_topk(lg.cpu().numpy(), cfg.k)
    assert np.array_equal(npi(idx), ridx)
    assert np.max(np.abs(np64(w) - rw)) < 2e-6


@pytest.mark.parametrize("T,E,k", [(333, 16, 3), (300, 256, 8), (129, 130, 6), (64, 12, 12)])
def test_router_bwd(T, E, k):
    lg = I.normal_f32(I.stream_key(5, 1), (T, E))
    idx, w = om.router_topk(lg.numpy(), k)
    dw = I.normal_f32(I.stream_key(5, 2), (T, k)).numpy()
    w32 = w.astype(np.float32)
    dl = ops.router_bwd(torch.from_numpy(idx).cuda(), torch.from_numpy(w32).cuda(),
                        torch.from_numpy(dw).cuda(), E)
    ref = om.router_backward(w32, dw, idx, E)
    assert_close(dl, ref, 1e-5, "d_logits")
    mask = ref == 0
    assert np.all(np64(dl)[mask] == 0)


def test_router_proj_bwd():
    T, d, E = 200, 96, 24
    x = _bf16(I.stream_key(6, 1), (T, d))
    dl = I.normal_f32(I.stream_key(6, 2), (T, E))
    got = ops.router_proj_bwd(x.cuda(), dl.cuda())
    ref = np64(x).T @ dl.double().numpy()
    check(got, candidates(ref), 1e-2, "dW_r")


# ------------------------------------------------------------------ dispatch

def _random_topk(T, E, k, seed, skew=False, force_empty=0):
    lg = I.normal_f32(I.stream_key(seed, 3), (T, E))
    if skew:
        lg = lg + torch.log(torch.arange(1, E + 1, dtype=torch.float32)) * -1.5
    if force_empty:
        lg[:, E - force_empty:] = -1e4
    idx, _ = om.router_topk(lg.numpy(), k)
    return idx


@pytest.mark.parametrize("T,d,E,k,skew,empty", [
    (1, 8, 4, 1, False, 0), (129, 64, 8, 2, False, 0), (1000, 136, 32, 4, True, 3),
    (4096, 256, 128, 8, False, 0), (300, 32, 1024, 3, False, 0), (257, 16, 6, 1, True, 2),
    (200, 48, 1, 1, False, 0)])
def test_permute_rows_bit_exact(T, d, E, k, skew, empty):
    idx = _random_topk(T, E, k, T + d, skew, empty)
    x = _bf16(I.stream_key(T, d), (T, d))
    counts, offsets, dest, src, xp, ws = ops.permute_rows(x.cuda(), torch.from_numpy(idx.astype(np.int32)).cuda(), E)
    rc, ro, rd, rs = om.dispatch_plan(idx, E)
    assert np.array_equal(npi(counts), rc)
    assert np.array_equal(npi(offsets), ro)
    assert np.array_equal(npi(dest), rd)
    assert np.array_equal(npi(src), rs)
    ref_xp = om.dispatch_rows(x.view(torch.int16).numpy(), rs)
    assert np.array_equal(xp.cpu().view(torch.int16).numpy(), ref_xp)
    assert int(ws[:4].view(torch.int32).item()) == 0


@pytest.mark.parametrize("T,d,E,k,skew,empty", [
    (1, 32, 4, 1, False, 0), (129, 64, 8, 2, False, 0), (1000, 1056, 32, 4, True, 3),
    (300, 2080, 16, 3, False, 0)])
def test_permute_rows_mxfp8_bit_exact(T, d, E, k, skew, empty):
    """The dispatch that also writes the row-wise MXFP8 encoding of the routed
    rows (d = 1056, 2080: a 1024-value chunk of the row loop plus a tail)."""
    idx = _random_topk(T, E, k, T + 3 * d, skew, empty)
    xs = I.normal_bf16(I.stream_key(T, d + 1), (T, d), 1.0).float()
    xs[0, :32] = 0.0                                  # all-zero block
    if T > 1:
        xs[1, 32:64] *= 2.0 ** -120                   # tiny block (clamped scale)
        xs[1, 0:32] *= 300.0                          # large values
    x = xs.to(torch.bfloat16)
    counts, offsets, dest, src, xp, codes, scales = ops.permute_rows_mxfp8(
        x.cuda(), torch.from_numpy(idx.astype(np.int32)).cuda(), E)
    rc, ro, rd, rs = om.dispatch_plan(idx, E)
    assert np.array_equal(npi(dest), rd) and np.array_equal(npi(src), rs)
    ref_xp = om.dispatch_rows(x.view(torch.int16).numpy(), rs)
    assert np.array_equal(xp.cpu().view(torch.int16).numpy(), ref_xp)
    ref_c, ref_s = om.mx_rowwise(np64(xp))
    assert np.array_equal(codes.cpu().numpy(), ref_c)
    assert np.array_equal(scales.cpu().numpy(), ref_s)


def test_permute_rejects_out_of_range_expert_without_fault():
    T, d, E, k = 64, 16, 4, 2
    idx = _random_topk(T, E, k, 9)
    idx[5, 1] = E + 3                      # corrupted index
    x = _bf16(I.stream_key(1, 1), (T, d))
    counts, offsets, dest, src, xp, ws = ops.permute_rows(x.cuda(), torch.from_numpy(idx.astype(np.int32)).cuda(), E)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) & (1 << 5)   # MOE_ERR_DEVICE_BOUNDS
    assert int(npi(dest)[5, 1]) == -1
    assert int(npi(counts).sum()) == T * k - 1


# ------------------------------------------------------------------ grouped GEMM

# expert row counts: partial and full 256-row (CTA pair) and 128-row tiles
RAGGED = [130, 0, 257, 1, 128, 64, 600, 384]


@pytest.mark.parametrize("N,K,b_mn", [(384, 192, False), (384, 192, True), (128, 64, False),
                                      (136, 200, True), (256, 1024, False)])
def test_grouped_gemm_ragged_m(N, K, b_mn):
    E = len(RAGGED)
    off = _offsets(RAGGED)
    Mt = int(off[-1]) + 5                  # trailing rows outside every group
    a = _bf16(I.stream_key(N, K), (Mt, K))
    b = _bf16(I.stream_key(K, N), (E, K, N) if b_mn else (E, N, K), 0.05)
    c = torch.full((Mt, N), 7.0, dtype=torch.bfloat16, device="cuda")
    ops.grouped_gemm(L.GG_RAGGED_M, a.cuda(), b.cuda(), torch.from_numpy(off.astype(np.int32)).cuda(),
                     E, N=N, K=K, b_mn_major=b_mn, c=c)
    ref = om.grouped_gemm_ragged_m(np64(a), np64(b), off, b_mn_major=b_mn)
    got = np64(c)
    check(got[:off[-1]], candidates(ref[:off[-1]]), TOL_BF16, "C")
    assert np.all(got[off[-1]:] == 7.0)    # rows outside the groups untouched


@pytest.mark.parametrize("f,K", [(320, 256), (128, 64), (1024, 128)])
def test_grouped_gemm_swiglu_epilogue(f, K):
    E = len(RAGGED)
    off = _offsets(RAGGED)
    Mt = int(off[-1])
    a = _bf16(I.stream_key(f, 1), (Mt, K))
    b = _bf16(I.stream_key(f, 2), (E, 2 * f, K), 0.05)
    gu, act = ops.grouped_gemm(L.GG_RAGGED_M, a.cuda(), b.cuda(),
                               torch.from_numpy(off.astype(np.int32)).cuda(), E, N=2 * f, K=K,
                               epilogue=L.EPI_SWIGLU)
    ref = om.grouped_gemm_ragged_m(np64(a), np64(b), off)
    check(gu, candidates(ref), TOL_BF16, "GU")
    check(act, candidates(om.silu(ref[:, :f]) * ref[:, f:]), TOL_BF16, "A")


@pytest.mark.parametrize("f,K,b_mn", [(320, 192, True), (256, 256, False), (128, 64, True)])
def test_grouped_gemm_swiglu_bwd_epilogue(f, K, b_mn):
    E = len(RAGGED)
    off = _offsets(RAGGED)
    Mt = int(off[-1])
    a = _bf16(I.stream_key(f, 3), (Mt, K))
    b = _bf16(I.stream_key(f, 4), (E, K, f) if b_mn else (E, f, K), 0.05)
    gu = _bf16(I.stream_key(f, 5), (Mt, 2 * f))
    dh = ops.grouped_gemm(L.GG_RAGGED_M, a.cuda(), b.cuda(), torch.from_numpy(off.astype(np.int32)).cuda(),
                          E, N=f, K=K, b_mn_major=b_mn, epilogue=L.EPI_SWIGLU_BWD, gu=gu.cuda())
    dA = om.grouped_gemm_ragged_m(np64(a), np64(b), off, b_mn_major=b_mn)
    g = np64(gu)
    dG, dU = om.swiglu_backward(dA, g[:, :f], g[:, f:])
    check(np64(dh)[:, :f], candidates(dG), TOL_BF16, "dG")
    check(np64(dh)[:, f:], candidates(dU), TOL_BF16, "dU")


# M >= 256 and N >= 256 run on CTA pairs (256 x 256 tiles; 384 x 320: tail
# tiles in both directions, K tails of 70, 1, 64, 129 and 200 rows, and tails
# of 48 and 16 rows that end exactly on an MMA's 16-row K slice)
@pytest.mark.parametrize("kmaps", [True, False], ids=["expert_maps", "smem_zeroing"])
@pytest.mark.parametrize("M,N,counts", [(192, 320, [70, 0, 200, 1, 64, 129]),
                                        (128, 128, [0, 0, 33]), (256, 512, [1000, 24, 0, 300]),
                                        (64, 136, [5]), (384, 320, [70, 0, 200, 1, 64, 129, 48, 16])])
def test_grouped_gemm_ragged_k(M, N, counts, kmaps):
    E = len(counts)
    off = _offsets(counts)
    Mt = int(off[-1])
    a = _bf16(I.stream_key(M, N), (Mt, M))
    b = _bf16(I.stream_key(N, M), (Mt, N))
    c = torch.full((E, M, N), 3.0, dtype=torch.bfloat16, device="cuda")
    ops.grouped_gemm(L.GG_RAGGED_K, a.cuda(), b.cuda(), torch.from_numpy(off.astype(np.int32)).cuda(),
                     E, M=M, N=N, c=c, kmaps=kmaps)
    ref = om.grouped_gemm_ragged_k(np64(a), np64(b), off)
    got = np64(c)
    for e in range(E):
        if counts[e] == 0:
            assert np.all(got[e] == 0), "empty expert must give exact zeros"
        else:
            check(got[e], candidates(ref[e]), TOL_BF16, f"C[{e}]")


# ------------------------------------------------------------------ combine / swiglu

# d = 4096 / 4104, k = 8: a token's rows fill 64 KB, so the bulk engine has
# only three stages
@pytest.mark.parametrize("T,d,E,k", [(1, 8, 2, 2), (517, 136, 8, 2), (300, 512, 64, 8),
                                     (301, 4096, 32, 8), (97, 4104, 16, 8)])
def test_combine_and_backward(T, d, E, k):
    idx = _random_topk(T, E, k, T * 3 + d)
    lg = I.normal_f32(I.stream_key(T, 9), (T, E)).numpy()
    _, w = om.router_topk(lg, k)
    w32 = w.astype(np.float32)
    _, off, dest, _ = om.dispatch_plan(idx, E)
    y = _bf16(I.stream_key(T, 7), (T * k, d))
    dout = _bf16(I.stream_key(T, 8), (T, d))
    dest_t = torch.from_numpy(dest.astype(np.int32)).cuda()
    w_t = torch.from_numpy(w32).cuda()
    out = ops.unpermute_combine(y.cuda(), dest_t, w_t)
    check(out, candidates(om.combine(np64(y), dest, w32, bf16=False)), TOL_BF16, "out")
    dy, dw = ops.unpermute_combine_bwd(dout.cuda(), y.cuda(), dest_t, w_t)
    rdy, rdw = om.combine_backward(np64(dout), np64(y), dest, w32, bf16=False)
    check(dy, candidates(rdy), TOL_BF16, "dY_perm")
    assert_close(dw, rdw, 1e-4, what="dw")
    dxp = _bf16(I.stream_key(T, 10), (T * k, d))
    dx = ops.unpermute_sum(dxp.cuda(), dest_t)
    check(dx, candidates(om.unpermute_sum(np64(dxp), dest, bf16=False)), TOL_BF16, "dx")


def test_unpermute_sum_with_router_term():
    T, d, E, k = 150, 64, 12, 3
    idx = _random_topk(T, E, k, 77)
    _, _, dest, _ = om.dispatch_plan(idx, E)
    dxp = _bf16(I.stream_key(1, 2), (T * k, d))
    dl = I.normal_f32(I.stream_key(1, 3), (T, E))
    wr = _bf16(I.stream_key(1, 4), (d, E), 0.1)
    dx = ops.unpermute_sum(dxp.cuda(), torch.from_numpy(dest.astype(np.int32)).cuda(), dl.cuda(), wr.cuda())
    extra = dl.double().numpy() @ np64(wr).T
    check(dx, candidates(om.unpermute_sum(np64(dxp), dest, extra, bf16=False)), TOL_BF16, "dx")


def test_swiglu_standalone():
    M, f = 333, 136
    gu = _bf16(I.stream_key(2, 1), (M, 2 * f), 2.0)
    da = _bf16(I.stream_key(2, 2), (M, f))
    a = ops.swiglu(gu.cuda(), f)
    g = np64(gu)
    check(a, candidates(om.silu(g[:, :f]) * g[:, f:]), TOL_BF16, "A")
    dh = ops.swiglu_bwd(gu.cuda(), da.cuda())
    dG, dU = om.swiglu_backward(np64(da), g[:, :f], g[:, f:])
    check(np64(dh)[:, :f], candidates(dG), TOL_BF16, "dG")
    check(np64(dh)[:, f:], candidates(dU), TOL_BF16, "dU")


# ------------------------------------------------------------------ MXFP8 quantize

@pytest.mark.parametrize("rows,cols", [(1, 32), (77, 96), (512, 4096)])
def test_mxfp8_rowwise_bit_exact(rows, cols):
    x = _bf16(I.stream_key(rows, cols), (rows, cols), 3.0)
    xs = x.float()
    xs[0, :32] = 0.0                                    # all-zero block
    xs[-1, -32:] = torch.tensor([2.0 ** j for j in range(-16, 16)])
    if cols > 40:
        xs[0, 40] = 1e-39                               # subnormal bf16 input
        xs[0, 41:64] = 0.0                              # block whose amax is subnormal
    x = xs.to(torch.bfloat16)
    codes, scales = ops.mxfp8_quantize(x.cuda(), 1)
    rc, rs = om.mx_rowwise(np64(x))
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(scales.cpu().numpy(), rs)


# 64 groups of 0..199 rows x 1056 columns: several items per CTA, partial
# blocks at every group end, a 32-column tail tile
MANY_GROUPS = np.random.default_rng(7).integers(0, 200, 64).tolist()


def _colwise_case(counts, cols):
    off = _offsets(counts)
    rows = int(off[-1])
    x = _bf16(I.stream_key(rows, 5), (rows, cols), 0.7).float()
    if rows >= 40 and cols >= 8:
        x[:32, 0] = 0.0                                 # all-zero block
        x[:32, 1] = 1e-39                               # block whose amax is subnormal
        x[5, 2] = 1e-39                                 # a subnormal value in a normal block
        x[7, 3] = -3.0e38                               # large magnitude (scale 2^119)
    x = x.to(torch.bfloat16)
    codes, scales = ops.mxfp8_quantize(x.cuda(), 0, torch.from_numpy(off.astype(np.int32)).cuda())
    rc, rs, _ = om.mx_colwise_grouped(np64(x), off)
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(scales.cpu().numpy()[:rs.shape[0]], rs)


@pytest.mark.parametrize("counts,cols", [([40, 0, 24, 1, 100], 64), ([512], 4096), ([33, 31, 32], 96),
                                         ([100, 7], 1056), (MANY_GROUPS, 1056)])
def test_mxfp8_colwise_grouped_bit_exact(counts, cols):
    _colwise_case(counts, cols)


def test_generator_is_device_independent():
    key = I.stream_key(123, 4)
    a = I.normal_bf16(key, (4096, 64), 0.02, device="cuda", start=1 << 20).cpu()
    b = I.normal_bf16(key, (4096, 64), 0.02, device="cpu", start=1 << 20)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    lg_g = I.make_logits(I.CONFIGS["skewed"], device="cuda").cpu()
    lg_c = I.make_logits(I.CONFIGS["skewed"], device="cpu")
    assert torch.equal(lg_g.view(torch.int32), lg_c.view(torch.int32))


# ------------------------------------------------------------------ MXFP8 grouped GEMM
# The GEMM is fed E4M3 codes and E8M0 scales produced by the oracle's own
# quantiser (uploaded), and compared with the oracle's fp64 product of the
# decoded operands.

def _mx_rows(a2d):
    """Oracle rowwise quantisation -> (codes, scales, decoded)."""
    c, s = om.mx_rowwise(a2d)
    return c, s, om.mx_rowwise_decoded(a2d)


def _mx_cols(a2d, offsets):
    c, s, _ = om.mx_colwise_grouped(a2d, offsets)
    return c, s, om.mx_colwise_decoded(a2d, offsets)


def _u8(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def _mx_gemm(mode, ac, asc, bc, bsc, off, E, **kw):
    from routing_grouped_gemm_moe_b200 import _lib as L2
    import ctypes as C
    dev = "cuda"
    M_total = ac.shape[0]
    epi = kw.get("epilogue", L2.EPI_NONE)
    N, K, M = kw["N"], kw.get("K", 0), kw.get("M", 0)
    if mode == L2.GG_RAGGED_K:
        c = torch.full((E, M, N), 5.0, dtype=torch.bfloat16, device=dev)
    elif epi == L2.EPI_SWIGLU_BWD:
        c = torch.empty(M_total, 2 * N, dtype=torch.bfloat16, device=dev)
    else:
        c = torch.empty(M_total, N, dtype=torch.bfloat16, device=dev)
    aux = torch.empty(M_total, N // 2, dtype=torch.bfloat16, device=dev) if epi == L2.EPI_SWIGLU else None
    gu = kw.get("gu")
    ts = [_u8(ac), _u8(asc), _u8(bc), _u8(bsc), torch.from_numpy(np.asarray(off, np.int32)).cuda()]
    args = L2.GGArgs(mode=mode, dtype=L2.DTYPE_MXFP8, epilogue=epi, E=E, M_total=M_total, M=M, N=N,
                     K=K, offsets=ops._p(ts[4]), a=ops._p(ts[0]), b=ops._p(ts[2]),
                     b_mn_major=int(kw.get("b_mn", False)), c=ops._p(c), aux=ops._p(aux),
                     gu=ops._p(gu), a_scales=ops._p(ts[1]), b_scales=ops._p(ts[3]),
                     status=ops._p(kw.get("status")))
    nb = int(L2.lib().moe_grouped_gemm_workspace_bytes(C.byref(args)))
    ws = torch.empty(max(nb, 16), dtype=torch.uint8, device=dev)
    args.workspace = ops._p(ws)
    args.workspace_bytes = nb
    q = None
    if kw.get("fused_q"):
        W = N // 2 if epi == L2.EPI_SWIGLU else 2 * N
        nblk = sum((int(off[e + 1]) - int(off[e]) + 31) // 32 for e in range(E))
        q = dict(row_codes=torch.zeros(M_total, W, dtype=torch.uint8, device=dev),
                 row_scales=torch.zeros(M_total, W // 32, dtype=torch.uint8, device=dev),
                 col_codes=torch.zeros(M_total, W, dtype=torch.uint8, device=dev),
                 col_scales=torch.zeros(max(nblk, 1), W, dtype=torch.uint8, device=dev))
        args.q_row_codes, args.q_row_scales = ops._p(q["row_codes"]), ops._p(q["row_scales"])
        args.q_col_codes, args.q_col_scales = ops._p(q["col_codes"]), ops._p(q["col_scales"])
    L2.call("moe_grouped_gemm", C.byref(args), ops._s())
    torch.cuda.synchronize()
    if q is not None:
        return c, aux, q
    return c, aux


MX_RAGGED = [130, 0, 257, 1, 128, 64, 600]


# N >= 256 runs 256 x 256 tiles on CTA pairs (320: a 64-column tail tile), smaller N
# 128 x 128 tiles on single CTAs
@pytest.mark.parametrize("N,K,b_mn", [(256, 256, False), (256, 192, True), (128, 128, False),
                                      (384, 512, True), (320, 256, False), (320, 128, True)])
def test_mxfp8_grouped_gemm_ragged_m(N, K, b_mn):
    E = len(MX_RAGGED)
    off = _offsets(MX_RAGGED)
    Mt = int(off[-1])
    a = np64(_bf16(I.stream_key(N, K + 1), (Mt, K)))
    b = np64(_bf16(I.stream_key(K, N + 1), (E, K, N) if b_mn else (E, N, K), 0.05))
    ac, asc, ad = _mx_rows(a)
    if b_mn:
        koff = np.arange(E + 1) * K
        bc, bsc, bd = _mx_cols(b.reshape(E * K, N), koff)
    else:
        bc, bsc, bd = _mx_rows(b.reshape(E * N, K))
    c, _ = _mx_gemm(L.GG_RAGGED_M, ac, asc, bc, bsc, off, E, N=N, K=K, b_mn=b_mn)
    ref = om.grouped_gemm_ragged_m(ad, bd.reshape(b.shape), off, b_mn_major=b_mn)
    check(np64(c), candidates(ref), TOL_BF16, "C")


def test_mxfp8_grouped_gemm_flags_offsets_that_go_down():
    """Offsets that go down are reported in the status word
    (MOE_ERR_DEVICE_BOUNDS); the scale tables then use the running maximum of
    the offsets, so the GEMM stays inside its buffers."""
    E, N, K = 3, 128, 128
    bad = np.array([0, 96, 0, 96], np.int64)
    Mt = 96
    a = np64(_bf16(I.stream_key(N, 41), (Mt, K)))
    b = np64(_bf16(I.stream_key(K, 42), (E, N, K), 0.05))
    ac, asc, _ = _mx_rows(a)
    bc, bsc, _ = _mx_rows(b.reshape(E * N, K))
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    _mx_gemm(L.GG_RAGGED_M, ac, asc, bc, bsc, bad, E, N=N, K=K, status=status)
    assert int(status[0].item()) & (1 << 5)   # MOE_ERR_DEVICE_BOUNDS


@pytest.mark.parametrize("f,K", [(256, 256), (320, 128), (64, 128)])
def test_mxfp8_grouped_gemm_swiglu(f, K):
    E = len(MX_RAGGED)
    off = _offsets(MX_RAGGED)
    Mt = int(off[-1])
    a = np64(_bf16(I.stream_key(f, 11), (Mt, K)))
    b = np64(_bf16(I.stream_key(f, 12), (E, 2 * f, K), 0.05))
    ac, asc, ad = _mx_rows(a)
    bc, bsc, bd = _mx_rows(b.reshape(E * 2 * f, K))
    gu, act = _mx_gemm(L.GG_RAGGED_M, ac, asc, bc, bsc, off, E, N=2 * f, K=K, epilogue=L.EPI_SWIGLU)
    ref = om.grouped_gemm_ragged_m(ad, bd.reshape(b.shape), off)
    check(gu, candidates(ref), TOL_BF16, "GU")
    check(act, candidates(om.silu(ref[:, :f]) * ref[:, f:]), TOL_BF16, "A")


def test_mxfp8_grouped_gemm_swiglu_bwd():
    f, K = 256, 128
    E = len(MX_RAGGED)
    off = _offsets(MX_RAGGED)
    Mt = int(off[-1])
    a = np64(_bf16(I.stream_key(f, 13), (Mt, K)))
    b = np64(_bf16(I.stream_key(f, 14), (E, K, f), 0.05))
    gu = _bf16(I.stream_key(f, 15), (Mt, 2 * f))
    ac, asc, ad = _mx_rows(a)
    bc, bsc, bd = _mx_cols(b.reshape(E * K, f), np.arange(E + 1) * K)
    dh, _ = _mx_gemm(L.GG_RAGGED_M, ac, asc, bc, bsc, off, E, N=f, K=K, b_mn=True,
                     epilogue=L.EPI_SWIGLU_BWD, gu=gu.cuda())
    dA = om.grouped_gemm_ragged_m(ad, bd.reshape(b.shape), off, b_mn_major=True)
    g = np64(gu)
    dG, dU = om.swiglu_backward(dA, g[:, :f], g[:, f:])
    check(np64(dh)[:, :f], candidates(dG), TOL_BF16, "dG")
    check(np64(dh)[:, f:], candidates(dU), TOL_BF16, "dU")


@pytest.mark.parametrize("M,N,counts", [(128, 256, [70, 0, 200, 1, 64, 129]), (256, 128, [0, 300, 31]),
                                        (96, 384, [33, 0, 190, 64, 96]),
                                        # CTA pairs (M >= 256, N >= 256): K tails, empty experts,
                                        # a partial 256-column tile
                                        (256, 256, [70, 0, 200, 1, 64, 129]), (512, 384, [0, 300, 31, 129])])
def test_mxfp8_grouped_gemm_ragged_k(M, N, counts):
    E = len(counts)
    off = _offsets(counts)
    Mt = int(off[-1])
    a = np64(_bf16(I.stream_key(M, 21), (Mt, M)))
    b = np64(_bf16(I.stream_key(N, 22), (Mt, N)))
    ac, asc, ad = _mx_cols(a, off)
    bc, bsc, bd = _mx_cols(b, off)
    c, _ = _mx_gemm(L.GG_RAGGED_K, ac, asc, bc, bsc, off, E, M=M, N=N)
    ref = om.grouped_gemm_ragged_k(ad, bd, off)
    got = np64(c)
    for e in range(E):
        if counts[e] == 0:
            assert np.all(got[e] == 0)
        else:
            check(got[e], candidates(ref[e]), TOL_BF16, f"C[{e}]")


# ------------------------------------------------------------------ routing balance

@pytest.mark.parametrize("T,E,k,zipf", [(1000, 8, 2, False), (4096, 64, 8, True), (300, 1024, 4, False)])
def test_router_balance_and_backward(T, E, k, zipf):
    lg = I.normal_f32(I.stream_key(T, E), (T, E))
    if zipf:
        lg = lg + torch.log(torch.arange(1, E + 1, dtype=torch.float32)) * -1.2
    idx, _ = om.router_topk(lg.numpy(), k)
    counts, _, _, _ = om.dispatch_plan(idx, E)
    ct = torch.from_numpy(counts.astype(np.int32)).cuda()
    stats, P = ops.router_balance(lg.cuda(), ct, k)
    ref = om.router_balance(lg.numpy(), counts, k)
    got = stats.cpu().numpy()
    assert abs(got[0] - ref["aux"]) <= 1e-5 * max(1.0, ref["aux"])
    assert abs(got[1] - ref["max_over_mean"]) <= 1e-6 * ref["max_over_mean"]
    assert abs(got[2] - ref["cv"]) <= 1e-5 * max(1.0, ref["cv"])
    assert got[3] == ref["empty_frac"]
    assert_close(P, ref["P"], 1e-5, "P")
    # the kernel accumulates into d_logits: start from a tensor of the
    # gradient's own magnitude, so that the fp32 rounding of the sum stays far
    # below the tolerance
    ref_d = om.router_balance_backward(lg.numpy(), counts, k, 0.01)
    rms = float(np.sqrt(np.mean(ref_d ** 2)))
    base = I.normal_f32(I.stream_key(T + 1, E), (T, E)) * rms
    d = base.clone().cuda()
    ops.router_balance_bwd(lg.cuda(), ct, k, 0.01, d)
    assert_close(d.cpu().double().numpy() - base.double().numpy(), ref_d, 1e-4, "d_logits")


# ------------------------------------------------------------------ fused MXFP8 quantisation of
# the SwiGLU / SwiGLU-backward outputs: equal, byte for byte, to quantising the
# stored bf16 output with mxfp8_quantize (itself bit-exact against the oracle)

def _check_fused_q(out_bf16, q, off, E):
    rc, rs = ops.mxfp8_quantize(out_bf16, axis=1)
    assert torch.equal(q["row_codes"], rc) and torch.equal(q["row_scales"], rs)
    offs = torch.from_numpy(np.asarray(off, np.int32)).cuda()
    cc, cs = ops.mxfp8_quantize(out_bf16, axis=0, group_offsets=offs)
    nblk = q["col_scales"].shape[0]
    assert torch.equal(q["col_codes"], cc)
    assert torch.equal(q["col_scales"], cs[:nblk])


FUSED_COUNTS = [130, 0, 257, 1, 128, 64, 33]


@pytest.mark.parametrize("f,K,dtype", [(256, 256, "mxfp8"), (320, 128, "mxfp8"), (256, 128, "bf16")])
def test_fused_quant_swiglu(f, K, dtype):
    E = len(FUSED_COUNTS)
    off = _offsets(FUSED_COUNTS)
    Mt = int(off[-1])
    a = _bf16(I.stream_key(f, 31), (Mt, K))
    b = _bf16(I.stream_key(f, 32), (E, 2 * f, K), 0.05)
    if dtype == "mxfp8":
        ac, asc, _ = _mx_rows(np64(a))
        bc, bsc, _ = _mx_rows(np64(b).reshape(E * 2 * f, K))
        gu, act, q = _mx_gemm(L.GG_RAGGED_M, ac, asc, bc, bsc, off, E, N=2 * f, K=K,
                              epilogue=L.EPI_SWIGLU, fused_q=True)
    else:
        gu, act, q = _bf16_gemm_fused(a, b, off, E, N=2 * f, K=K, epilogue=L.EPI_SWIGLU)
    _check_fused_q(act, q, off, E)


@pytest.mark.parametrize("f,K,dtype", [(256, 128, "mxfp8"), (192, 256, "bf16"), (512, 128, "bf16")])
def test_fused_quant_swiglu_bwd(f, K, dtype):
    E = len(FUSED_COUNTS)
    off = _offsets(FUSED_COUNTS)
    Mt = int(off[-1])
    a = _bf16(I.stream_key(f, 33), (Mt, K))
    b = _bf16(I.stream_key(f, 34), (E, K, f), 0.05)
    gu = _bf16(I.stream_key(f, 35), (Mt, 2 * f)).cuda()
    if dtype == "mxfp8":
        ac, asc, _ = _mx_rows(np64(a))
        bc, bsc, _ = _mx_cols(np64(b).reshape(E * K, f), np.arange(E + 1) * K)
        dh, _, q = _mx_gemm(L.GG_RAGGED_M, ac, asc, bc, bsc, off, E, N=f, K=K, b_mn=True,
                            epilogue=L.EPI_SWIGLU_BWD, gu=gu, fused_q=True)
    else:
        dh, _, q = _bf16_gemm_fused(a, b, off, E, N=f, K=K, epilogue=L.EPI_SWIGLU_BWD, gu=gu, b_mn=True)
    _check_fused_q(dh, q, off, E)


def _bf16_gemm_fused(a, b, off, E, N, K, epilogue, gu=None, b_mn=False):
    import ctypes as C
    dev = "cuda"
    a, b = a.cuda(), b.cuda()
    Mt = a.shape[0]
    offs = torch.from_numpy(np.asarray(off, np.int32)).cuda()
    if epilogue == L.EPI_SWIGLU:
        c = torch.empty(Mt, N, dtype=torch.bfloat16, device=dev)
        aux = torch.empty(Mt, N // 2, dtype=torch.bfloat16, device=dev)
        W = N // 2
    else:
        c = torch.empty(Mt, 2 * N, dtype=torch.bfloat16, device=dev)
        aux = None
        W = 2 * N
    nblk = sum((int(off[e + 1]) - int(off[e]) + 31) // 32 for e in range(E))
    q = dict(row_codes=torch.zeros(Mt, W, dtype=torch.uint8, device=dev),
             row_scales=torch.zeros(Mt, W // 32, dtype=torch.uint8, device=dev),
             col_codes=torch.zeros(Mt, W, dtype=torch.uint8, device=dev),
             col_scales=torch.zeros(max(nblk, 1), W, dtype=torch.uint8, device=dev))
    args = L.GGArgs(mode=L.GG_RAGGED_M, dtype=L.DTYPE_BF16, epilogue=epilogue, E=E, M_total=Mt, M=0,
                    N=N, K=K, offsets=ops._p(offs), a=ops._p(a), b=ops._p(b), b_mn_major=int(b_mn),
                    c=ops._p(c), aux=ops._p(aux), gu=ops._p(gu), status=None,
                    q_row_codes=ops._p(q["row_codes"]), q_row_scales=ops._p(q["row_scales"]),
                    q_col_codes=ops._p(q["col_codes"]), q_col_scales=ops._p(q["col_scales"]))
    L.call("moe_grouped_gemm", C.byref(args), ops._s())
    torch.cuda.synchronize()
    return c, aux, q


@pytest.mark.parametrize("counts,cols", [([40, 0, 24, 1, 100], 64), ([512, 33], 4096), ([33, 31, 32], 320),
                                         ([65], 2080), (MANY_GROUPS, 1056)])
def test_mxfp8_rowcol_equals_both_quantisers(counts, cols):
    """One read, both encodings: byte for byte what the two single-axis
    quantisers write (themselves bit-exact against the oracle)."""
    off = _offsets(counts)
    rows = int(off[-1])
    x = _bf16(I.stream_key(rows, cols), (rows, cols)).cuda()
    offs = torch.from_numpy(off.astype(np.int32)).cuda()
    rc, rs, cc, cs = ops.mxfp8_quantize_rowcol(x, offs)
    rc1, rs1 = ops.mxfp8_quantize(x, axis=1)
    cc1, cs1 = ops.mxfp8_quantize(x, axis=0, group_offsets=offs)
    assert torch.equal(rc, rc1) and torch.equal(rs, rs1)
    assert torch.equal(cc, cc1) and torch.equal(cs, cs1)


# The alternative tilings that environment switches select (read once per
# process): single CTAs instead of CTA pairs for BF16 and MXFP8 256-wide tiles,
# 128 x 128 MXFP8 tiles, single-CTA BF16 SwiGLU backward, persistent CTAs
# not kept in step, M = 256 pair MMAs on every row tile.
ALT_TILINGS = [{"MOE_GG_NO_PAIRS": "1", "MOE_GG_MX_NO_PAIRS": "1"},
               {"MOE_GG_MX_NARROW": "1", "MOE_GG_SINGLE_BWD": "1", "MOE_GG_SYNC_SLACK": "0",
                "MOE_GG_NO_HALF_TILES": "1"}]


@pytest.mark.parametrize("flags", ALT_TILINGS, ids=["single_cta", "narrow_mx"])
def test_alternative_tilings(flags):
    """The grouped-GEMM tests above, run again in a child process with the
    switches set: the tilings they select must be just as correct."""
    import os
    import subprocess
    import sys
    if os.environ.get("MOE_TEST_CHILD"):
        pytest.skip("inside the child run")
    env = dict(os.environ, MOE_TEST_CHILD="1", **flags)
    r = subprocess.run([sys.executable, "-m", "pytest", __file__, "-q", "-x", "-p", "no:cacheprovider",
                        "-m", "gpu", "-k", "grouped_gemm or fused"],
                       env=env, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
