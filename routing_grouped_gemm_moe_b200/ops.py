"""PyTorch-facing binding of the MoE layer library.

Every function here only allocates output tensors (PyTorch owns device memory)
and passes pointers, sizes and the current CUDA stream to the C ABI; all
arithmetic runs in the library's CUDA kernels.  Tensors must be contiguous
CUDA tensors of the stated dtypes; bf16 tensors travel as their bit patterns.
"""
from __future__ import annotations

import ctypes as C
from dataclasses import dataclass

import torch

from . import _lib as L


def _p(t):
    if t is None:
        return None
    assert t.is_cuda and t.is_contiguous(), "expected a contiguous CUDA tensor"
    return C.c_void_p(t.data_ptr())


def _s():
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def _bf16(t):
    assert t.dtype == torch.bfloat16
    return t


def expect(t, name: str, shape, dtype, device=None):
    """Raise ValueError unless `t` is a contiguous tensor of exactly this shape
    and dtype (on `device` when given): the library reads and writes that many
    bytes through the raw pointer and cannot check them itself."""
    if t is None:
        raise ValueError(f"{name}: a tensor is required")
    shape = tuple(int(v) for v in shape)
    if tuple(t.shape) != shape or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous {dtype} tensor of shape {shape}, got "
                         f"{'a non-contiguous ' if not t.is_contiguous() else ''}{t.dtype} "
                         f"{tuple(t.shape)}")
    if device is not None:
        want = torch.device(device)  # "cuda" without an index accepts any CUDA device
        if t.device.type != want.type or (want.index is not None and t.device.index != want.index):
            raise ValueError(f"{name}: expected a tensor on {device}, got one on {t.device}")
    return t


# --------------------------------------------------------------------- router

def router_topk(logits: torch.Tensor, k: int):
    T, E = logits.shape
    expect(logits, "logits", (T, E), torch.float32)
    idx = torch.empty(T, k, dtype=torch.int32, device=logits.device)
    w = torch.empty(T, k, dtype=torch.float32, device=logits.device)
    L.call("moe_router_topk", _p(logits), T, E, k, _p(idx), _p(w), _s())
    return idx, w


def router_topk_proj(x: torch.Tensor, w_r: torch.Tensor, k: int):
    T, d = x.shape
    E = w_r.shape[1]
    expect(x, "x", (T, d), torch.bfloat16)
    expect(w_r, "w_r", (d, E), torch.bfloat16, x.device)
    logits = torch.empty(T, E, dtype=torch.float32, device=x.device)
    idx = torch.empty(T, k, dtype=torch.int32, device=x.device)
    w = torch.empty(T, k, dtype=torch.float32, device=x.device)
    L.call("moe_router_topk_proj", _p(_bf16(x)), _p(_bf16(w_r)), T, d, E, k, _p(logits), _p(idx),
           _p(w), _s())
    return logits, idx, w


def router_bwd(idx, w, dw, E: int):
    T, k = idx.shape
    expect(idx, "idx", (T, k), torch.int32)
    expect(w, "w", (T, k), torch.float32, idx.device)
    expect(dw, "dw", (T, k), torch.float32, idx.device)
    dl = torch.empty(T, E, dtype=torch.float32, device=idx.device)
    L.call("moe_router_bwd", _p(idx), _p(w), _p(dw), T, E, k, _p(dl), _s())
    return dl


def router_proj_bwd(x, d_logits):
    T, d = x.shape
    E = d_logits.shape[1]
    expect(x, "x", (T, d), torch.bfloat16)
    expect(d_logits, "d_logits", (T, E), torch.float32, x.device)
    dwr = torch.empty(d, E, dtype=torch.bfloat16, device=x.device)
    L.call("moe_router_proj_bwd", _p(_bf16(x)), _p(d_logits), T, d, E, _p(dwr), _s())
    return dwr


def router_balance(logits, counts, k: int):
    """Returns (stats fp32 [4] = [aux loss, max/mean load, cv of load, empty
    fraction], P fp32 [E] = mean softmax probability per expert)."""
    T, E = logits.shape
    expect(logits, "logits", (T, E), torch.float32)
    expect(counts, "counts", (E,), torch.int32, logits.device)
    stats = torch.empty(4, dtype=torch.float32, device=logits.device)
    P = torch.empty(E, dtype=torch.float32, device=logits.device)
    nb = int(L.lib().moe_router_balance_workspace_bytes(T, E))
    ws = torch.empty(max(nb, 16), dtype=torch.uint8, device=logits.device)
    L.call("moe_router_balance", _p(logits), _p(counts), T, E, k, _p(stats), _p(P), _p(ws), nb,
           _s())
    return stats, P


def router_balance_bwd(logits, counts, k: int, scale: float, d_logits):
    """d_logits += d(scale * aux loss) / d logits (counts held fixed); in place."""
    T, E = logits.shape
    expect(logits, "logits", (T, E), torch.float32)
    expect(counts, "counts", (E,), torch.int32, logits.device)
    expect(d_logits, "d_logits", (T, E), torch.float32, logits.device)
    L.call("moe_router_balance_bwd", _p(logits), _p(counts), T, E, k, float(scale),
           _p(d_logits), _s())
    return d_logits


# ------------------------------------------------------------------- dispatch

def permute_workspace_bytes(T: int, E: int) -> int:
    return int(L.lib().moe_permute_workspace_bytes(T, E))


def _dispatch_inputs(x, idx):
    """(T, d, k) of a dispatch after checking x (bf16 [T, d]) and idx (int32
    [T, k] on x's device): an int64 idx (torch.topk's default) would be read
    as pairs of int32 and route silently wrong."""
    if x is None or idx is None or x.dim() != 2 or idx.dim() != 2:
        raise ValueError("x must be a [T, d] and idx a [T, k] tensor")
    T, d = x.shape
    k = idx.shape[1]
    expect(x, "x", (T, d), torch.bfloat16)
    expect(idx, "idx", (T, k), torch.int32, x.device)
    return T, d, k


def _check_workspace(ws, nbytes: int, device):
    if ws.dtype != torch.uint8 or not ws.is_contiguous() or ws.numel() < nbytes:
        raise ValueError(f"workspace: expected a contiguous uint8 tensor of at least {nbytes} "
                         f"bytes, got {ws.dtype} {tuple(ws.shape)}")
    expect(ws, "workspace", tuple(ws.shape), torch.uint8, device)


def permute_rows(x: torch.Tensor, idx: torch.Tensor, E: int, workspace=None):
    """Returns (counts, offsets, dest_pos, src_token, x_perm, workspace)."""
    T, d, k = _dispatch_inputs(x, idx)
    dev = x.device
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    dest = torch.empty(T, k, dtype=torch.int32, device=dev)
    src = torch.empty(T * k, dtype=torch.int32, device=dev)
    x_perm = torch.empty(T * k, d, dtype=torch.bfloat16, device=dev)
    nbytes = permute_workspace_bytes(T, E)
    if workspace is None:
        workspace = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
    _check_workspace(workspace, nbytes, dev)
    L.call("moe_permute_rows", _p(_bf16(x)), _p(idx), T, d, E, k, _p(counts), _p(offsets),
           _p(dest), _p(src), _p(x_perm), _p(workspace), workspace.numel(), _s())
    return counts, offsets, dest, src, x_perm, workspace


def permute_rows_mxfp8(x: torch.Tensor, idx: torch.Tensor, E: int, workspace=None):
    """moe_permute_rows_mxfp8: the dispatch plus the row-wise MXFP8 encoding of
    every routed row.  Returns (counts, offsets, dest_pos, src_token, x_perm,
    x_perm_codes, x_perm_scales)."""
    T, d, k = _dispatch_inputs(x, idx)
    dev = x.device
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    dest = torch.empty(T, k, dtype=torch.int32, device=dev)
    src = torch.empty(T * k, dtype=torch.int32, device=dev)
    x_perm = torch.empty(T * k, d, dtype=torch.bfloat16, device=dev)
    codes = torch.empty(T * k, d, dtype=torch.uint8, device=dev)
    scales = torch.empty(T * k, d // 32, dtype=torch.uint8, device=dev)
    nbytes = permute_workspace_bytes(T, E)
    if workspace is None:
        workspace = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
    _check_workspace(workspace, nbytes, dev)
    L.call("moe_permute_rows_mxfp8", _p(_bf16(x)), _p(idx), T, d, E, k, _p(counts), _p(offsets),
           _p(dest), _p(src), _p(x_perm), _p(codes), _p(scales), _p(workspace), workspace.numel(),
           _s())
    return counts, offsets, dest, src, x_perm, codes, scales


def permute_rows_noalloc(x: torch.Tensor, idx: torch.Tensor, E: int):
    """moe_permute_rows_noalloc: the same dispatch with the library's own fixed
    scratch (no workspace).  Returns (counts, offsets, dest_pos, src_token, x_perm)."""
    T, d, k = _dispatch_inputs(x, idx)
    dev = x.device
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    dest = torch.empty(T, k, dtype=torch.int32, device=dev)
    src = torch.empty(T * k, dtype=torch.int32, device=dev)
    x_perm = torch.empty(T * k, d, dtype=torch.bfloat16, device=dev)
    L.call("moe_permute_rows_noalloc", _p(_bf16(x)), _p(idx), T, d, E, k, _p(counts),
           _p(offsets), _p(dest), _p(src), _p(x_perm), _s())
    return counts, offsets, dest, src, x_perm


# --------------------------------------------------------------- grouped GEMM

def grouped_gemm(mode: int, a, b, offsets, E: int, *, N: int, K: int = 0, M: int = 0,
                 b_mn_major: bool = False, epilogue: int = L.EPI_NONE, c=None, aux=None,
                 gu=None, status=None, kmaps: bool = True):
    """Raw grouped GEMM (see moe_grouped_gemm in include/moe_b200.h).  Output
    buffers are allocated when not given; every tensor is checked against the
    sizes the call implies.  kmaps (RAGGED_K): give the call its optional
    workspace of per-expert tensor maps (False: the kernel zeroes the rows
    past each expert in shared memory instead)."""
    dev = a.device
    M_total = a.shape[0]
    bf = torch.bfloat16
    expect(offsets, "offsets", (E + 1,), torch.int32, dev)
    if mode == L.GG_RAGGED_K:
        expect(a, "a", (M_total, M), bf, dev)
        expect(b, "b", (M_total, N), bf, dev)
    else:
        expect(a, "a", (M_total, K), bf, dev)
        expect(b, "b", (E, K, N) if b_mn_major else (E, N, K), bf, dev)
        if epilogue == L.EPI_SWIGLU_BWD:
            expect(gu, "gu", (M_total, 2 * N), bf, dev)
    if c is None:
        if mode == L.GG_RAGGED_K:
            c = torch.empty(E, M, N, dtype=torch.bfloat16, device=dev)
        elif epilogue == L.EPI_SWIGLU_BWD:
            c = torch.empty(M_total, 2 * N, dtype=torch.bfloat16, device=dev)
        else:
            c = torch.empty(M_total, N, dtype=torch.bfloat16, device=dev)
    if epilogue == L.EPI_SWIGLU and aux is None:
        aux = torch.empty(M_total, N // 2, dtype=torch.bfloat16, device=dev)
    if mode == L.GG_RAGGED_K:
        expect(c, "c", (E, M, N), bf, dev)
    else:
        expect(c, "c", (M_total, 2 * N if epilogue == L.EPI_SWIGLU_BWD else N), bf, dev)
    if epilogue == L.EPI_SWIGLU:
        expect(aux, "aux", (M_total, N // 2), bf, dev)
    args = L.GGArgs(mode=mode, dtype=L.DTYPE_BF16, epilogue=epilogue, E=E, M_total=M_total, M=M,
                    N=N, K=K, offsets=_p(offsets), a=_p(a), b=_p(b), b_mn_major=int(b_mn_major),
                    c=_p(c), aux=_p(aux), gu=_p(gu), a_scales=None, b_scales=None,
                    status=_p(status))
    nb = int(L.lib().moe_grouped_gemm_workspace_bytes(C.byref(args)))
    if nb and kmaps:
        ws = torch.empty(nb, dtype=torch.uint8, device=dev)
        args.workspace = _p(ws)
        args.workspace_bytes = nb
    L.call("moe_grouped_gemm", C.byref(args), _s())
    return (c, aux) if epilogue == L.EPI_SWIGLU else c


def swiglu(gu, f: int):
    M = gu.shape[0]
    expect(gu, "gu", (M, 2 * f), torch.bfloat16)
    a = torch.empty(M, f, dtype=torch.bfloat16, device=gu.device)
    L.call("moe_swiglu", _p(gu), _p(a), M, f, _s())
    return a


def swiglu_bwd(gu, da):
    M, f = da.shape
    expect(da, "da", (M, f), torch.bfloat16)
    expect(gu, "gu", (M, 2 * f), torch.bfloat16, da.device)
    dh = torch.empty(M, 2 * f, dtype=torch.bfloat16, device=gu.device)
    L.call("moe_swiglu_bwd", _p(gu), _p(da), _p(dh), M, f, _s())
    return dh


# -------------------------------------------------------------------- combine

def unpermute_combine(y_perm, dest_pos, topk_w):
    T, k = dest_pos.shape
    d = y_perm.shape[1]
    expect(dest_pos, "dest_pos", (T, k), torch.int32)
    expect(y_perm, "y_perm", (T * k, d), torch.bfloat16, dest_pos.device)
    expect(topk_w, "topk_w", (T, k), torch.float32, dest_pos.device)
    out = torch.empty(T, d, dtype=torch.bfloat16, device=y_perm.device)
    L.call("moe_unpermute_combine", _p(y_perm), _p(dest_pos), _p(topk_w), T, d, k, _p(out), _s())
    return out


def unpermute_combine_bwd(dout, y_perm, dest_pos, topk_w):
    T, k = dest_pos.shape
    d = y_perm.shape[1]
    expect(dest_pos, "dest_pos", (T, k), torch.int32)
    expect(y_perm, "y_perm", (T * k, d), torch.bfloat16, dest_pos.device)
    expect(topk_w, "topk_w", (T, k), torch.float32, dest_pos.device)
    expect(dout, "dout", (T, d), torch.bfloat16, dest_pos.device)
    dy = torch.empty_like(y_perm)
    dw = torch.empty(T, k, dtype=torch.float32, device=y_perm.device)
    L.call("moe_unpermute_combine_bwd", _p(dout), _p(y_perm), _p(dest_pos), _p(topk_w), T, d, k,
           _p(dy), _p(dw), _s())
    return dy, dw


def unpermute_sum(dx_perm, dest_pos, d_logits=None, w_r=None):
    T, k = dest_pos.shape
    d = dx_perm.shape[1]
    E = d_logits.shape[1] if d_logits is not None else 0
    expect(dest_pos, "dest_pos", (T, k), torch.int32)
    expect(dx_perm, "dx_perm", (T * k, d), torch.bfloat16, dest_pos.device)
    if (d_logits is None) != (w_r is None):
        raise ValueError("d_logits and w_r: give both (router projection term) or neither")
    if d_logits is not None:
        expect(d_logits, "d_logits", (T, E), torch.float32, dest_pos.device)
        expect(w_r, "w_r", (d, E), torch.bfloat16, dest_pos.device)
    dx = torch.empty(T, d, dtype=torch.bfloat16, device=dx_perm.device)
    L.call("moe_unpermute_sum", _p(dx_perm), _p(dest_pos), T, d, k, _p(d_logits), _p(w_r), E,
           _p(dx), _s())
    return dx


# ---------------------------------------------------------------------- MXFP8

def _group_offsets(group_offsets, x):
    """Number of groups after checking group_offsets (int32 [G+1] on x's
    device, or None for one group)."""
    if group_offsets is None:
        return 1
    if group_offsets.dim() != 1 or group_offsets.numel() < 2:
        raise ValueError("group_offsets: expected an int32 tensor of G + 1 >= 2 values")
    expect(group_offsets, "group_offsets", (group_offsets.numel(),), torch.int32, x.device)
    return group_offsets.numel() - 1


def mxfp8_quantize(x, axis: int, group_offsets=None):
    """Returns (codes uint8 like x, scales uint8)."""
    rows, cols = x.shape
    expect(x, "x", (rows, cols), torch.bfloat16)
    codes = torch.empty(rows, cols, dtype=torch.uint8, device=x.device)
    if axis == 1:
        scales = torch.empty(rows, cols // 32, dtype=torch.uint8, device=x.device)
        ng = 0
    else:
        ng = _group_offsets(group_offsets, x)
        scales = torch.zeros(rows // 32 + ng, cols, dtype=torch.uint8, device=x.device)
    L.call("mxfp8_quantize", _p(_bf16(x)), rows, cols, axis, _p(group_offsets), ng, _p(codes),
           _p(scales), None, _s())
    return codes, scales


def mxfp8_quantize_rowcol(x, group_offsets=None):
    """Both encodings from one read: (row_codes, row_scales, col_codes, col_scales)."""
    rows, cols = x.shape
    expect(x, "x", (rows, cols), torch.bfloat16)
    ng = _group_offsets(group_offsets, x)
    rc = torch.empty(rows, cols, dtype=torch.uint8, device=x.device)
    rs = torch.empty(rows, cols // 32, dtype=torch.uint8, device=x.device)
    cc = torch.empty(rows, cols, dtype=torch.uint8, device=x.device)
    cs = torch.zeros(rows // 32 + ng, cols, dtype=torch.uint8, device=x.device)
    L.call("mxfp8_quantize_rowcol", _p(_bf16(x)), rows, cols, _p(group_offsets), ng, _p(rc), _p(rs),
           _p(cc), _p(cs), _s())
    return rc, rs, cc, cs


# ---------------------------------------------------------------------- layer

def make_events(n: int):
    """n timing events, created on the current stream (recorded once)."""
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for e in evs:
        e.record()
    return evs


def kernel_launches() -> int:
    return int(L.lib().moe_kernel_launches())


MX_GEMM_NAMES = {"gemm1": L.MX_GEMM1, "gemm2": L.MX_GEMM2, "dA": L.MX_DA, "dW2": L.MX_DW2,
                 "dX": L.MX_DX, "dW13": L.MX_DW13}


def mx_gemm_mask(names) -> int:
    """MOE_MX_* bit mask for an iterable of GEMM names (None: 0 = all six)."""
    if names is None:
        return 0
    mask = 0
    for n in names:
        if n not in MX_GEMM_NAMES:
            raise ValueError(f"unknown GEMM {n!r}; expected one of {sorted(MX_GEMM_NAMES)}")
        mask |= MX_GEMM_NAMES[n]
    if mask == 0:
        raise ValueError("mx_gemms selects no GEMM; use dtype='bf16' instead")
    return mask


def layer_workspace_bytes(T: int, d: int, E: int, k: int, f: int, router: str = "logits",
                          dtype: str = "bf16", recompute: bool = False, mx_gemms=None,
                          mx_keep_weights: bool = False) -> int:
    """Workspace bytes of a layer of this shape (moe_layer_workspace_bytes)."""
    desc = L.LayerDesc(T=T, d=d, E=E, k=k, f=f,
                       dtype=L.DTYPE_MXFP8 if dtype == "mxfp8" else L.DTYPE_BF16,
                       router_mode=L.ROUTER_PROJ if router == "proj" else L.ROUTER_LOGITS,
                       recompute=int(bool(recompute)), mx_gemms=mx_gemm_mask(mx_gemms),
                       mx_keep_weights=int(bool(mx_keep_weights)))
    return int(L.lib().moe_layer_workspace_bytes(C.byref(desc)))


@dataclass
class LayerState:
    """Device buffers the forward writes and the backward reads."""
    logits: torch.Tensor | None
    topk_idx: torch.Tensor
    topk_w: torch.Tensor
    counts: torch.Tensor
    offsets: torch.Tensor
    dest_pos: torch.Tensor
    src_token: torch.Tensor
    x_perm: torch.Tensor
    gu: torch.Tensor | None      # None in recompute mode
    a: torch.Tensor | None
    y_perm: torch.Tensor

    def c_struct(self) -> L.LayerSaved:
        return L.LayerSaved(logits=_p(self.logits), topk_idx=_p(self.topk_idx),
                            topk_w=_p(self.topk_w), counts=_p(self.counts),
                            offsets=_p(self.offsets), dest_pos=_p(self.dest_pos),
                            src_token=_p(self.src_token), x_perm=_p(self.x_perm),
                            gu=_p(self.gu), a=_p(self.a), y_perm=_p(self.y_perm))


class MoELayer:
    """One MoE expert layer on one GPU: buffers sized once for (T, d, E, k, f)."""

    def __init__(self, T: int, d: int, E: int, k: int, f: int, router: str = "logits",
                 dtype: str = "bf16", device="cuda", recompute: bool = False,
                 mx_gemms=None, mx_keep_weights: bool = False, workspace=None):
        """recompute: keep [G | U] and A only in the workspace and run GEMM1 +
        SwiGLU again in the backward.  mx_gemms (dtype "mxfp8" only): names
        from MX_GEMM_NAMES of the GEMMs that take MXFP8 operands (None: all).
        mx_keep_weights: the forward quantises each weight for its forward and
        its backward GEMM in one read and the backward reuses the second
        encoding (the backward must get the forward's weights).
        workspace: a uint8 device tensor of at least workspace_bytes() to use
        instead of a new one.  Layers that run one after the other on one
        stream may share one: the backward reads nothing from the workspace
        that its forward wrote -- except with mx_keep_weights (the kept
        weight encodings), which therefore refuses a shared workspace."""
        self.T, self.d, self.E, self.k, self.f = T, d, E, k, f
        self.router_mode = L.ROUTER_PROJ if router == "proj" else L.ROUTER_LOGITS
        self.dtype = L.DTYPE_MXFP8 if dtype == "mxfp8" else L.DTYPE_BF16
        self.recompute = bool(recompute)
        self.mx_mask = mx_gemm_mask(mx_gemms)
        self.desc = L.LayerDesc(T=T, d=d, E=E, k=k, f=f, dtype=self.dtype,
                                router_mode=self.router_mode, recompute=int(self.recompute),
                                mx_gemms=self.mx_mask, mx_keep_weights=int(bool(mx_keep_weights)))
        dev = torch.device(device)
        M = T * k
        bf = torch.bfloat16
        self.state = LayerState(
            logits=torch.empty(T, E, dtype=torch.float32, device=dev)
            if self.router_mode == L.ROUTER_PROJ else None,
            topk_idx=torch.empty(T, k, dtype=torch.int32, device=dev),
            topk_w=torch.empty(T, k, dtype=torch.float32, device=dev),
            counts=torch.empty(E, dtype=torch.int32, device=dev),
            offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
            dest_pos=torch.empty(T, k, dtype=torch.int32, device=dev),
            src_token=torch.empty(M, dtype=torch.int32, device=dev),
            x_perm=torch.empty(M, d, dtype=bf, device=dev),
            gu=None if self.recompute else torch.empty(M, 2 * f, dtype=bf, device=dev),
            a=None if self.recompute else torch.empty(M, f, dtype=bf, device=dev),
            y_perm=torch.empty(M, d, dtype=bf, device=dev),
        )
        nbytes = self.workspace_bytes()
        if workspace is None:
            self.workspace = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
        else:
            if mx_keep_weights:
                raise ValueError("mx_keep_weights keeps weight encodings in the workspace from "
                                 "the forward to the backward: give this layer its own")
            _check_workspace(workspace, nbytes, dev)
            self.workspace = workspace
        self.out = torch.empty(T, d, dtype=bf, device=dev)
        self.dx = torch.empty(T, d, dtype=bf, device=dev)
        self.dw13 = torch.empty(E, 2 * f, d, dtype=bf, device=dev)
        self.dw2 = torch.empty(E, d, f, dtype=bf, device=dev)
        self.dw_r = (torch.empty(d, E, dtype=bf, device=dev)
                     if self.router_mode == L.ROUTER_PROJ else None)
        self.d_logits = torch.empty(T, E, dtype=torch.float32, device=dev)
        self._saved = self.state.c_struct()

    def workspace_bytes(self) -> int:
        return int(L.lib().moe_layer_workspace_bytes(C.byref(self.desc)))

    def saved_bytes(self) -> int:
        """Device bytes of the state this layer keeps from its forward for its
        backward (routing, x_perm, Y_perm, and [G | U], A unless recompute)."""
        return sum(t.numel() * t.element_size() for t in vars(self.state).values()
                   if t is not None)

    def _set_events(self, events):
        """Stage events (torch.cuda.Event, already created) the next call records."""
        if events is None:
            self.desc.stage_events = None
            return
        self._ev_arr = (C.c_void_p * len(events))(*[C.c_void_p(e.cuda_event) for e in events])
        self.desc.stage_events = C.cast(self._ev_arr, C.POINTER(C.c_void_p))

    def _params(self, x, w13, w2, logits=None, w_r=None) -> L.LayerParams:
        T, d, E, f = self.T, self.d, self.E, self.f
        dev, bf = self.workspace.device, torch.bfloat16
        expect(x, "x", (T, d), bf, dev)
        expect(w13, "w13", (E, 2 * f, d), bf, dev)
        expect(w2, "w2", (E, d, f), bf, dev)
        if self.router_mode == L.ROUTER_LOGITS:
            expect(logits, "logits", (T, E), torch.float32, dev)
        else:
            expect(w_r, "w_r", (d, E), bf, dev)
        return L.LayerParams(x=_p(x), logits=_p(logits), w_r=_p(w_r), w13=_p(w13), w2=_p(w2))

    def forward(self, x, w13, w2, logits=None, w_r=None, events=None, out=None):
        """out: optional [T, d] bf16 destination (default: self.out)."""
        prm = self._params(x, w13, w2, logits, w_r)
        self._set_events(events)
        out = self.out if out is None else expect(out, "out", (self.T, self.d), torch.bfloat16,
                                                  self.workspace.device)
        L.call("moe_layer_fwd", C.byref(self.desc), C.byref(prm), C.byref(self._saved),
               _p(out), _p(self.workspace), self.workspace.numel(), _s())
        return out

    def backward(self, dout, x, w13, w2, logits=None, w_r=None, events=None, dx=None):
        """dx: optional [T, d] bf16 destination (default: self.dx)."""
        prm = self._params(x, w13, w2, logits, w_r)
        expect(dout, "dout", (self.T, self.d), torch.bfloat16, self.workspace.device)
        self._set_events(events)
        dx = self.dx if dx is None else expect(dx, "dx", (self.T, self.d), torch.bfloat16,
                                               self.workspace.device)
        gr = L.LayerGrads(dx=_p(dx), dw13=_p(self.dw13), dw2=_p(self.dw2),
                          dw_r=_p(self.dw_r), d_logits=_p(self.d_logits))
        L.call("moe_layer_bwd", C.byref(self.desc), C.byref(prm), C.byref(self._saved),
               _p(dout), C.byref(gr), _p(self.workspace), self.workspace.numel(), _s())
        return dx

    def device_status(self, clear: bool = True) -> int:
        out = C.c_int32(0)
        L.call("moe_read_device_status", _p(self.workspace), int(clear), C.byref(out), _s())
        return int(out.value)


class HostStreamedSteps:
    """Forward + backward steps of a MoELayer on batches held in pinned host
    memory, with each step's host-to-device and device-to-host copies
    overlapped with the compute of the neighbouring steps.

    Two device sets of inputs (x, dOut, and logits in logits mode) and outputs
    (out, dx) alternate between steps; copies in run on one stream, copies out
    on another, the layer on the caller's current stream, ordered by events.
    A step's forward waits only for its forward inputs (x, logits) and its
    backward for dOut, which is still being copied while the forward runs;
    `out` leaves as soon as the forward has written it and `dx` after the
    backward.  Step i's inputs are copied while step i-1 computes.  run()
    returns after enqueueing; the copies and the compute of every step lie
    between work enqueued on the current stream before and after the call."""

    def __init__(self, layer: "MoELayer"):
        self.layer = layer
        dev = layer.workspace.device
        T, d, E = layer.T, layer.d, layer.E
        bf = torch.bfloat16
        self.fwd_names = ["x"] + (["logits"] if layer.router_mode == L.ROUTER_LOGITS else [])
        self.names = self.fwd_names + ["dout"]
        shapes = {"x": ((T, d), bf), "dout": ((T, d), bf), "logits": ((T, E), torch.float32)}
        self.dev_in = [{n: torch.empty(*shapes[n][0], dtype=shapes[n][1], device=dev) for n in self.names}
                       for _ in range(2)]
        self.dev_out = [{"out": torch.empty(T, d, dtype=bf, device=dev),
                         "dx": torch.empty(T, d, dtype=bf, device=dev)} for _ in range(2)]
        self.h2d = torch.cuda.Stream(device=dev)
        self.d2h = torch.cuda.Stream(device=dev)
        mk = lambda: [torch.cuda.Event() for _ in range(2)]  # noqa: E731
        self.fwd_in, self.bwd_in, self.fwd_done, self.done, self.copied = mk(), mk(), mk(), mk(), mk()

    def bytes_per_step(self, host_inputs) -> tuple:
        h2d = sum(host_inputs[n].numel() * host_inputs[n].element_size() for n in self.names)
        d2h = sum(t.numel() * t.element_size() for t in self.dev_out[0].values())
        return h2d, d2h

    def run(self, w13, w2, host_inputs, host_outputs, steps: int, w_r=None):
        """host_inputs[i % len]: dict of pinned tensors (x, dout[, logits]) for
        step i; host_outputs[i % len]: dict of pinned tensors (out, dx)."""
        comp = torch.cuda.current_stream()
        self.h2d.wait_stream(comp)
        self.d2h.wait_stream(comp)

        def copy_in(i):
            b = i % 2
            src = host_inputs[i % len(host_inputs)]
            with torch.cuda.stream(self.h2d):
                if i >= 2:
                    self.h2d.wait_event(self.done[b])  # step i-2 no longer reads set b
                for n in self.fwd_names:
                    self.dev_in[b][n].copy_(src[n], non_blocking=True)
                self.fwd_in[b].record(self.h2d)
                self.dev_in[b]["dout"].copy_(src["dout"], non_blocking=True)
                self.bwd_in[b].record(self.h2d)

        copy_in(0)
        for i in range(steps):
            b = i % 2
            if i + 1 < steps:
                copy_in(i + 1)
            comp.wait_event(self.fwd_in[b])
            if i >= 2:
                comp.wait_event(self.copied[b])  # step i-2's outputs have left set b
            dv, do = self.dev_in[b], self.dev_out[b]
            dst = host_outputs[i % len(host_outputs)]
            lg = dv.get("logits")
            self.layer.forward(dv["x"], w13, w2, logits=lg, w_r=w_r, out=do["out"])
            self.fwd_done[b].record(comp)
            with torch.cuda.stream(self.d2h):
                self.d2h.wait_event(self.fwd_done[b])
                dst["out"].copy_(do["out"], non_blocking=True)
            comp.wait_event(self.bwd_in[b])
            self.layer.backward(dv["dout"], dv["x"], w13, w2, logits=lg, w_r=w_r, dx=do["dx"])
            self.done[b].record(comp)
            with torch.cuda.stream(self.d2h):
                self.d2h.wait_event(self.done[b])
                dst["dx"].copy_(do["dx"], non_blocking=True)
                self.copied[b].record(self.d2h)
        comp.wait_stream(self.h2d)
        comp.wait_stream(self.d2h)
