"""CPU oracle of the MoE expert layer, forward and backward (test infrastructure).

Plain numpy fp64.  Matrix products use numpy's ``@`` as a library step; there
is no blocking, fusion or reordering beyond what each definition states.

Notation: T tokens, d model width, E experts, k experts per token, f expert
hidden width, M = T k routed rows.  Weights use the out x in convention:
W13 [E, 2f, d] (rows 0..f-1 are the gate W1, rows f..2f-1 the up projection
W3), W2 [E, d, f], router projection W_r [d, E].

What the pages fix, and the readings taken where they are silent:

* A router sends each token to a small selection of feed-forward experts
  ("Ai2 rebuilds Olmo's training stack for trillion-parameter MoEs",
  introduction; "Supercharging Olmo-core ...", Summary: 4 experts per token).
  Reading: softmax over the E logits, keep the k largest, renormalise over
  them -- equal to a softmax over the k selected logits.  Selection compares
  fp32 logits, larger first, equal values (+0 == -0) go to the lower expert
  index; slot order is selection order.
* Routed token rows are written straight into contiguous per-expert input
  buffers ("Routing work stays on the GPU", first bullet).  Reading: buffers
  are unpadded and back to back in expert order (offsets = exclusive prefix sum
  of counts); inside an expert, rows are in ascending token order.
* Many small expert matmuls are combined into grouped operations (same
  section, third bullet).  Each expert is a SwiGLU FFN: a = silu(x W1^T) *
  (x W3^T), y = a W2^T, silu(z) = z / (1 + exp(-z)).
* The output is the routing-weighted sum of the k expert outputs.
* Stored intermediates are rounded to bf16 where the device stores bf16
  (GU, A, Y_perm, out, dY_perm, dH, dX_perm, dx, dW*); every sum is fp64.
  ``bf16=False`` keeps everything in fp64 (used by the finite-difference pin).
* MXFP8 ("MXFP8 reduces compute and memory costs"): each grouped-GEMM operand
  is quantised to E4M3 with one E8M0 scale per 32 consecutive values along
  that GEMM's reduction axis (blocks restart at every expert boundary), and
  the GEMM runs on the decoded values.  See ``numerics``.  Selective use (same
  section): ``mx`` is either a bool (all six grouped GEMMs or none) or a
  collection of the names in ``MX_GEMMS``; the GEMMs not named run on the
  bf16 operands.
"""
from __future__ import annotations

import numpy as np

from .numerics import round_bf16, mx_quantize_blocks, mx_dequantize

MX_BLOCK = 32
MX_GEMMS = ("gemm1", "gemm2", "dA", "dW2", "dX", "dW13")


def _mx_on(mx, gemm: str) -> bool:
    """Whether grouped GEMM ``gemm`` takes MXFP8 operands under selection ``mx``."""
    if isinstance(mx, (bool, np.bool_)):
        return bool(mx)
    unknown = set(mx) - set(MX_GEMMS)
    if unknown:
        raise ValueError(f"unknown GEMM names {sorted(unknown)}")
    return gemm in mx


def _r(x, bf16: bool):
    return round_bf16(x) if bf16 else np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# Router
# ---------------------------------------------------------------------------

def router_logits(x, wr) -> np.ndarray:
    """logits[t, e] = sum_c x[t, c] W_r[c, e] (fp64)."""
    return np.asarray(x, np.float64) @ np.asarray(wr, np.float64)


def router_topk(logits32, k: int, weight_logits=None):
    """Top-k selection and renormalised weights.

    ``logits32`` are fp32 values (the comparison precision).  For each token the
    experts are ordered by (logit descending, expert index ascending); the first
    k are taken in that order.  Weights (fp64):
        w_i = exp(l_i - l_max) / sum_{j in top-k} exp(l_j - l_max)
    taken on ``logits32`` or, if given, on the unrounded ``weight_logits``.
    Returns (idx int32 [T, k], w fp64 [T, k])."""
    lg = np.asarray(logits32, dtype=np.float32)
    T, E = lg.shape
    # numpy's lexsort is stable and compares keys arithmetically (+0 == -0)
    neg = -lg.astype(np.float64)
    order = np.empty((T, E), dtype=np.int64)
    eidx = np.arange(E)
    for t in range(T):
        order[t] = np.lexsort((eidx, neg[t]))
    idx = order[:, :k].astype(np.int32)
    src = lg if weight_logits is None else weight_logits
    return idx, router_weights(src, idx)


def router_weights(logits, idx):
    """Renormalised weights of a given selection idx [T, k] (slot 0 = largest):
    w_i = exp(l_i - l_0) / sum_j exp(l_j - l_0)   (fp64)."""
    sel = np.take_along_axis(np.asarray(logits, np.float64), np.asarray(idx, np.int64), axis=1)
    ex = np.exp(sel - sel[:, :1])
    return ex / ex.sum(axis=1, keepdims=True)


# ---------------------------------------------------------------------------
# Dispatch plan (counts, offsets, row positions)
# ---------------------------------------------------------------------------

def dispatch_plan(idx, E: int):
    """counts[e] = #{(t, i): idx[t, i] = e}; offsets = exclusive prefix sum with
    offsets[E] = T k; dest_pos[t, i] = offsets[e] + #{t' < t : e in top-k(t')}
    (stable counting sort of the (t, i) pairs by expert); src_token[dest_pos] = t.
    """
    idx = np.asarray(idx, dtype=np.int64)
    T, k = idx.shape
    flat = idx.reshape(-1)
    counts = np.bincount(flat, minlength=E).astype(np.int64)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    order = np.argsort(flat, kind="stable")       # (t, i) pairs grouped by expert
    dest = np.empty(T * k, dtype=np.int64)
    dest[order] = np.arange(T * k)
    src_token = order // k
    return (counts.astype(np.int32), offsets.astype(np.int32),
            dest.reshape(T, k).astype(np.int32), src_token.astype(np.int32))


def dispatch_rows(x, src_token) -> np.ndarray:
    """x_perm[r] = x[src_token[r]] (an exact copy)."""
    return np.asarray(x)[np.asarray(src_token, dtype=np.int64)]


# ---------------------------------------------------------------------------
# MXFP8 helpers (quantise along a GEMM's reduction axis, then decode)
# ---------------------------------------------------------------------------

def mx_rowwise(a):
    """Quantise [R, K] in 1x32 blocks along K; returns (codes, scales [R, ceil(K/32)])."""
    a = np.asarray(a, np.float64)
    R, K = a.shape
    nb = -(-K // MX_BLOCK)
    codes = np.zeros((R, K), np.uint8)
    scales = np.zeros((R, nb), np.uint8)
    for b in range(nb):
        c, s = mx_quantize_blocks(a[:, b * MX_BLOCK:(b + 1) * MX_BLOCK])
        codes[:, b * MX_BLOCK:(b + 1) * MX_BLOCK] = c
        scales[:, b] = s
    return codes, scales


def mx_rowwise_decoded(a) -> np.ndarray:
    codes, scales = mx_rowwise(a)
    K = codes.shape[1]
    out = np.empty(codes.shape, np.float64)
    for b in range(scales.shape[1]):
        out[:, b * MX_BLOCK:(b + 1) * MX_BLOCK] = mx_dequantize(
            codes[:, b * MX_BLOCK:min(K, (b + 1) * MX_BLOCK)], scales[:, b])
    return out


def mx_colwise_grouped(a, offsets):
    """Quantise [R, C] in 32x1 blocks along R; blocks restart at each group
    start offsets[g] and the last block of a group holds its remaining rows.
    Returns (codes [R, C], scales [n_blocks, C], block_base [G]) where the
    block of row r in group g is block_base[g] + (r - offsets[g]) // 32."""
    a = np.asarray(a, np.float64)
    R, C = a.shape
    off = np.asarray(offsets, np.int64)
    G = len(off) - 1
    nblk = [-(-int(off[g + 1] - off[g]) // MX_BLOCK) for g in range(G)]
    base = np.zeros(G, np.int64)
    base[1:] = np.cumsum(nblk)[:-1]
    codes = np.zeros((R, C), np.uint8)
    scales = np.zeros((int(sum(nblk)), C), np.uint8)
    for g in range(G):
        for b in range(nblk[g]):
            r0 = int(off[g]) + b * MX_BLOCK
            r1 = min(int(off[g + 1]), r0 + MX_BLOCK)
            c, s = mx_quantize_blocks(a[r0:r1].T)          # [C, rows]
            codes[r0:r1] = c.T
            scales[base[g] + b] = s
    return codes, scales, base


def mx_colwise_decoded(a, offsets) -> np.ndarray:
    codes, scales, base = mx_colwise_grouped(a, offsets)
    off = np.asarray(offsets, np.int64)
    out = np.zeros(codes.shape, np.float64)
    for g in range(len(off) - 1):
        m = int(off[g + 1] - off[g])
        for b in range(-(-m // MX_BLOCK)):
            r0 = int(off[g]) + b * MX_BLOCK
            r1 = min(int(off[g + 1]), r0 + MX_BLOCK)
            out[r0:r1] = mx_dequantize(codes[r0:r1].T, scales[base[g] + b]).T
    return out


def _q_k_last(a, mx: bool):
    """Operand whose reduction axis is its last axis."""
    return mx_rowwise_decoded(a) if mx else np.asarray(a, np.float64)


def _q_k_first(a, mx: bool, offsets=None):
    """Operand whose reduction axis is its first axis (optionally grouped)."""
    if not mx:
        return np.asarray(a, np.float64)
    if offsets is None:
        offsets = [0, np.asarray(a).shape[0]]
    return mx_colwise_decoded(a, offsets)


# ---------------------------------------------------------------------------
# Expert FFN and combine (forward)
# ---------------------------------------------------------------------------

def silu(z):
    z = np.asarray(z, np.float64)
    return z / (1.0 + np.exp(-z))


def expert_forward(x_perm, w13, w2, offsets, bf16=True, mx=False, preact=None):
    """Per expert e over its rows R_e = [offsets[e], offsets[e+1]):
        G = x_perm[R_e] W1_e^T,  U = x_perm[R_e] W3_e^T        (stored as GU)
        A = silu(G) * U   (from the unrounded G, U)
        Y = A W2_e^T      (A as stored)
    Returns GU [M, 2f], A [M, f], Y [M, d]."""
    x_perm = np.asarray(x_perm, np.float64)
    E, f2, d = w13.shape
    f = f2 // 2
    M = x_perm.shape[0]
    GU = np.zeros((M, 2 * f))
    A = np.zeros((M, f))
    Y = np.zeros((M, d))
    m1, m2 = _mx_on(mx, "gemm1"), _mx_on(mx, "gemm2")
    xq = _q_k_last(x_perm, m1)
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 == r0:
            continue
        W = _q_k_last(np.asarray(w13[e], np.float64), m1)
        gu = xq[r0:r1] @ W.T
        if preact is not None:
            preact[r0:r1] = gu                 # unrounded [G | U], for callers that need it
        GU[r0:r1] = _r(gu, bf16)
        A[r0:r1] = _r(silu(gu[:, :f]) * gu[:, f:], bf16)
    Aq = _q_k_last(A, m2)
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 == r0:
            continue
        W2e = _q_k_last(np.asarray(w2[e], np.float64), m2)
        Y[r0:r1] = _r(Aq[r0:r1] @ W2e.T, bf16)
    return GU, A, Y


def combine(y_perm, dest_pos, w, bf16=True):
    """out[t] = sum_{i < k} w[t, i] Y_perm[dest_pos[t, i]]."""
    y_perm = np.asarray(y_perm, np.float64)
    dest = np.asarray(dest_pos, np.int64)
    w = np.asarray(w, np.float64)
    out = np.zeros((dest.shape[0], y_perm.shape[1]))
    for i in range(dest.shape[1]):
        out += w[:, i:i + 1] * y_perm[dest[:, i]]
    return _r(out, bf16)


# ---------------------------------------------------------------------------
# Backward (chain rule of the forward above; loss gradient dOut = dL/dout)
# ---------------------------------------------------------------------------

def combine_backward(dout, y_perm, dest_pos, w, bf16=True):
    """dY_perm[dest_pos[t, i]] = w[t, i] dOut[t];
    dw[t, i] = sum_c dOut[t, c] Y_perm[dest_pos[t, i], c]."""
    dout = np.asarray(dout, np.float64)
    y_perm = np.asarray(y_perm, np.float64)
    dest = np.asarray(dest_pos, np.int64)
    w = np.asarray(w, np.float64)
    T, k = dest.shape
    dY = np.zeros_like(y_perm)
    dw = np.zeros((T, k))
    for i in range(k):
        dY[dest[:, i]] = w[:, i:i + 1] * dout
        dw[:, i] = np.sum(dout * y_perm[dest[:, i]], axis=1)
    return _r(dY, bf16), dw


def swiglu_backward(dA, G, U):
    """With s = sigmoid(G):  dG = dA U s (1 + G (1 - s)),  dU = dA silu(G)."""
    G = np.asarray(G, np.float64)
    U = np.asarray(U, np.float64)
    s = 1.0 / (1.0 + np.exp(-G))
    return dA * U * s * (1.0 + G * (1.0 - s)), dA * G * s


def expert_backward(dY_perm, GU, A, x_perm, w13, w2, offsets, bf16=True, mx=False, dA_out=None):
    """Per expert e over R_e:
        dA   = dY W2_e;           [dG | dU] = swiglu_backward(dA, G, U)   (dH)
        dW2_e  = dY^T A;          dX_perm = dH W13_e;    dW13_e = dH^T x_perm
    An expert with no rows gets dW2_e = dW13_e = 0.
    Returns dH [M, 2f], dW2 [E, d, f], dX_perm [M, d], dW13 [E, 2f, d]."""
    dY = np.asarray(dY_perm, np.float64)
    GU = np.asarray(GU, np.float64)
    A = np.asarray(A, np.float64)
    xp = np.asarray(x_perm, np.float64)
    E, f2, d = w13.shape
    f = f2 // 2
    M = dY.shape[0]
    dH = np.zeros((M, 2 * f))
    dX = np.zeros((M, d))
    dW2 = np.zeros((E, d, f))
    dW13 = np.zeros((E, 2 * f, d))
    mA, mW2, mX, mW13 = (_mx_on(mx, g) for g in ("dA", "dW2", "dX", "dW13"))
    dYq = _q_k_last(dY, mA)                                  # dA: reduce over d
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 == r0:
            continue
        W2e = _q_k_first(np.asarray(w2[e], np.float64), mA)  # [d, f], reduce over d
        dA = dYq[r0:r1] @ W2e
        if dA_out is not None:
            dA_out[r0:r1] = dA
        dG, dU = swiglu_backward(dA, GU[r0:r1, :f], GU[r0:r1, f:])
        dH[r0:r1, :f] = _r(dG, bf16)
        dH[r0:r1, f:] = _r(dU, bf16)
    dHq = _q_k_last(dH, mX)                                  # dX: reduce over 2f
    # dW GEMMs reduce over the rows of each expert
    dYg = _q_k_first(dY, mW2, offsets)
    Ag = _q_k_first(A, mW2, offsets)
    dHg = _q_k_first(dH, mW13, offsets)
    xg = _q_k_first(xp, mW13, offsets)
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 == r0:
            continue
        W13e = _q_k_first(np.asarray(w13[e], np.float64), mX)  # [2f, d], reduce over 2f
        dX[r0:r1] = _r(dHq[r0:r1] @ W13e, bf16)
        dW2[e] = _r(dYg[r0:r1].T @ Ag[r0:r1], bf16)
        dW13[e] = _r(dHg[r0:r1].T @ xg[r0:r1], bf16)
    return dH, dW2, dX, dW13


def router_backward(w, dw, idx, E: int):
    """Softmax-over-top-k Jacobian: for j in top-k(t)
        d_logits[t, idx[t, j]] = w_j (dw_j - sum_i w_i dw_i),
    and 0 for experts outside the top-k (selection is piecewise constant)."""
    w = np.asarray(w, np.float64)
    dw = np.asarray(dw, np.float64)
    idx = np.asarray(idx, np.int64)
    T, k = idx.shape
    dl = np.zeros((T, E))
    inner = np.sum(w * dw, axis=1, keepdims=True)
    np.put_along_axis(dl, idx, w * (dw - inner), axis=1)
    return dl


def unpermute_sum(dX_perm, dest_pos, extra=None, bf16=True):
    """dx[t] = sum_i dX_perm[dest_pos[t, i]] (+ extra[t])."""
    dX = np.asarray(dX_perm, np.float64)
    dest = np.asarray(dest_pos, np.int64)
    dx = np.zeros((dest.shape[0], dX.shape[1]))
    for i in range(dest.shape[1]):
        dx += dX[dest[:, i]]
    if extra is not None:
        dx += extra
    return _r(dx, bf16)


def router_proj_backward(x, wr, d_logits):
    """For logits = x W_r:  dx_router = d_logits W_r^T,  dW_r = x^T d_logits."""
    dl = np.asarray(d_logits, np.float64)
    return dl @ np.asarray(wr, np.float64).T, np.asarray(x, np.float64).T @ dl


# ---------------------------------------------------------------------------
# Whole layer
# ---------------------------------------------------------------------------

def layer_forward(x, w13, w2, k, logits32=None, wr=None, bf16=True, mx=False):
    """Forward pass.  Routing is decided on fp32 logits: either given
    (``logits32``) or x W_r computed in fp64 and rounded to fp32.  The weights
    use the fp32 logits, except in pure fp64 mode (``bf16=False``) with a
    projection, where they use the fp64 logits."""
    x = np.asarray(x, np.float64)
    E = w13.shape[0]
    res = {}
    wl = None
    if logits32 is None:
        lg64 = router_logits(x, wr)
        res["logits"] = lg64
        logits32 = lg64.astype(np.float32)
        wl = None if bf16 else lg64
    idx, w = router_topk(logits32, k, wl)
    counts, offsets, dest, src = dispatch_plan(idx, E)
    x_perm = dispatch_rows(x, src)
    GU, A, Y = expert_forward(x_perm, w13, w2, offsets, bf16, mx)
    out = combine(Y, dest, w, bf16)
    res.update(topk_idx=idx, topk_w=w, counts=counts, offsets=offsets, dest_pos=dest,
               src_token=src, x_perm=x_perm, GU=GU, A=A, Y_perm=Y, out=out)
    return res


def layer_backward(fwd, dout, x, w13, w2, wr=None, bf16=True, mx=False):
    """Backward pass from the forward record ``fwd`` and dOut = dL/dout."""
    E = w13.shape[0]
    dY, dw = combine_backward(dout, fwd["Y_perm"], fwd["dest_pos"], fwd["topk_w"], bf16)
    dH, dW2, dX, dW13 = expert_backward(dY, fwd["GU"], fwd["A"], fwd["x_perm"], w13, w2,
                                        fwd["offsets"], bf16, mx)
    dl = router_backward(fwd["topk_w"], dw, fwd["topk_idx"], E)
    res = dict(dY_perm=dY, dw=dw, dH=dH, dW2=dW2, dX_perm=dX, dW13=dW13, d_logits=dl)
    extra = None
    if wr is not None:
        dx_r, dWr = router_proj_backward(x, wr, dl)
        extra = dx_r
        res["dWr"] = _r(dWr, bf16)
    res["dx"] = unpermute_sum(dX, fwd["dest_pos"], extra, bf16)
    return res


# ---------------------------------------------------------------------------
# Per-token evaluation (no permutation): used for sampled checks at full size
# and as a brute-force pin of the grouped path.
# ---------------------------------------------------------------------------

def token_forward(x_t, w13_sel, w2_sel, w_t, bf16=True):
    """One token through its k experts without any dispatch:
    out = sum_i w_i y_i with y_i = (silu(x W1^T) * (x W3^T)) W2^T of expert i.
    ``w13_sel`` [k, 2f, d] and ``w2_sel`` [k, d, f] are the token's experts in
    slot order.  Returns (out [d], y [k, d], gu [k, 2f], a [k, f])."""
    x_t = np.asarray(x_t, np.float64)
    k, f2, d = w13_sel.shape
    f = f2 // 2
    ys, gus, as_ = [], [], []
    for i in range(k):
        gu = np.asarray(w13_sel[i], np.float64) @ x_t
        a = _r(silu(gu[:f]) * gu[f:], bf16)
        y = _r(np.asarray(w2_sel[i], np.float64) @ a, bf16)
        ys.append(y)
        gus.append(_r(gu, bf16))
        as_.append(a)
    ys = np.stack(ys)
    out = _r(np.sum(np.asarray(w_t, np.float64)[:, None] * ys, axis=0), bf16)
    return out, ys, np.stack(gus), np.stack(as_)


def expert_preactivation(x_t, w13_e):
    """[G | U] of one token and one expert before any rounding: W13_e x (fp64)."""
    return np.asarray(w13_e, np.float64) @ np.asarray(x_t, np.float64)


def token_backward(dout_t, x_t, w13_sel, w2_sel, w_t, fwd_tok, bf16=True):
    """Backward of ``token_forward`` for one token: returns (dx_experts [d]
    (sum over its slots of dX rows), dw [k], dH [k, 2f], dY [k, d])."""
    dout_t = np.asarray(dout_t, np.float64)
    _, ys, gus, _ = fwd_tok
    k, f2, d = w13_sel.shape
    f = f2 // 2
    dx = np.zeros(d)
    dws, dHs, dYs = [], [], []
    for i in range(k):
        dY = _r(w_t[i] * dout_t, bf16)
        dws.append(float(np.sum(dout_t * ys[i])))
        dA = np.asarray(w2_sel[i], np.float64).T @ dY
        dG, dU = swiglu_backward(dA, gus[i][:f], gus[i][f:])
        dH = np.concatenate([_r(dG, bf16), _r(dU, bf16)])
        dx += _r(np.asarray(w13_sel[i], np.float64).T @ dH, bf16)
        dHs.append(dH)
        dYs.append(dY)
    return dx, np.array(dws), np.stack(dHs), np.stack(dYs)


# ---------------------------------------------------------------------------
# Grouped GEMM definitions (the two shapes the layer's matmuls take)
# ---------------------------------------------------------------------------

def grouped_gemm_ragged_m(a, b, offsets, b_mn_major=False):
    """For each group e with rows R_e = [offsets[e], offsets[e+1]):
    C[R_e] = A[R_e] B_e^T, where B_e is [N, K] (or stored [K, N] when
    ``b_mn_major``).  Rows outside every group stay zero."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    E = b.shape[0]
    N = b.shape[2] if b_mn_major else b.shape[1]
    c = np.zeros((a.shape[0], N))
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        be = b[e].T if b_mn_major else b[e]
        c[r0:r1] = a[r0:r1] @ be.T
    return c


def grouped_gemm_ragged_k(a, b, offsets):
    """For each group e: C_e = A[R_e]^T B[R_e] (a sum over the group's rows);
    an empty group gives zeros."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    E = len(offsets) - 1
    c = np.zeros((E, a.shape[1], b.shape[1]))
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        c[e] = a[r0:r1].T @ b[r0:r1]
    return c


# ---------------------------------------------------------------------------
# Routing balance ("Ai2 rebuilds Olmo's training stack for trillion-parameter
# MoEs", "Four failure modes from the report", first bullet: a routing-balance
# score can improve while the actual load gets less balanced).  The pages name
# no formula; reading: the common auxiliary balance loss
#     L = E * sum_e f_e P_e,   f_e = counts_e / (T k),   P_e = mean_t softmax(l_t)_e,
# (1 for a perfectly balanced router) next to the actual imbalance of the
# counts: max_e counts_e / mean_e counts_e and their coefficient of variation.
# ---------------------------------------------------------------------------

def softmax_rows(logits):
    l = np.asarray(logits, np.float64)
    z = np.exp(l - l.max(axis=1, keepdims=True))
    return z / z.sum(axis=1, keepdims=True)


def router_balance(logits, counts, k):
    """Returns dict(aux, max_over_mean, cv, empty_frac, P, f)."""
    counts = np.asarray(counts, np.float64)
    T, E = np.asarray(logits).shape
    p = softmax_rows(logits)
    P = p.mean(axis=0)
    f = counts / (T * k)
    mean = counts.mean()
    return dict(aux=float(E * np.sum(f * P)), max_over_mean=float(counts.max() / mean),
                cv=float(counts.std() / mean), empty_frac=float(np.mean(counts == 0)), P=P, f=f)


def router_balance_backward(logits, counts, k, scale=1.0):
    """d(scale * L)/d logits with the counts held fixed (selection is piecewise
    constant):  scale * (E / T) * p_tj * (f_j - sum_e f_e p_te)."""
    T, E = np.asarray(logits).shape
    p = softmax_rows(logits)
    f = np.asarray(counts, np.float64) / (T * k)
    inner = p @ f
    return scale * (E / T) * p * (f[None, :] - inner[:, None])
