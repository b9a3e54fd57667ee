"""Pins of the CPU oracle to facts outside itself (no GPU).

Each test ties one oracle function to a closed form, an invariant, a library
routine, a brute-force recomputation or finite differences, chosen so that a
dropped term, a wrong sign or index, or a transposed operand fails one of
them.  Nothing here comes from the CUDA path.
"""
import math

import numpy as np
import pytest
import torch

from oracle import numerics as nm
from oracle import moe as om


# ---------------------------------------------------------------------------
# bf16 and E4M3 / E8M0 numerics
# ---------------------------------------------------------------------------

def test_bf16_round_matches_torch_on_fp32_values():
    g = torch.Generator().manual_seed(1)
    v = torch.randn(200000, generator=g) * torch.exp2(torch.randint(-40, 40, (200000,), generator=g).float())
    # exact halfway cases: low 16 bits = 0x8000 with both parities of bit 16
    base = torch.randint(0, 1 << 30, (4096,), generator=g, dtype=torch.int32)
    half = ((base & ~0xFFFF) | 0x8000).view(torch.float32)
    v = torch.cat([v, half, torch.tensor([0.0, -0.0, 1e-40, -3e-39, 3.0e38])])
    ref = v.to(torch.bfloat16).to(torch.float64).numpy()
    got = nm.round_bf16(v.to(torch.float64).numpy())
    assert np.array_equal(got, ref)
    assert np.array_equal(np.signbit(got), np.signbit(ref))


def test_e4m3_decode_all_codes_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = nm.e4m3_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert set(np.nonzero(nan)[0].tolist()) == {0x7F, 0xFF}
    assert np.array_equal(got[~nan], ref[~nan])


def test_e4m3_anchor_values_from_spec():
    # OFP8 E4M3: max finite 448 = S.1111.110, min normal 2^-6, min subnormal 2^-9, 1.0 = 0.0111.000
    vals = np.array([448.0, 2.0 ** -6, 2.0 ** -9, 1.0, -0.0, 0.0, -448.0, 1000.0, -1e9, 2.0 ** -11])
    want = [0x7E, 0x08, 0x01, 0x38, 0x80, 0x00, 0xFE, 0x7E, 0xFE, 0x00]
    assert nm.e4m3_encode(vals).tolist() == want


def test_e4m3_encode_matches_torch_in_range():
    g = torch.Generator().manual_seed(2)
    v = torch.randn(300000, generator=g, dtype=torch.float64) * torch.exp2(
        torch.randint(-12, 8, (300000,), generator=g).double())
    v = v.clamp(-448.0, 448.0)
    # torch converts fp32 with round-to-nearest-even; feed exactly fp32 values
    v32 = v.float()
    ref = v32.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = nm.e4m3_encode(v32.double().numpy())
    assert np.array_equal(got, ref)


def test_mx_scale_closed_forms():
    # X = floor(log2 amax) - 8, scale byte = X + 127
    blocks = np.array([
        [1.0] + [0.0] * 31,          # amax 1 -> X = -8 -> 119
        [448.0] + [1.0] * 31,        # amax 448 -> X = 0 -> 127
        [0.0] * 32,                  # all zero -> 127, codes 0
        [3.0] * 32,                  # amax 3 -> X = -7; 3 * 2^7 = 384 = 1.5 * 2^8 -> 0x7C
        [-2.0 ** -140] * 32,         # tiny amax -> X clamps to -127 -> 0
        [2.0 ** 140] * 32,           # huge amax -> X clamps to 127 -> 254, value saturates
    ])
    codes, scales = nm.mx_quantize_blocks(blocks)
    assert scales.tolist() == [119, 127, 127, 120, 0, 254]
    assert codes[2].tolist() == [0] * 32
    assert codes[3].tolist() == [0x7C] * 32
    assert codes[5].tolist() == [0x7E] * 32
    assert codes[0][0] == 0x78 and codes[0][1:].tolist() == [0] * 31   # 1 * 2^8 = 256


def test_mx_roundtrip_and_error_bound():
    g = np.random.default_rng(3)
    x = g.standard_normal((64, 32)) * np.exp2(g.integers(-20, 20, (64, 1)))
    codes, scales = nm.mx_quantize_blocks(x)
    deq = nm.mx_dequantize(codes, scales)
    X = scales.astype(np.int64) - 127
    # values are below 2^(X + 9) in magnitude; E4M3 has 4 significant bits:
    # relative error <= 2^-4 for normals, absolute <= 2^(X - 10) below 2^(X - 6),
    # and values above 448 2^X saturate to 448 2^X
    sat = np.abs(x) - 448.0 * np.ldexp(1.0, X)[:, None]
    bound = np.maximum(np.maximum(np.abs(x) * 2.0 ** -4, np.ldexp(1.0, X - 10)[:, None]), sat)
    assert np.all(np.abs(deq - x) <= bound * (1 + 1e-12))
    # exactly representable values survive unchanged
    y = np.array([[2.0 ** j for j in range(-3, 5)] * 4])
    c2, s2 = nm.mx_quantize_blocks(y)
    assert np.array_equal(nm.mx_dequantize(c2, s2), y)


def test_mx_colwise_blocks_restart_at_groups():
    # two groups of 40 and 24 rows with different magnitudes
    g = np.random.default_rng(4)
    a = np.concatenate([g.standard_normal((40, 3)) * 100.0, g.standard_normal((24, 3)) * 0.01])
    codes, scales, base = om.mx_colwise_grouped(a, [0, 40, 64])
    assert base.tolist() == [0, 2]
    assert scales.shape == (3, 3)
    for blk, (r0, r1) in enumerate([(0, 32), (32, 40), (40, 64)]):
        amax = np.max(np.abs(a[r0:r1]), axis=0)
        assert np.array_equal(scales[blk].astype(int) - 127, nm.mx_scale_exponent(amax))
    deq = om.mx_colwise_decoded(a, [0, 40, 64])
    assert np.max(np.abs(deq - a) / np.maximum(np.abs(a), 1e-30)) < 2 ** -3


# ---------------------------------------------------------------------------
# Router
# ---------------------------------------------------------------------------

def test_router_topk_brute_force_sort():
    g = np.random.default_rng(5)
    lg = g.standard_normal((50, 9)).astype(np.float32)
    lg[3, 2] = lg[3, 7]          # an exact tie
    idx, w = om.router_topk(lg, 3)
    for t in range(50):
        order = sorted(range(9), key=lambda e: (-float(lg[t, e]), e))[:3]
        assert idx[t].tolist() == order
        ex = [math.exp(float(lg[t, e]) - float(lg[t, order[0]])) for e in order]
        assert np.allclose(w[t], [v / sum(ex) for v in ex], rtol=0, atol=1e-15)


def test_router_ties_and_signed_zero_go_to_lower_index():
    lg = np.array([[0.0, -0.0, 0.0, -1.0],
                   [-0.0, 0.0, 5.0, 5.0],
                   [1.0, 1.0, 1.0, 1.0]], dtype=np.float32)
    idx, w = om.router_topk(lg, 2)
    assert idx.tolist() == [[0, 1], [2, 3], [0, 1]]
    assert np.allclose(w, 0.5, atol=0)


def test_router_weights_closed_form():
    # logits ln 1..4: top-2 are experts 3, 2 with weights 4/7, 3/7
    lg = np.log(np.array([[1.0, 2.0, 3.0, 4.0]])).astype(np.float32)
    idx, w = om.router_topk(lg, 2)
    assert idx.tolist() == [[3, 2]]
    l = lg.astype(np.float64)[0]
    assert np.allclose(w[0], [1 / (1 + math.exp(l[2] - l[3])), 1 / (1 + math.exp(l[3] - l[2]))])
    assert abs(w[0, 0] - 4 / 7) < 1e-7 and abs(w[0, 1] - 3 / 7) < 1e-7
    # k = E gives the full softmax
    idx, w = om.router_topk(lg, 4)
    assert np.allclose(w[0], np.array([4, 3, 2, 1]) / 10.0, atol=1e-7)


def test_router_weights_sum_to_one():
    g = np.random.default_rng(6)
    lg = (g.standard_normal((400, 32)) * 3).astype(np.float32)
    _, w = om.router_topk(lg, 4)
    assert np.max(np.abs(w.sum(axis=1) - 1.0)) < 1e-12
    assert np.all(np.diff(w, axis=1) <= 0)  # slot order = descending logit


# ---------------------------------------------------------------------------
# Dispatch plan
# ---------------------------------------------------------------------------

def _rand_idx(rng, T, E, k, skew=False):
    p = None
    if skew:
        p = 1.0 / np.arange(1, E + 1) ** 1.2
        p[-2:] = 0
        p /= p.sum()
    return np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)


@pytest.mark.parametrize("skew", [False, True])
def test_dispatch_plan_invariants_and_brute_force(skew):
    rng = np.random.default_rng(7)
    T, E, k = 300, 11, 3
    idx = _rand_idx(rng, T, E, k, skew)
    counts, offsets, dest, src = om.dispatch_plan(idx, E)
    assert counts.sum() == T * k and offsets[0] == 0 and offsets[-1] == T * k
    assert np.all(np.diff(offsets) == counts)
    for e in range(E):
        assert counts[e] == int(np.sum(idx == e))
    # brute force: dest = offsets[e] + #{t' < t : e in topk(t')}
    for t in range(T):
        for i in range(k):
            e = idx[t, i]
            assert dest[t, i] == offsets[e] + int(np.sum(np.any(idx[:t] == e, axis=1)))
            assert src[dest[t, i]] == t
    assert sorted(dest.reshape(-1).tolist()) == list(range(T * k))
    for e in range(E):                            # ascending token order in each expert
        assert np.all(np.diff(src[offsets[e]:offsets[e + 1]]) > 0)
    if skew:
        assert counts[-1] == 0 and counts[-2] == 0
        assert offsets[-1] == offsets[-2] == offsets[-3]


def test_permute_then_unpermute_is_identity():
    rng = np.random.default_rng(8)
    T, E, k, d = 64, 5, 2, 7
    x = rng.standard_normal((T, d))
    idx = _rand_idx(rng, T, E, k)
    _, _, dest, src = om.dispatch_plan(idx, E)
    xp = om.dispatch_rows(x, src)
    for i in range(k):
        assert np.array_equal(xp[dest[:, i]], x)


# ---------------------------------------------------------------------------
# Expert FFN and combine
# ---------------------------------------------------------------------------

def test_swiglu_expert_scalar_closed_form():
    # d = f = 1: g = 1, u = 2, a = silu(1) * 2, y = 3 a ; silu(1) = 1 / (1 + e^-1)
    w13 = np.array([[[1.0], [2.0]]])
    w2 = np.array([[[3.0]]])
    GU, A, Y = om.expert_forward(np.array([[1.0]]), w13, w2, [0, 1], bf16=False)
    assert GU.tolist() == [[1.0, 2.0]]
    assert abs(A[0, 0] - 2 * 0.7310585786300049) < 1e-15
    assert abs(Y[0, 0] - 6 * 0.7310585786300049) < 1e-14


def test_dense_mlp_special_case():
    # E = 1, k = 1: the layer is a dense SwiGLU MLP (weight 1), written as explicit loops
    rng = np.random.default_rng(9)
    T, d, f = 5, 6, 4
    x = rng.standard_normal((T, d))
    w13 = rng.standard_normal((1, 2 * f, d))
    w2 = rng.standard_normal((1, d, f))
    res = om.layer_forward(x, w13, w2, 1, logits32=np.zeros((T, 1), np.float32), bf16=False)
    for t in range(T):
        h = []
        for j in range(f):
            g = sum(x[t, c] * w13[0, j, c] for c in range(d))
            u = sum(x[t, c] * w13[0, f + j, c] for c in range(d))
            h.append(g / (1 + math.exp(-g)) * u)
        for c in range(d):
            y = sum(h[j] * w2[0, c, j] for j in range(f))
            assert abs(res["out"][t, c] - y) < 1e-12


def test_equal_logits_k_equals_E_is_expert_mean():
    rng = np.random.default_rng(10)
    T, d, f, E = 4, 5, 3, 3
    x = rng.standard_normal((T, d))
    w13 = rng.standard_normal((E, 2 * f, d))
    w2 = rng.standard_normal((E, d, f))
    res = om.layer_forward(x, w13, w2, E, logits32=np.full((T, E), 0.25, np.float32), bf16=False)
    ys = []
    for e in range(E):
        one = om.layer_forward(x, w13[e:e + 1], w2[e:e + 1], 1,
                               logits32=np.zeros((T, 1), np.float32), bf16=False)
        ys.append(one["out"])
    assert np.allclose(res["out"], np.mean(ys, axis=0), atol=1e-13)


@pytest.mark.parametrize("bf16", [False, True])
def test_grouped_path_matches_per_token_evaluation(bf16):
    rng = np.random.default_rng(11)
    T, d, f, E, k = 40, 16, 8, 6, 2
    x = om.round_bf16(rng.standard_normal((T, d)))
    w13 = om.round_bf16(rng.standard_normal((E, 2 * f, d)) * 0.2)
    w2 = om.round_bf16(rng.standard_normal((E, d, f)) * 0.2)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    lg[:, E - 1] = -1e4                                       # one empty expert
    res = om.layer_forward(x, w13, w2, k, logits32=lg, bf16=bf16)
    assert res["counts"][E - 1] == 0
    dout = om.round_bf16(rng.standard_normal((T, d)))
    bwd = om.layer_backward(res, dout, x, w13, w2, bf16=bf16)
    assert np.all(bwd["dW13"][E - 1] == 0) and np.all(bwd["dW2"][E - 1] == 0)
    # the two paths sum in different orders: fp64 results agree to rounding,
    # bf16-stored results to one bf16 unit in the last place
    tol = dict(rtol=2.0 ** -7, atol=1e-6) if bf16 else dict(rtol=1e-11, atol=1e-13)
    for t in range(T):
        sel = res["topk_idx"][t]
        ft = om.token_forward(x[t], w13[sel], w2[sel], res["topk_w"][t], bf16)
        assert np.allclose(ft[0], res["out"][t], **tol)
        assert np.allclose(ft[1], res["Y_perm"][res["dest_pos"][t]], **tol)
        dx_t, dw_t, dH_t, _ = om.token_backward(dout[t], x[t], w13[sel], w2[sel],
                                                res["topk_w"][t], ft, bf16)
        assert np.allclose(dw_t, bwd["dw"][t], rtol=1e-6 if bf16 else 1e-11, atol=1e-9)
        assert np.allclose(dH_t, bwd["dH"][res["dest_pos"][t]], **tol)
        assert np.allclose(om.round_bf16(dx_t) if bf16 else dx_t, bwd["dx"][t], **tol)


# ---------------------------------------------------------------------------
# Backward: central finite differences (pure fp64, routing held fixed)
# ---------------------------------------------------------------------------

def _loss(x, w13, w2, wr, dout, k):
    r = om.layer_forward(x, w13, w2, k, wr=wr, bf16=False)
    return float(np.sum(r["out"] * dout)), r["topk_idx"]


def test_backward_finite_differences():
    rng = np.random.default_rng(12)
    T, d, f, E, k = 6, 8, 5, 4, 2
    x = rng.standard_normal((T, d))
    w13 = rng.standard_normal((E, 2 * f, d)) * 0.5
    w2 = rng.standard_normal((E, d, f)) * 0.5
    wr = rng.standard_normal((d, E))
    dout = rng.standard_normal((T, d))
    fwd = om.layer_forward(x, w13, w2, k, wr=wr, bf16=False)
    bwd = om.layer_backward(fwd, dout, x, w13, w2, wr=wr, bf16=False)
    eps = 1e-6
    checks = [("x", x, bwd["dx"]), ("w13", w13, bwd["dW13"]), ("w2", w2, bwd["dW2"]),
              ("wr", wr, bwd["dWr"])]
    for name, arr, grad in checks:
        num = np.zeros_like(arr)
        it = np.nditer(arr, flags=["multi_index"])
        for _ in it:
            ix = it.multi_index
            args = {"x": x, "w13": w13, "w2": w2, "wr": wr}
            p = arr.copy(); p[ix] += eps
            m = arr.copy(); m[ix] -= eps
            args[name] = p
            lp, ip = _loss(args["x"], args["w13"], args["w2"], args["wr"], dout, k)
            args[name] = m
            lm, im = _loss(args["x"], args["w13"], args["w2"], args["wr"], dout, k)
            assert np.array_equal(ip, fwd["topk_idx"]) and np.array_equal(im, fwd["topk_idx"])
            num[ix] = (lp - lm) / (2 * eps)
        err = np.max(np.abs(num - grad)) / max(np.max(np.abs(num)), 1e-30)
        assert err < 1e-6, (name, err)


def test_router_backward_finite_differences_on_logits():
    rng = np.random.default_rng(13)
    T, d, f, E, k = 5, 6, 4, 5, 3
    x = rng.standard_normal((T, d))
    w13 = rng.standard_normal((E, 2 * f, d)) * 0.5
    w2 = rng.standard_normal((E, d, f)) * 0.5
    lg = rng.standard_normal((T, E))
    dout = rng.standard_normal((T, d))

    def loss(l64):
        # evaluate with fp64 logits (selection on the same values)
        idx, _ = om.router_topk(l64.astype(np.float32), k)
        sel = np.take_along_axis(l64, idx.astype(np.int64), axis=1)
        w = np.exp(sel - sel[:, :1]); w /= w.sum(axis=1, keepdims=True)
        r = om.layer_forward(x, w13, w2, k, logits32=l64.astype(np.float32), bf16=False)
        out = om.combine(r["Y_perm"], r["dest_pos"], w, bf16=False)
        return float(np.sum(out * dout))

    fwd = om.layer_forward(x, w13, w2, k, logits32=lg.astype(np.float32), bf16=False)
    _, dw = om.combine_backward(dout, fwd["Y_perm"], fwd["dest_pos"], fwd["topk_w"], bf16=False)
    # weights recomputed from fp64 logits for the check
    sel = np.take_along_axis(lg, fwd["topk_idx"].astype(np.int64), axis=1)
    w = np.exp(sel - sel[:, :1]); w /= w.sum(axis=1, keepdims=True)
    dl = om.router_backward(w, dw, fwd["topk_idx"], E)
    eps = 1e-6
    num = np.zeros_like(lg)
    for t in range(T):
        for e in range(E):
            p = lg.copy(); p[t, e] += eps
            m = lg.copy(); m[t, e] -= eps
            num[t, e] = (loss(p) - loss(m)) / (2 * eps)
    assert np.max(np.abs(num - dl)) < 1e-6 * max(1.0, np.max(np.abs(num)))
    # outside the top-k the gradient is exactly zero
    mask = np.ones_like(lg, bool)
    np.put_along_axis(mask, fwd["topk_idx"].astype(np.int64), False, axis=1)
    assert np.all(dl[mask] == 0)


def test_mxfp8_gemm_is_product_of_decoded_operands():
    # with operands that are exactly representable in MXFP8 the MXFP8 layer
    # equals the exact layer
    rng = np.random.default_rng(14)
    T, d, f, E, k = 8, 32, 32, 2, 1
    pick = np.array([0.5, 1.0, -1.0, 2.0, -0.25, 0.0, 1.5, -3.0])
    x = rng.choice(pick, size=(T, d))
    w13 = rng.choice(pick, size=(E, 2 * f, d)) / 8
    w2 = rng.choice(pick, size=(E, d, f)) / 8
    lg = rng.standard_normal((T, E)).astype(np.float32)
    a = om.layer_forward(x, w13, w2, k, logits32=lg, bf16=False, mx=False)
    b = om.layer_forward(x, w13, w2, k, logits32=lg, bf16=False, mx=True)
    assert np.array_equal(a["GU"], b["GU"])
    # A = silu(G) U is not exactly representable, so later GEMMs differ by the
    # MXFP8 rounding of A only: bounded by 2^-4 relative per element
    rel = np.max(np.abs(a["out"] - b["out"])) / np.sqrt(np.mean(a["out"] ** 2))
    assert 0 < rel < 0.1


# outputs each grouped GEMM feeds, by the chain rule of the forward (router
# logits given, so dx reaches no router term)
_FEEDS = {
    "gemm1": {"GU", "A", "Y_perm", "out", "d_logits", "dH", "dX_perm", "dx", "dW2", "dW13"},
    "gemm2": {"Y_perm", "out", "d_logits"},
    "dA": {"dH", "dX_perm", "dx", "dW13"},
    "dW2": {"dW2"},
    "dX": {"dX_perm", "dx"},
    "dW13": {"dW13"},
}


def _layer_outputs(x, w13, w2, k, lg, dout, mx):
    fwd = om.layer_forward(x, w13, w2, k, logits32=lg, mx=mx)
    bwd = om.layer_backward(fwd, dout, x, w13, w2, mx=mx)
    keys = ("GU", "A", "Y_perm", "out")
    res = {n: fwd[n] for n in keys}
    res.update({n: bwd[n] for n in ("d_logits", "dH", "dX_perm", "dx", "dW2", "dW13")})
    return res


def test_selective_mxfp8_changes_only_what_the_selected_gemm_feeds():
    rng = np.random.default_rng(17)
    T, d, f, E, k = 24, 64, 64, 3, 2
    x = om.round_bf16(rng.standard_normal((T, d)))
    w13 = om.round_bf16(rng.standard_normal((E, 2 * f, d)) * 0.1)
    w2 = om.round_bf16(rng.standard_normal((E, d, f)) * 0.1)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    dout = om.round_bf16(rng.standard_normal((T, d)))
    bf = _layer_outputs(x, w13, w2, k, lg, dout, False)
    # the empty selection is the BF16 layer, the full one the all-MXFP8 layer
    for n, v in _layer_outputs(x, w13, w2, k, lg, dout, set()).items():
        assert np.array_equal(v, bf[n]), n
    allmx = _layer_outputs(x, w13, w2, k, lg, dout, True)
    for n, v in _layer_outputs(x, w13, w2, k, lg, dout, set(om.MX_GEMMS)).items():
        assert np.array_equal(v, allmx[n]), n
    for g in om.MX_GEMMS:
        one = _layer_outputs(x, w13, w2, k, lg, dout, {g})
        for n, v in one.items():
            if n in _FEEDS[g]:
                assert not np.array_equal(v, bf[n]), (g, n)
            else:
                assert np.array_equal(v, bf[n]), (g, n)
    with pytest.raises(ValueError):
        om.layer_forward(x, w13, w2, k, logits32=lg, mx={"gemm3"})


# ---------------------------------------------------------------------------
# Grouped GEMM definitions
# ---------------------------------------------------------------------------

def test_grouped_gemm_ragged_m_brute_force():
    rng = np.random.default_rng(15)
    off = [0, 3, 3, 7]                      # one empty group
    a = rng.standard_normal((9, 4))          # rows 7, 8 belong to no group
    b = rng.standard_normal((3, 5, 4))
    c = om.grouped_gemm_ragged_m(a, b, off)
    cm = om.grouped_gemm_ragged_m(a, np.ascontiguousarray(b.transpose(0, 2, 1)), off, b_mn_major=True)
    assert np.array_equal(c, cm)
    for e in range(3):
        for r in range(off[e], off[e + 1]):
            for n in range(5):
                assert abs(c[r, n] - sum(a[r, q] * b[e, n, q] for q in range(4))) < 1e-12
    assert np.all(c[7:] == 0)


def test_grouped_gemm_ragged_k_brute_force():
    rng = np.random.default_rng(16)
    off = [0, 0, 5, 6]
    a = rng.standard_normal((6, 3))
    b = rng.standard_normal((6, 2))
    c = om.grouped_gemm_ragged_k(a, b, off)
    assert np.all(c[0] == 0)
    for e in range(3):
        ref = np.zeros((3, 2))
        for r in range(off[e], off[e + 1]):
            ref += np.outer(a[r], b[r])
        assert np.allclose(c[e], ref, atol=1e-13)


# ---------------------------------------------------------------------------
# Routing balance
# ---------------------------------------------------------------------------

def test_balance_closed_forms():
    T, E, k = 64, 8, 2
    # equal logits and equal counts: P_e = 1/E, f_e = 1/E -> L = 1; no imbalance
    b = om.router_balance(np.zeros((T, E)), np.full(E, T * k // E), k)
    assert abs(b["aux"] - 1.0) < 1e-12 and b["max_over_mean"] == 1.0 and b["cv"] == 0.0
    # every slot to expert 0 with that expert dominating the softmax: L -> E
    lg = np.full((T, E), -50.0)
    lg[:, 0] = 50.0
    counts = np.zeros(E)
    counts[0] = T * k
    b = om.router_balance(lg, counts, k)
    assert abs(b["aux"] - E) < 1e-9
    assert b["max_over_mean"] == E and b["empty_frac"] == (E - 1) / E


def test_balance_gerrymandering_example():
    # the score can fall while the actual load gets worse: a router that keeps
    # mean probabilities uniform but sends more tokens to one expert
    T, E, k = 200, 4, 1
    rng = np.random.default_rng(17)
    lg = rng.standard_normal((T, E)) * 0.01
    even = om.router_balance(lg, np.full(E, T // E), k)
    skew = om.router_balance(lg, np.array([110, 30, 30, 30]), k)
    assert skew["max_over_mean"] > even["max_over_mean"]
    assert abs(skew["aux"] - even["aux"]) < 1e-2   # the score barely notices


def test_balance_backward_finite_differences():
    rng = np.random.default_rng(18)
    T, E, k = 7, 5, 2
    lg = rng.standard_normal((T, E))
    counts = np.array([4, 0, 3, 5, 2])
    g = om.router_balance_backward(lg, counts, k, scale=0.3)
    eps = 1e-6
    num = np.zeros_like(lg)
    for t in range(T):
        for e in range(E):
            p = lg.copy(); p[t, e] += eps
            m = lg.copy(); m[t, e] -= eps
            num[t, e] = 0.3 * (om.router_balance(p, counts, k)["aux"]
                               - om.router_balance(m, counts, k)["aux"]) / (2 * eps)
    assert np.max(np.abs(num - g)) < 1e-8
