"""Pins of the C oracle (``oracle/moe_ref.c``) and its agreement with the numpy
oracle (CPU only).

The C oracle restates the layer with plain fp64 loops per token and selected
expert, its own bf16 rounding (on the fp64 bit pattern) and its own E4M3
encoder (the nearest entry of the code table).  It is pinned here to library
conversions (torch's bf16 and float8_e4m3fn), closed forms, invariants, the
dense special case and finite differences; then both oracles must agree: the
integer outputs exactly, every stored bf16 tensor bit for bit (two fp64
evaluations that differ by ~1e-16 round to different bf16 values only within
~1e-16 of a rounding midpoint), unrounded values to fp64 precision.
"""
import numpy as np
import pytest
import torch

from oracle import moe as om
from oracle import ref_c as rc
from routing_grouped_gemm_moe_b200 import inputs as I


def f64(t):
    return t.float().double().numpy()


# ------------------------------------------------------------------ number formats

def test_c_round_bf16_matches_torch_on_fp32_values():
    """All fp32 classes: normals, subnormals, near-overflow, exact ties."""
    rng = np.random.default_rng(11)
    bits = rng.integers(0, 0x7F800000, size=200000, dtype=np.int64).astype(np.uint32)
    bits[:4096] = np.arange(4096, dtype=np.uint32)                 # fp32 subnormals
    bits[4096:8192] = 0x7F7FF000 + np.arange(4096, dtype=np.uint32)  # next to FLT_MAX
    bits[8192:12288] = (bits[8192:12288] & 0xFFFF0000) | 0x8000     # exact bf16 ties
    v = bits.view(np.float32)
    v = np.where(rng.random(v.size) < 0.5, -v, v).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).double().numpy()
    got = rc.round_bf16(v.astype(np.float64))
    assert np.array_equal(got, ref, equal_nan=True)
    assert np.array_equal(np.signbit(got), np.signbit(ref))


def test_c_e4m3_decode_all_codes_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    got = rc.e4m3_decode(codes)
    assert np.array_equal(got, ref, equal_nan=True)
    assert np.isnan(got[0x7F]) and np.isnan(got[0xFF])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6


def test_c_e4m3_encode_matches_torch_in_range():
    """|v| <= 448 (torch's cast does not saturate beyond), ties included."""
    rng = np.random.default_rng(12)
    v = np.concatenate([rng.uniform(-448, 448, 50000), rng.normal(0, 2.0 ** -7, 50000),
                        rc.e4m3_decode(np.arange(0x7E)) * (1 + 2.0 ** -5)])  # halfway points
    v = v.astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = rc.e4m3_encode(v.astype(np.float64))
    assert np.array_equal(got, ref)
    assert rc.e4m3_encode(np.array([500.0, -1e9]))[0] == 0x7E          # satfinite
    assert rc.e4m3_encode(np.array([-1e-12]))[0] == 0x80                 # sign of zero kept


def test_c_mx_scale_closed_forms():
    """X = floor(log2 amax) - 8; byte X + 127; all-zero block -> byte 127."""
    a = np.zeros((4, 64))
    a[0, 0] = 1.0                  # X = -8, 1 * 2^8 = 256 = code 0x78
    a[1, 5] = -3.0                 # floor(log2 3) = 1 -> X = -7; -3 * 2^7 = -384 = 0xFC
    a[2, 40] = 2.0 ** -130         # X clamped to -127
    codes, scales = rc.mx_rowwise(a)
    assert scales[0, 0] == 119 and codes[0, 0] == 0x78
    assert scales[1, 0] == 120 and codes[1, 5] == 0xFC
    assert scales[2, 1] == 0 and scales[3, 0] == 127 and scales[3, 1] == 127
    assert np.all(codes[3] == 0)


# ------------------------------------------------------------------ layer pins

def _tiny(T=6, d=32, E=4, k=2, f=32, seed=3, proj=True):
    rng = np.random.default_rng(seed)
    x = rng.normal(0, 1, (T, d))
    w13 = rng.normal(0, 0.2, (E, 2 * f, d))
    w2 = rng.normal(0, 0.2, (E, d, f))
    wr = rng.normal(0, 0.5, (d, E)) if proj else None
    dout = rng.normal(0, 1, (T, d))
    return x, w13, w2, wr, dout


def test_c_dispatch_invariants():
    cfg = I.LayerConfig("z", T=300, d=64, E=6, k=3, f=64, logits="zipf", n_empty=1, zipf_s=0.8,
                        seed=81)
    inp = I.make_inputs(cfg)
    x = f64(inp["x"])
    r = rc.layer_forward(x, f64(inp["w13"]), f64(inp["w2"]), cfg.k, logits32=inp["logits"].numpy())
    T, k = cfg.T, cfg.k
    assert r["counts"].sum() == T * k and np.any(r["counts"] == 0)
    assert np.array_equal(np.diff(r["offsets"]), r["counts"])
    dest = r["dest_pos"].reshape(-1)
    assert np.array_equal(np.sort(dest), np.arange(T * k))                # a permutation
    assert np.array_equal(r["src_token"][dest], np.repeat(np.arange(T), k))
    assert np.array_equal(r["x_perm"][r["dest_pos"]], np.broadcast_to(x[:, None], (T, k, cfg.d)))
    np.testing.assert_allclose(r["topk_w"].sum(axis=1), 1.0, rtol=0, atol=1e-15)
    for e in range(cfg.E):           # rows of one expert in ascending token order
        toks = r["src_token"][r["offsets"][e]:r["offsets"][e + 1]]
        assert np.all(np.diff(toks) > 0)


def test_c_router_ties_go_to_lower_index():
    T, E, k, d, f = 3, 5, 2, 32, 32
    lg = np.array([[1.0, 3.0, 3.0, 0.0, 3.0],
                   [0.0, -0.0, 0.0, -1.0, -2.0],
                   [-5.0, -5.0, -4.0, -4.0, -6.0]], np.float32)
    x, w13, w2, _, _ = _tiny(T, d, E, k, f, proj=False)
    r = rc.layer_forward(x, w13, w2, k, logits32=lg)
    assert r["topk_idx"].tolist() == [[1, 2], [0, 1], [2, 3]]
    np.testing.assert_allclose(r["topk_w"], 0.5, rtol=0, atol=1e-16)


def test_c_dense_special_case():
    """E = k = 1: every token through one SwiGLU MLP, weight 1 (fp64 mode),
    against torch's fp64 matmul."""
    x, w13, w2, _, _ = _tiny(T=9, d=32, E=1, k=1, f=48, proj=False)
    r = rc.layer_forward(x, w13, w2, 1, logits32=np.zeros((9, 1), np.float32), bf16=False)
    xt, w13t, w2t = (torch.from_numpy(a) for a in (x, w13[0], w2[0]))
    gu = xt @ w13t.T
    ref = (torch.nn.functional.silu(gu[:, :48]) * gu[:, 48:]) @ w2t.T
    np.testing.assert_allclose(r["out"], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_c_backward_finite_differences():
    """fp64 mode, router projection: dL/d(x, W13, W2, W_r) of L = <out, dOut>
    against central differences (steps small enough to keep the selection)."""
    x, w13, w2, wr, dout = _tiny()
    k = 2

    def loss(x_, w13_, w2_, wr_):
        r = rc.layer_forward(x_, w13_, w2_, k, wr=wr_, bf16=False)
        return float(np.sum(r["out"] * dout)), r["topk_idx"]

    fwd = rc.layer_forward(x, w13, w2, k, wr=wr, bf16=False)
    bwd = rc.layer_backward(fwd, dout, x, w13, w2, wr=wr, bf16=False)
    rng = np.random.default_rng(5)
    h = 1e-6
    for name, arr, grad in (("x", x, bwd["dx"]), ("w13", w13, bwd["dW13"]),
                            ("w2", w2, bwd["dW2"]), ("wr", wr, bwd["dWr"])):
        for _ in range(12):
            i = tuple(rng.integers(0, s) for s in arr.shape)
            args = dict(x_=x, w13_=w13, w2_=w2, wr_=wr)
            key = {"x": "x_", "w13": "w13_", "w2": "w2_", "wr": "wr_"}[name]
            p, m = arr.copy(), arr.copy()
            p[i] += h
            m[i] -= h
            lp, ip = loss(**{**args, key: p})
            lm, im = loss(**{**args, key: m})
            assert np.array_equal(ip, fwd["topk_idx"]) and np.array_equal(im, fwd["topk_idx"])
            fd = (lp - lm) / (2 * h)
            assert abs(fd - grad[i]) <= 1e-6 * max(1.0, abs(fd)), (name, i, fd, grad[i])


# ------------------------------------------------------------------ agreement with numpy

CASES = {
    "tiny_proj": (I.CONFIGS["tiny"], False),
    "zipf_empty": (I.LayerConfig("z", T=300, d=256, E=6, k=2, f=384, logits="zipf", n_empty=1,
                                 zipf_s=0.8, seed=71), False),
    "mx_proj": (I.LayerConfig("m", T=200, d=128, E=8, k=2, f=256, router="proj", dtype="mxfp8",
                              seed=76), True),
    "mx_selective": (I.LayerConfig("mz", T=300, d=256, E=6, k=2, f=384, logits="zipf", n_empty=1,
                                   zipf_s=0.8, dtype="mxfp8", seed=75), ("gemm2", "dA", "dW13")),
    "one_token": (I.LayerConfig("o", T=1, d=64, E=4, k=2, f=64, seed=73), False),
}
INT_KEYS = ("topk_idx", "counts", "offsets", "dest_pos", "src_token")
BF16_FWD = ("GU", "A", "Y_perm", "out")
BF16_BWD = ("dY_perm", "dH", "dX_perm", "dW2", "dW13", "dx", "dWr")
F64_FWD = ("topk_w",)
F64_BWD = ("dw", "d_logits")


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("bf16", [True, False])
def test_c_oracle_matches_numpy_oracle(name, bf16):
    cfg, mx = CASES[name]
    inp = I.make_inputs(cfg)
    x, w13, w2, dout = (f64(inp[n]) for n in ("x", "w13", "w2", "dout"))
    wr = f64(inp["wr"]) if "wr" in inp else None
    lg = inp["logits"].numpy() if "logits" in inp else None
    a = om.layer_forward(x, w13, w2, cfg.k, logits32=lg, wr=wr, bf16=bf16, mx=mx)
    ab = om.layer_backward(a, dout, x, w13, w2, wr=wr, bf16=bf16, mx=mx)
    b = rc.layer_forward(x, w13, w2, cfg.k, logits32=lg, wr=wr, bf16=bf16, mx=mx)
    bb = rc.layer_backward(b, dout, x, w13, w2, wr=wr, bf16=bf16, mx=mx)
    for key in INT_KEYS:
        assert np.array_equal(a[key], b[key]), key

    def rel(u, v):
        u, v = np.asarray(u), np.asarray(v)
        rms = np.sqrt(np.mean(u * u)) if u.size else 0.0
        return 0.0 if rms == 0 else float(np.max(np.abs(u - v)) / rms)

    for key in F64_FWD:
        assert rel(a[key], b[key]) <= 1e-14, key
    for key in F64_BWD:
        assert rel(ab[key], bb[key]) <= 1e-13, key
    for src, dst, keys in ((a, b, BF16_FWD), (ab, bb, BF16_BWD)):
        for key in keys:
            if key not in src:
                continue
            if bf16:
                assert np.array_equal(src[key], dst[key]), key
            else:
                assert rel(src[key], dst[key]) <= 1e-12, key
