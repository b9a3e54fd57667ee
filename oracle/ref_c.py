"""ctypes binding of the C oracle ``moe_ref.c`` (test infrastructure).

The C oracle is a second statement of the layer, written independently of the
numpy one in ``moe``: per token and per selected expert with plain fp64 loops,
its own bf16 rounding (on the fp64 bit pattern) and its own E4M3 encoder (the
nearest entry of the decoded code table).  ``layer_forward`` and
``layer_backward`` take and return the same arrays, under the same names, as
``moe.layer_forward`` / ``moe.layer_backward``.

The shared object is built from source by ``make`` in this directory when it
is missing or older than the source.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

from .moe import MX_GEMMS, _mx_on

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_ref.c")
_SO = os.path.join(_HERE, "libmoe_ref.so")
_lib = None


class Shape(C.Structure):
    _fields_ = [("T", C.c_int), ("d", C.c_int), ("E", C.c_int), ("k", C.c_int), ("f", C.c_int),
                ("round_bf16", C.c_int), ("mx", C.c_uint)]


def build() -> str:
    """Compile ``libmoe_ref.so`` if it is missing or stale; returns its path."""
    if not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        subprocess.run(["make", "-s", "-C", _HERE, "libmoe_ref.so"], check=True)
    return _SO


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        _lib.moe_ref_forward.restype = C.c_int
        _lib.moe_ref_backward.restype = C.c_int
        for name in ("moe_ref_round_bf16", "moe_ref_e4m3_decode", "moe_ref_e4m3_encode",
                     "moe_ref_mx_rowwise"):
            getattr(_lib, name).restype = None
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def mx_bits(mx) -> int:
    """Bit g set when grouped GEMM MX_GEMMS[g] runs on MXFP8 operands."""
    return sum(1 << g for g, name in enumerate(MX_GEMMS) if _mx_on(mx, name))


def _shape(T, d, E, k, f, bf16, mx):
    return Shape(T, d, E, k, f, 1 if bf16 else 0, mx_bits(mx))


def layer_forward(x, w13, w2, k, logits32=None, wr=None, bf16=True, mx=False):
    """The layer forward; see ``moe.layer_forward`` for the arguments and keys."""
    x, w13, w2, wr = _f64(x), _f64(w13), _f64(w2), _f64(wr)
    T, d = x.shape
    E, f2, _ = w13.shape
    f = f2 // 2
    M = T * k
    lg_in = None if logits32 is None else np.ascontiguousarray(logits32, dtype=np.float32)
    r = dict(topk_idx=np.zeros((T, k), np.int32), topk_w=np.zeros((T, k)),
             counts=np.zeros(E, np.int32), offsets=np.zeros(E + 1, np.int32),
             dest_pos=np.zeros((T, k), np.int32), src_token=np.zeros(M, np.int32),
             GU=np.zeros((M, f2)), A=np.zeros((M, f)), Y_perm=np.zeros((M, d)),
             out=np.zeros((T, d)))
    logits = np.zeros((T, E)) if lg_in is None else None
    s = _shape(T, d, E, k, f, bf16, mx)
    rc = lib().moe_ref_forward(
        C.byref(s), _p(x), _p(lg_in), _p(wr), _p(w13), _p(w2), _p(logits),
        *(_p(r[n]) for n in ("topk_idx", "topk_w", "counts", "offsets", "dest_pos",
                             "src_token", "GU", "A", "Y_perm", "out")))
    if rc != 0:
        raise RuntimeError(f"moe_ref_forward failed with status {rc}")
    if logits is not None:
        r["logits"] = logits
    r["x_perm"] = x[r["src_token"].astype(np.int64)]
    return r


def layer_backward(fwd, dout, x, w13, w2, wr=None, bf16=True, mx=False):
    """The layer backward; see ``moe.layer_backward`` for the arguments and keys."""
    x, w13, w2, wr, dout = _f64(x), _f64(w13), _f64(w2), _f64(wr), _f64(dout)
    T, d = x.shape
    E, f2, _ = w13.shape
    f = f2 // 2
    k = fwd["topk_idx"].shape[1]
    M = T * k
    rec = {n: np.ascontiguousarray(fwd[n], dtype=np.int32)
           for n in ("topk_idx", "offsets", "dest_pos", "src_token")}
    rec.update({n: _f64(fwd[n]) for n in ("topk_w", "GU", "A", "Y_perm")})
    r = dict(dY_perm=np.zeros((M, d)), dw=np.zeros((T, k)), dH=np.zeros((M, f2)),
             dX_perm=np.zeros((M, d)), dW2=np.zeros((E, d, f)), dW13=np.zeros((E, f2, d)),
             d_logits=np.zeros((T, E)), dx=np.zeros((T, d)))
    dwr = np.zeros((d, E)) if wr is not None else None
    s = _shape(T, d, E, k, f, bf16, mx)
    rc = lib().moe_ref_backward(
        C.byref(s), _p(x), _p(wr), _p(w13), _p(w2), _p(dout),
        *(_p(rec[n]) for n in ("topk_idx", "topk_w", "offsets", "dest_pos", "src_token",
                               "GU", "A", "Y_perm")),
        *(_p(r[n]) for n in ("dY_perm", "dw", "dH", "dX_perm", "dW2", "dW13", "d_logits", "dx")),
        _p(dwr))
    if rc != 0:
        raise RuntimeError(f"moe_ref_backward failed with status {rc}")
    if dwr is not None:
        r["dWr"] = dwr
    return r


def round_bf16(x) -> np.ndarray:
    x = _f64(np.atleast_1d(x))
    out = np.empty_like(x)
    lib().moe_ref_round_bf16(_p(x), C.c_int64(x.size), _p(out))
    return out


def e4m3_decode(codes) -> np.ndarray:
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, np.float64)
    lib().moe_ref_e4m3_decode(_p(c), C.c_int64(c.size), _p(out))
    return out


def e4m3_encode(v) -> np.ndarray:
    v = _f64(np.atleast_1d(v))
    out = np.empty(v.shape, np.uint8)
    lib().moe_ref_e4m3_encode(_p(v), C.c_int64(v.size), _p(out))
    return out


def mx_rowwise(a):
    """(codes [R, K], scale bytes [R, ceil(K / 32)]) of blocks of 32 along each row."""
    a = _f64(a)
    R, K = a.shape
    codes = np.empty((R, K), np.uint8)
    scales = np.empty((R, -(-K // 32)), np.uint8)
    lib().moe_ref_mx_rowwise(_p(a), C.c_int64(R), C.c_int64(K), _p(codes), _p(scales))
    return codes, scales
