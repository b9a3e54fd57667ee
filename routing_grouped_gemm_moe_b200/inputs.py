"""Seeded synthetic inputs for the MoE expert layer.

This module only draws numbers; it holds none of the layer's arithmetic.  It
is shared by the tests, the benchmark and the CPU checker so that every side
sees identical bytes.

Generator (counter based, device independent):

* ``splitmix64`` (Steele, Lea & Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014) turns a per-tensor key plus the element's flat
  index into 64 random bits.  Only wrapping 64-bit integer arithmetic is used,
  so a CPU tensor and a CUDA tensor produce the same bits.
* A normal deviate is read from a 65 537-entry table of standard-normal
  quantiles ``Phi^-1((i + 0.5) / 65536)`` (computed once on the host with
  ``statistics.NormalDist``) indexed by the top 16 bits, and linearly
  interpolated with the next 16 bits.  Interpolation uses one fp64 multiply
  and one fp64 add in separate correctly rounded steps, so it is bit-identical
  on every device.  The tails are cut at about +-4.3 sigma.
* bf16 tensors are rounded from fp32 with round-to-nearest-even done on the
  integer bit pattern (again device independent).

Workloads follow the five layer configurations of the method's benchmark
description: tiny, fine-grained (learned-style router projection), expert-pool
sweep (i.i.d. N(0,1) logits), skewed (N(0,1) + Zipf(1.2) popularity bias with
four experts that receive no tokens) and large (i.i.d. logits, timed in BF16
and MXFP8).
"""
from __future__ import annotations

import math
import statistics
from dataclasses import dataclass, field, replace

import torch

_GOLDEN = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB


def _s64(v: int) -> int:
    """Reinterpret an unsigned 64-bit integer as signed (torch int64)."""
    v &= (1 << 64) - 1
    return v - (1 << 64) if v >= (1 << 63) else v


def _mix_int(z: int) -> int:
    z &= (1 << 64) - 1
    z = ((z ^ (z >> 30)) * _M1) & ((1 << 64) - 1)
    z = ((z ^ (z >> 27)) * _M2) & ((1 << 64) - 1)
    return z ^ (z >> 31)


def _lsr(x: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 bit patterns."""
    return (x >> s) & ((1 << (64 - s)) - 1)


def _mix(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _lsr(z, 30)) * _s64(_M1)
    z = (z ^ _lsr(z, 27)) * _s64(_M2)
    return z ^ _lsr(z, 31)


def stream_key(seed: int, tensor_id: int) -> int:
    """64-bit key of one named random stream."""
    return _mix_int((seed * 0x100000001B3 + tensor_id * 0x1F123BB5 + 0x51) & ((1 << 64) - 1))


def random_bits(key: int, start: int, n: int, device) -> torch.Tensor:
    """64 random bits (as int64) for flat indices ``start .. start+n-1``."""
    i = torch.arange(start + 1, start + n + 1, dtype=torch.int64, device=device)
    return _mix(i * _s64(_GOLDEN) + _s64(key))


_QTABLE_CACHE: dict = {}


def _quantile_table(device) -> torch.Tensor:
    dev = torch.device(device)
    if dev not in _QTABLE_CACHE:
        nd = statistics.NormalDist()
        q = [nd.inv_cdf((i + 0.5) / 65536.0) for i in range(65536)]
        q.append(q[-1])
        _QTABLE_CACHE[dev] = torch.tensor(q, dtype=torch.float64, device=dev)
    return _QTABLE_CACHE[dev]


def normal_f64(key: int, start: int, n: int, device="cpu") -> torch.Tensor:
    """Standard-normal deviates (fp64) for flat indices start..start+n-1."""
    bits = random_bits(key, start, n, device)
    hi = _lsr(bits, 48)
    frac = (_lsr(bits, 32) & 0xFFFF).to(torch.float64) * (1.0 / 65536.0)
    tab = _quantile_table(device)
    lo_v = tab[hi]
    step = tab[hi + 1] - lo_v
    return lo_v + step * frac


def f32_to_bf16_bits(x: torch.Tensor) -> torch.Tensor:
    """fp32 -> bf16 bit pattern (int16 storage) with round-to-nearest-even."""
    b = x.contiguous().view(torch.int32).to(torch.int64) & 0xFFFFFFFF
    lsb = (b >> 16) & 1
    r = (b + 0x7FFF + lsb) >> 16
    return (r & 0xFFFF).to(torch.int32).to(torch.int16)


def normal_bf16(key: int, shape, std: float, device="cpu", start: int = 0,
                chunk: int = 1 << 26) -> torch.Tensor:
    """A bf16 tensor of N(0, std^2) deviates (flat indices start..)."""
    n = 1
    for s in shape:
        n *= int(s)
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    ov = out.view(torch.int16)
    for c0 in range(0, n, chunk):
        m = min(chunk, n - c0)
        v = (normal_f64(key, start + c0, m, device) * std).to(torch.float32)
        ov[c0:c0 + m] = f32_to_bf16_bits(v)
    return out.view(*shape)


def normal_f32(key: int, shape, std: float = 1.0, device="cpu", start: int = 0,
               chunk: int = 1 << 26) -> torch.Tensor:
    n = 1
    for s in shape:
        n *= int(s)
    out = torch.empty(n, dtype=torch.float32, device=device)
    for c0 in range(0, n, chunk):
        m = min(chunk, n - c0)
        out[c0:c0 + m] = (normal_f64(key, start + c0, m, device) * std).to(torch.float32)
    return out.view(*shape)


# ---------------------------------------------------------------------------
# Workload descriptions
# ---------------------------------------------------------------------------

TID_X, TID_WR, TID_W13, TID_W2, TID_DOUT, TID_LOGITS, TID_PERM = 1, 2, 3, 4, 5, 6, 7


@dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int
    d: int
    E: int
    k: int
    f: int
    router: str = "logits"      # "proj": logits = x . W_r ; "logits": given fp32 logits
    logits: str = "iid"         # "iid" N(0,1) | "zipf" N(0,1) + Zipf bias
    zipf_s: float = 1.2
    n_empty: int = 0            # experts forced to receive no tokens (zipf only)
    dtype: str = "bf16"         # "bf16" | "mxfp8"
    x_std: float = 1.0
    w_std: float = 0.02
    seed: int = 0
    extra: dict = field(default_factory=dict, compare=False)

    @property
    def M(self) -> int:
        return self.T * self.k

    def with_(self, **kw) -> "LayerConfig":
        return replace(self, **kw)

    def gemm_flops_fwd_bwd(self) -> int:
        """Algorithmic grouped-GEMM work: 6 T k d f forward, 12 T k d f backward."""
        return 18 * self.T * self.k * self.d * self.f


CONFIGS = {
    "tiny": LayerConfig("tiny", T=256, d=128, E=8, k=2, f=256, router="proj", seed=1000),
    "fine": LayerConfig("fine", T=4096, d=2048, E=32, k=4, f=1024, router="proj", seed=2000),
    "pool_e8": LayerConfig("pool_e8", T=16384, d=2048, E=8, k=4, f=1024, seed=3008),
    "pool_e32": LayerConfig("pool_e32", T=16384, d=2048, E=32, k=4, f=1024, seed=3032),
    "pool_e128": LayerConfig("pool_e128", T=16384, d=2048, E=128, k=4, f=1024, seed=3128),
    "skewed": LayerConfig("skewed", T=8192, d=4096, E=64, k=8, f=1536, logits="zipf",
                          n_empty=4, seed=4000),
    "large": LayerConfig("large", T=32768, d=4096, E=128, k=8, f=2048, dtype="mxfp8",
                         seed=5000),
    "large_bf16": LayerConfig("large_bf16", T=32768, d=4096, E=128, k=8, f=2048, seed=5000),
}


def zipf_bias(cfg: LayerConfig) -> torch.Tensor:
    """Per-expert fp32 logit bias: a seeded random ranking r_e of the E - n_empty
    live experts gets ``-s * ln(r_e)`` (popularity ~ r^-s); the n_empty experts
    get -1e4 so that they never reach the top-k."""
    key = stream_key(cfg.seed, TID_PERM)
    bits = random_bits(key, 0, cfg.E, "cpu")
    order = sorted(range(cfg.E), key=lambda e: (int(bits[e]), e))
    bias = [0.0] * cfg.E
    live = cfg.E - cfg.n_empty
    for rank0, e in enumerate(order):
        bias[e] = -cfg.zipf_s * math.log(rank0 + 1) if rank0 < live else -1.0e4
    return torch.tensor(bias, dtype=torch.float32)


def make_logits(cfg: LayerConfig, device="cpu", rows=None) -> torch.Tensor:
    """Given fp32 router logits [T, E] (or the listed token rows)."""
    key = stream_key(cfg.seed, TID_LOGITS)
    if rows is None:
        lg = normal_f32(key, (cfg.T, cfg.E), 1.0, device)
    else:
        lg = torch.stack([normal_f32(key, (cfg.E,), 1.0, device, start=int(t) * cfg.E)
                          for t in rows])
    if cfg.logits == "zipf":
        lg = lg + zipf_bias(cfg).to(device)
    return lg


def make_x(cfg, device="cpu", rows=None):
    key = stream_key(cfg.seed, TID_X)
    if rows is None:
        return normal_bf16(key, (cfg.T, cfg.d), cfg.x_std, device)
    return torch.stack([normal_bf16(key, (cfg.d,), cfg.x_std, device, start=int(t) * cfg.d)
                        for t in rows])


def make_dout(cfg, device="cpu", rows=None):
    key = stream_key(cfg.seed, TID_DOUT)
    if rows is None:
        return normal_bf16(key, (cfg.T, cfg.d), 1.0, device)
    return torch.stack([normal_bf16(key, (cfg.d,), 1.0, device, start=int(t) * cfg.d)
                        for t in rows])


def make_wr(cfg, device="cpu"):
    """Router projection W_r [d, E] (used when cfg.router == 'proj')."""
    return normal_bf16(stream_key(cfg.seed, TID_WR), (cfg.d, cfg.E), cfg.w_std, device)


def make_w13(cfg, device="cpu", experts=None):
    """W13 [E, 2f, d]: rows 0..f-1 of each expert are W1 (gate), f..2f-1 are W3 (up)."""
    key = stream_key(cfg.seed, TID_W13)
    per = 2 * cfg.f * cfg.d
    if experts is None:
        return normal_bf16(key, (cfg.E, 2 * cfg.f, cfg.d), cfg.w_std, device)
    return torch.stack([normal_bf16(key, (2 * cfg.f, cfg.d), cfg.w_std, device, start=int(e) * per)
                        for e in experts])


def make_w2(cfg, device="cpu", experts=None):
    """W2 [E, d, f]."""
    key = stream_key(cfg.seed, TID_W2)
    per = cfg.d * cfg.f
    if experts is None:
        return normal_bf16(key, (cfg.E, cfg.d, cfg.f), cfg.w_std, device)
    return torch.stack([normal_bf16(key, (cfg.d, cfg.f), cfg.w_std, device, start=int(e) * per)
                        for e in experts])


def make_inputs(cfg: LayerConfig, device="cpu") -> dict:
    """All inputs of one forward+backward step of the layer."""
    out = {
        "x": make_x(cfg, device),
        "w13": make_w13(cfg, device),
        "w2": make_w2(cfg, device),
        "dout": make_dout(cfg, device),
    }
    if cfg.router == "proj":
        out["wr"] = make_wr(cfg, device)
    else:
        out["logits"] = make_logits(cfg, device)
    return out
