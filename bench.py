#!/usr/bin/env python
"""Benchmark of the single-GPU MoE expert layer (forward + backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one forward + backward of the whole layer on one batch of synthetic
input: router top-k, rowwise dispatch, GEMM1 + SwiGLU, GEMM2, combine,
combine backward, dA GEMM + SwiGLU backward, dW2, dX, dW13, router backward,
unpermute-sum.  Default workload: the large uniform layer (T=32768,
d_model=4096, E=128, k=8, d_ff=2048, i.i.d. N(0,1) router logits) in BF16.

N > 1 (torchrun, one process per GPU): every rank runs an independent replica
on its own batch (weak scaling, no data-path collective); the time is the max
over ranks of the device-timed region.

Rank 0 prints one JSON line.  `value` is tokens/s with inputs resident in HBM
(device time, CUDA events); `e2e` is the same metric through the same API with
the step's inputs copied in from pinned host memory and out/dx copied back
inside the timed region.  `roofline` reports the grouped GEMM (the dominant
kernel) against the measured bf16 tensor-core peak.  `cpu_baseline` times the
CPU oracle on a bounded sample of the same workload.  `--impl reference` runs
only that oracle sample as the reference arm.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE layer fwd+bwd tokens/s and grouped-GEMM TFLOP/s (% of B200 peak), 1 GPU"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["source"] = "fallback"
    return d


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.fh,
                stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                    power.append(float(parts[3]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax),
                "power_w_max": max(power), "samples": len(sm), "reasons": sorted(reasons)}


# ----------------------------------------------------------------- workload helpers

def describe(cfg) -> str:
    lg = {"iid": "i.i.d. N(0,1) router logits",
          "zipf": f"N(0,1) + Zipf({cfg.zipf_s}) router bias, {cfg.n_empty} empty experts"}[cfg.logits]
    if cfg.router == "proj":
        lg = "router projection x W_r (W_r ~ N(0, 0.02^2))"
    return (f"{cfg.name}: T={cfg.T} d_model={cfg.d} E={cfg.E} top-k={cfg.k} d_ff={cfg.f} SwiGLU, "
            f"{lg}, {'MXFP8' if cfg.dtype == 'mxfp8' else 'BF16'} grouped GEMMs")


KERNEL_SOURCES = ["grouped_gemm.cu", "ptx.cuh", "mx_encode.cuh", "common.cuh"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "gemm_traffic.json")


def kernel_source_hash() -> str:
    """First 16 hex digits of sha256 over the grouped-GEMM kernel sources."""
    import hashlib
    csrc = os.path.join(ROOT, "routing_grouped_gemm_moe_b200", "csrc")
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def gemm_traffic(workload, mx_sel, recompute, path=TRAFFIC_FILE):
    """DRAM bytes per step of the six GEMM launches, from the committed
    capture totals (JSON), while the kernel sources still hash to the value
    they were captured with; None otherwise."""
    if mx_sel or recompute:
        return None
    try:
        with open(path) as fh:
            d = json.load(fh)
    except (OSError, ValueError):
        return None
    if d.get("source_hash") != kernel_source_hash():
        return None
    v = d.get("bytes_per_step", {}).get(workload)
    return int(v) if v is not None else None


def gemm_algorithmic_bytes(cfg, mx=False) -> int:
    """DRAM bytes the six GEMMs must move per step: each operand read once,
    each output written once (MXFP8 operands: 1 byte + 1/32 scale byte)."""
    M, d, f, E = cfg.T * cfg.k, cfg.d, cfg.f, cfg.E
    op = (1 + 1 / 32) if mx else 2
    x, gu, a, y = M * d, M * 2 * f, M * f, M * d
    w13, w2 = E * 2 * f * d, E * d * f
    reads = op * ((x + w13) + (a + w2) + (y + w2) + (y + a) + (gu + w13) + (gu + x)) + 2 * gu  # + saved [G|U]
    writes = 2 * ((gu + a) + y + gu + w2 + x + w13)
    return int(reads + writes)


def l2_note(cfg) -> str:
    """How the timed steps stay honest about the 126 MB L2 (no flush is done)."""
    x = cfg.T * cfg.d * 2
    w = cfg.E * 3 * cfg.f * cfg.d * 2
    act = cfg.T * cfg.k * (2 * cfg.d + 3 * cfg.f) * 2
    big = "larger" if min(w, act) > 126e6 else "not all larger"
    return (f"no flush; operands {big} than the 126 MB L2: x {x / 2**20:.0f} MiB, "
            f"W13+W2 {w / 2**20:.0f} MiB, routed activations {act / 2**20:.0f} MiB per step")


def gemm_flops(cfg, recompute=False) -> dict:
    M = cfg.T * cfg.k
    d, f = cfg.d, cfg.f
    fl = {"gemm1_swiglu": 2 * M * d * 2 * f, "gemm2": 2 * M * f * d,
          "dA_swiglu_bwd": 2 * M * d * f, "dW2": 2 * M * d * f,
          "dX": 2 * M * 2 * f * d, "dW13": 2 * M * 2 * f * d}
    if recompute:
        fl["recompute"] = fl["gemm1_swiglu"]
    return fl


# stage name -> the name ops.MoELayer(mx_gemms=...) uses for that GEMM
MX_NAME = {"gemm1_swiglu": "gemm1", "recompute": "gemm1", "gemm2": "gemm2",
           "dA_swiglu_bwd": "dA", "dW2": "dW2", "dX": "dX", "dW13": "dW13"}


def memory_bytes(cfg, mx_dispatch=False) -> dict:
    """Algorithmic HBM bytes of the memory-bound stages (what must move).
    mx_dispatch: the dispatch also writes x_perm's row-wise MXFP8 codes and
    scales (an MXFP8 GEMM1)."""
    T, d, E, k = cfg.T, cfg.d, cfg.E, cfg.k
    M = T * k
    return {
        "router": 4 * T * E + 8 * T * k,
        "dispatch": 2 * T * d + 2 * M * d + 12 * M + 4 * T * k + ((M * d + M * d // 32) if mx_dispatch else 0),
        "combine": 2 * M * d + 2 * T * d + 8 * T * k,
        "combine_bwd": 2 * T * d + 4 * M * d + 8 * T * k + 4 * T * k,
        "unpermute_sum": 2 * M * d + 2 * T * d + 4 * T * k,
        "router_bwd": 4 * T * E + 12 * T * k,
    }


FWD_STAGES = ["router", "dispatch", "gemm1_swiglu", "gemm2", "combine"]
BWD_STAGES = ["recompute", "combine_bwd", "dA_swiglu_bwd", "dW2", "dX", "dW13", "router_bwd",
              "unpermute_sum"]


# ----------------------------------------------------------------- CPU oracle sample

def oracle_sample_setup(cfg):
    """Routing of the whole batch by the oracle (untimed set-up for the sample):
    the given logits, or x W_r (fp64, rounded to fp32) for router-projection
    workloads."""
    import numpy as np

    from oracle import moe as om
    from routing_grouped_gemm_moe_b200 import inputs as I
    wr = None
    if cfg.router == "logits":
        lg = I.make_logits(cfg).numpy()
    else:
        wr = I.make_wr(cfg).float().double().numpy()
        lg = om.router_logits(I.make_x(cfg).float().double().numpy(), wr).astype(np.float32)
    idx, w = om.router_topk(lg, cfg.k)
    counts, offsets, dest, src = om.dispatch_plan(idx, cfg.E)
    return dict(lg=lg, wr=wr, idx=idx, w=w, counts=counts, offsets=offsets, dest=dest, src=src)


def oracle_sample_step(cfg, setup, expert: int, rows: int):
    """One bounded sample: oracle router (projection when the workload has one)
    + top-k + dispatch plan for rows/k tokens, then the expert FFN forward +
    backward (oracle.expert_forward / expert_backward) of `rows` routed rows
    of one expert.  Returns (seconds, tokens equivalent)."""
    import numpy as np

    from oracle import moe as om
    from routing_grouped_gemm_moe_b200 import inputs as I
    off = setup["offsets"]
    r0 = int(off[expert])
    m = min(rows, int(off[expert + 1]) - r0)
    toks = setup["src"][r0:r0 + m]
    f64 = lambda t: t.float().double().numpy()  # noqa: E731
    x = f64(I.make_x(cfg, rows=toks))
    dout = f64(I.make_dout(cfg, rows=toks))
    w13 = f64(I.make_w13(cfg, experts=[expert]))
    w2 = f64(I.make_w2(cfg, experts=[expert]))
    # routing weight of each sampled row
    slot = np.argmax(setup["idx"][toks] == expert, axis=1)
    wrow = setup["w"][toks, slot]
    ntok = max(1, m // cfg.k)
    t0 = time.perf_counter()
    if setup["wr"] is not None:
        lg_part = om.router_logits(x[:ntok], setup["wr"]).astype(np.float32)
    else:
        lg_part = setup["lg"][:ntok]
    idx_p, _ = om.router_topk(lg_part, cfg.k)
    om.dispatch_plan(idx_p, cfg.E)
    sub_off = [0, m]
    GU, A, Y = om.expert_forward(x, w13, w2, sub_off)
    dY = om.round_bf16(wrow[:, None] * dout)
    om.expert_backward(dY, GU, A, x, w13, w2, sub_off)
    dt = time.perf_counter() - t0
    return dt, m / cfg.k


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_baseline(cfg, min_seconds=10.0):
    """The oracle on whole experts of the workload until about `min_seconds`
    of CPU work have been timed (at most all E experts)."""
    setup = oracle_sample_setup(cfg)
    total_t, total_tok, rows, n = 0.0, 0.0, 0, 0
    for e in range(cfg.E):
        m = int(setup["offsets"][e + 1] - setup["offsets"][e])
        dt, tok = oracle_sample_step(cfg, setup, e, m)
        total_t += dt
        total_tok += tok
        rows += m
        n += 1
        if total_t >= min_seconds:
            break
    return {"value": total_tok / total_t, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": (f"numpy fp64 oracle on {n} of the {cfg.E} experts of the same workload: "
                       f"the SwiGLU expert forward+backward of all {rows} rows routed to them, "
                       f"plus router {'projection + ' if cfg.router == 'proj' else ''}top-k + "
                       f"dispatch plan of rows/k tokens; value = "
                       f"tokens-equivalent (rows / k) per second"),
            "seconds": total_t}


# ----------------------------------------------------------------- reference arm

def run_reference(args, rank, world):
    from routing_grouped_gemm_moe_b200 import inputs as I
    if rank != 0:
        return
    cfg = I.CONFIGS[args.workload]
    setup = oracle_sample_setup(cfg)
    rows = args.ref_rows
    for i in range(args.warmup):
        oracle_sample_step(cfg, setup, i % cfg.E, rows)
    total_t, total_tok = 0.0, 0.0
    for i in range(args.steps):
        dt, tok = oracle_sample_step(cfg, setup, (args.warmup + i) % cfg.E, rows)
        total_t += dt
        total_tok += tok
    value = total_tok / total_t
    router = "router projection + top-k" if cfg.router == "proj" else "router top-k"
    sample = (f"each step: numpy fp64 oracle {router} + dispatch plan of {rows // cfg.k} tokens "
              f"and the SwiGLU expert forward+backward of {rows} routed rows of one expert")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * total_t / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": describe(cfg)},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- GPU arm

# ----------------------------------------------------------------- replicas (N > 1)

def replica_inputs(cfg, rank: int, world: int, device):
    """Inputs of one data-parallel replica: each rank draws its own batch (its
    own seed: weak scaling), the weights are the same on every rank."""
    from routing_grouped_gemm_moe_b200 import inputs as I
    cfg_r = cfg.with_(seed=cfg.seed + 7919 * rank) if world > 1 else cfg
    inp = I.make_inputs(cfg_r, device=device)
    if world > 1:
        for n in ("w13", "w2", "wr"):
            if n in inp:
                inp[n] = getattr(I, "make_" + n)(cfg, device=device)
    return inp


def max_over_ranks(ms: float, device) -> float:
    """This rank's device-timed milliseconds -> the maximum over all ranks (one
    host-side all-reduce after the timed region; nothing in the data path)."""
    import torch
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, tokens_per_rank: int, steps: int, ms: float) -> float:
    """Whole-job tokens/s: the tokens all ranks processed over the slowest rank's time."""
    return world * tokens_per_rank * steps / (ms / 1000.0)


def time_steps(layer, inp, steps: int, warmup: int, world: int, clocks=None):
    """`warmup` untimed forward + backward steps, then `steps` timed ones
    (CUDA events on the current stream, barrier + synchronize on both sides,
    per-stage events).  Returns (ms over the timed steps, stage ms per step,
    kernel launches, clock record)."""
    import torch
    import torch.distributed as dist

    from routing_grouped_gemm_moe_b200 import ops
    lg, wr = inp.get("logits"), inp.get("wr")

    def step(ef=None, eb=None):
        layer.forward(inp["x"], inp["w13"], inp["w2"], logits=lg, w_r=wr, events=ef)
        layer.backward(inp["dout"], inp["x"], inp["w13"], inp["w2"], logits=lg, w_r=wr, events=eb)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if layer.device_status() != 0:
        raise SystemExit("device status word set during warm-up")
    ev_f = [ops.make_events(len(FWD_STAGES) + 1) for _ in range(steps)]
    ev_b = [ops.make_events(len(BWD_STAGES) + 1) for _ in range(steps)]
    t_start, t_end = ops.make_events(2)
    if clocks:
        clocks.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = ops.kernel_launches()
    t_start.record()
    for i in range(steps):
        step(ev_f[i], ev_b[i])
    t_end.record()
    torch.cuda.synchronize()
    launches = ops.kernel_launches() - launches0
    if world > 1:
        dist.barrier()
    clk = clocks.stop() if clocks else None
    ms = t_start.elapsed_time(t_end)
    stage_ms = {}
    for names, evs in ((FWD_STAGES, ev_f), (BWD_STAGES, ev_b)):
        for j, n in enumerate(names):
            stage_ms[n] = sum(e[j].elapsed_time(e[j + 1]) for e in evs) / steps
    if layer.device_status() != 0:
        raise SystemExit("device status word set during the timed region")
    return ms, stage_ms, launches, clk


def gemm_record(cfg, stage_ms, peaks, mx_sel=None, recompute=False):
    """GEMM TFLOP/s of a timed step against the peak of its dtype mix."""
    mx = cfg.dtype == "mxfp8"
    fl = gemm_flops(cfg, recompute)
    gemm_ms = sum(stage_ms[n] for n in fl)
    achieved = sum(fl.values()) / (gemm_ms / 1000.0) / 1e12
    mx_stage = {n: mx and (mx_sel is None or MX_NAME[n] in mx_sel) for n in fl}
    # an MXFP8 contraction takes the fp8 peak: the measured bf16 peak x the
    # nominal fp8 / bf16 ratio (4.5 / 2.25 PFLOP/s dense); with selective
    # MXFP8 the peak is the one of the mix: the flops over the time each GEMM
    # would take at its own dtype's peak
    pk = peaks["bf16_tflops_sustained"]
    t_ideal = sum(fl[n] / (pk * (2.0 if mx_stage[n] else 1.0)) for n in fl)
    t_nominal = sum(fl[n] / (4500.0 if mx_stage[n] else 2250.0) for n in fl)
    peak = sum(fl.values()) / t_ideal
    nominal = sum(fl.values()) / t_nominal
    per = {n: {"ms": stage_ms[n], "tflops": fl[n] / (stage_ms[n] / 1000.0) / 1e12} for n in fl}
    return dict(achieved=achieved, peak=peak, nominal=nominal, per_gemm=per, mx_stage=mx_stage,
                flops=sum(fl.values()))


def sub_record(ops, I, cfg, dev, peaks, steps=8, warmup=3, **layer_opts):
    """One more workload timed in the same run (not the headline): tokens/s
    and GEMM TFLOP/s of its forward + backward."""
    import torch
    inp = I.make_inputs(cfg, device=dev)
    layer = ops.MoELayer(cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, router=cfg.router, dtype=cfg.dtype,
                         device=dev, **layer_opts)
    ms, stage_ms, _, _ = time_steps(layer, inp, steps, warmup, 1)
    g = gemm_record(cfg, stage_ms, peaks)
    rec = {"workload": describe(cfg), "tokens_per_s": cfg.T * steps / (ms / 1000.0),
           "ms_per_step": ms / steps, "gemm_tflops": g["achieved"], "gemm_peak_tflops": g["peak"],
           "gemm_frac": g["achieved"] / g["peak"], "steps": steps, "warmup": warmup}
    del layer, inp
    torch.cuda.empty_cache()
    return rec


def router_isolated(ops, cfg, dev, nbuf=16, n=64):
    """The router kernels alone, back to back, each launch on one of `nbuf`
    logits buffers taken in turn (together larger than L2, so every launch
    reads from DRAM), next to a device-to-device copy of the same bytes: the
    stage events of the step add their own gaps around kernels this short."""
    import torch
    T, E, k = cfg.T, cfg.E, cfg.k
    g = torch.Generator(device=dev).manual_seed(0)
    lgs = [torch.randn(T, E, device=dev, generator=g) for _ in range(nbuf)]
    dws = [torch.randn(T, k, device=dev, generator=g) for _ in range(nbuf)]
    sel = [ops.router_topk(lg, k) for lg in lgs]

    def per_launch_us(fn):
        for i in range(8):
            fn(i)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda._sleep(2_000_000)  # the host queues the launches ahead of the GPU
        e0.record()
        for i in range(n):
            fn(i)
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n * 1000.0

    topk = per_launch_us(lambda i: ops.router_topk(lgs[i % nbuf], k))
    bwd = per_launch_us(lambda i: ops.router_bwd(sel[i % nbuf][0], sel[i % nbuf][1], dws[i % nbuf], E))
    copy = per_launch_us(lambda i: lgs[(i + 1) % nbuf].copy_(lgs[i % nbuf]))
    b_topk, b_bwd = 4 * T * E + 8 * T * k, 4 * T * E + 12 * T * k
    return {"topk": {"us": topk, "gbs": b_topk / topk / 1e3},
            "bwd": {"us": bwd, "gbs": b_bwd / bwd / 1e3},
            "copy_same_bytes_us": copy,
            "how": f"{n} launches back to back over {nbuf} rotating [T, E] fp32 buffers "
                   f"({nbuf * 4 * T * E / 2**20:.0f} MiB), CUDA events around the launches; the copy "
                   "moves one [T, E] fp32 buffer (read + write)"}


def library_reference(ops, dev, S=8192, seconds=1.5):
    """Library GEMMs on this GPU next to ours, one dense S x S x S product each,
    timed in loops of about `seconds` (long enough for the power cap to set
    the clock): cuBLAS bf16 (torch.matmul), cuBLAS MXFP8 (torch._scaled_mm
    with 1x32 E8M0 block scales), and the repository's grouped GEMM given one
    group of S rows, bf16 and MXFP8 (its call includes building the scale
    atoms from the canonical scales).  Measuring sticks only: none of these
    library calls is on the layer's path."""
    import ctypes as C

    import torch
    from routing_grouped_gemm_moe_b200 import _lib as L
    bf = torch.bfloat16
    g = torch.Generator(device=dev).manual_seed(0)
    a = torch.randn(S, S, device=dev, generator=g).to(bf)
    b = torch.randn(S, S, device=dev, generator=g).to(bf)
    c = torch.empty(S, S, device=dev, dtype=bf)
    offs = torch.tensor([0, S], dtype=torch.int32, device=dev)
    flops = 2.0 * S ** 3

    def sustained(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(5):
            fn()
        e1.record()
        torch.cuda.synchronize()
        reps = max(5, int(seconds * 1000.0 / (e0.elapsed_time(e1) / 5)))
        clk = ClockSampler(dev.index or 0)
        clk.start()
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        ck = clk.stop()
        ms = e0.elapsed_time(e1) / reps
        return {"tflops": flops / ms / 1e9, "ms": ms, "launches": reps, "sm_mhz": ck.get("sm_mhz"),
                "reasons": ck.get("reasons")}

    rec = {"shape": f"{S} x {S} x {S}, bf16 out",
           "how": f"each a loop of about {seconds} s after 3 warm-up calls, CUDA events, "
                  "nvidia-smi clocks during the loop"}
    rec["cublas_bf16"] = sustained(lambda: torch.matmul(a, b.t(), out=c))
    rec["ours_bf16"] = sustained(lambda: ops.grouped_gemm(L.GG_RAGGED_M, a, b.view(1, S, S), offs, 1,
                                                          N=S, K=S, c=c))
    ac, asc = ops.mxfp8_quantize(a, 1)
    bc, bsc = ops.mxfp8_quantize(b, 1)
    args = L.GGArgs(mode=L.GG_RAGGED_M, dtype=L.DTYPE_MXFP8, epilogue=L.EPI_NONE, E=1, M_total=S,
                    M=0, N=S, K=S, offsets=ops._p(offs), a=ops._p(ac), b=ops._p(bc), b_mn_major=0,
                    c=ops._p(c), aux=None, gu=None, a_scales=ops._p(asc), b_scales=ops._p(bsc),
                    status=None)
    nb = int(L.lib().moe_grouped_gemm_workspace_bytes(C.byref(args)))
    ws = torch.empty(max(nb, 1), dtype=torch.uint8, device=dev)
    args.workspace, args.workspace_bytes = ops._p(ws), nb
    rec["ours_mxfp8"] = sustained(lambda: L.call("moe_grouped_gemm", C.byref(args), ops._s()))
    try:
        # cuBLAS wants the scales in its own tiled order; their values do not
        # change the time, so every scale is 2^0 here
        ones = torch.full((S * S // 32,), 127, dtype=torch.uint8, device=dev).view(torch.float8_e8m0fnu)
        a8, b8 = ac.view(torch.float8_e4m3fn), bc.view(torch.float8_e4m3fn)
        rec["cublas_mxfp8"] = sustained(lambda: torch._scaled_mm(a8, b8.t(), ones, ones, out_dtype=bf))
    except Exception as e:  # noqa: BLE001 -- a torch build without MX scaled_mm
        rec["cublas_mxfp8"] = {"unavailable": repr(e)[:200]}
    rec["ours_over_cublas_bf16"] = rec["ours_bf16"]["tflops"] / rec["cublas_bf16"]["tflops"]
    if "tflops" in rec["cublas_mxfp8"]:
        rec["ours_over_cublas_mxfp8"] = rec["ours_mxfp8"]["tflops"] / rec["cublas_mxfp8"]["tflops"]
    del a, b, c, ac, bc, ws
    torch.cuda.empty_cache()
    return rec


def model_like_memory(ops, I, cfg, dev, n_layers=4, steps=3, warmup=2):
    """n_layers MoE layers of one shape used as a model uses them: every
    layer's forward, then every layer's backward in reverse order, so that
    each layer's saved state is held until its backward.  The layers share
    the weights and one workspace.  Stored-activation mode against recompute
    mode ([G | U] and A not kept: the backward runs GEMM1 + SwiGLU again into
    the shared workspace): peak device memory and per-layer tokens/s."""
    import torch
    inp = I.make_inputs(cfg, device=dev)
    lg = inp.get("logits")
    out = {}
    for mode in (False, True):
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        base = torch.cuda.memory_allocated(dev)
        torch.cuda.reset_peak_memory_stats(dev)
        nb = ops.layer_workspace_bytes(cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, router=cfg.router,
                                       recompute=mode)
        ws = torch.zeros(nb, dtype=torch.uint8, device=dev)
        layers = [ops.MoELayer(cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, router=cfg.router, device=dev,
                               recompute=mode, workspace=ws) for _ in range(n_layers)]

        def step():
            for ly in layers:
                ly.forward(inp["x"], inp["w13"], inp["w2"], logits=lg)
            for ly in reversed(layers):
                ly.backward(inp["dout"], inp["x"], inp["w13"], inp["w2"], logits=lg)

        for _ in range(warmup):
            step()
        t0, t1 = ops.make_events(2)
        torch.cuda.synchronize()
        t0.record()
        for _ in range(steps):
            step()
        t1.record()
        torch.cuda.synchronize()
        if layers[0].device_status() != 0:
            raise SystemExit("device status word set in the model-like run")
        ms = t0.elapsed_time(t1)
        out["recompute" if mode else "stored"] = {
            "peak_memory_gib": (torch.cuda.max_memory_allocated(dev) - base) / 2 ** 30,
            "saved_state_gib_per_layer": layers[0].saved_bytes() / 2 ** 30,
            "workspace_gib": nb / 2 ** 30,
            "layer_tokens_per_s": cfg.T * n_layers * steps / (ms / 1000.0)}
        del layers, ws
    torch.cuda.empty_cache()
    st, rc = out["stored"], out["recompute"]
    return {"workload": describe(cfg), "layers": n_layers,
            "use": ("every layer's forward, then every backward in reverse order; weights and one "
                    "workspace shared by the layers; per-layer gradients, outputs and saved state "
                    "are each layer's own; peak = max allocated above the inputs"),
            "stored": st, "recompute": rc,
            "peak_memory_saved_gib": st["peak_memory_gib"] - rc["peak_memory_gib"],
            "throughput_ratio": rc["layer_tokens_per_s"] / st["layer_tokens_per_s"]}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="large_bf16")
    ap.add_argument("--dtype", choices=["bf16", "mxfp8"], default=None,
                    help="override the workload's grouped-GEMM precision")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the sub-records (MXFP8, the other workloads, recompute memory)")
    ap.add_argument("--ref-rows", type=int, default=512)
    ap.add_argument("--recompute", action="store_true",
                    help="keep [G | U] and A only transiently; the backward runs GEMM1 again")
    ap.add_argument("--mx-requantize-weights", action="store_true",
                    help="with MXFP8: quantise the weights again in the backward instead of "
                         "keeping the forward's second layout")
    ap.add_argument("--slice", type=int, default=1,
                    help="run 1/N of the workload: T / N tokens over E / N experts (the same rows "
                         "per expert), for profiler captures that must stay small")
    ap.add_argument("--mx-gemms", default=None,
                    help="with MXFP8: comma-separated subset of gemm1,gemm2,dA,dW2,dX,dW13")
    ap.add_argument("--library-only", action="store_true",
                    help="only the library_reference record: cuBLAS bf16 / MXFP8 and the "
                         "repository's grouped GEMM on one dense product (rank 0, 1 GPU)")
    ap.add_argument("--library-seconds", type=float, default=1.5,
                    help="length of each library_reference timing loop")
    args = ap.parse_args()
    assert args.warmup >= 3, "at least 3 warm-up steps"

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist

    from routing_grouped_gemm_moe_b200 import inputs as I
    from routing_grouped_gemm_moe_b200 import ops

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.library_only:
        if rank == 0:
            print(json.dumps({"library_reference": library_reference(ops, dev, seconds=args.library_seconds)}))
        return
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    cfg = I.CONFIGS[args.workload]
    if args.dtype:
        cfg = cfg.with_(dtype=args.dtype)
    if args.slice > 1:
        if cfg.T % args.slice or cfg.E % args.slice or cfg.n_empty:
            raise SystemExit(f"--slice {args.slice} does not divide {cfg.name}")
        cfg = cfg.with_(name=f"{cfg.name}_slice{args.slice}", T=cfg.T // args.slice, E=cfg.E // args.slice)
    mx = cfg.dtype == "mxfp8"
    inp = replica_inputs(cfg, rank, world, dev)
    mx_sel = args.mx_gemms.split(",") if (mx and args.mx_gemms) else None
    layer = ops.MoELayer(cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, router=cfg.router, dtype=cfg.dtype,
                         device=dev, recompute=args.recompute, mx_gemms=mx_sel,
                         mx_keep_weights=mx and not args.mx_requantize_weights)
    wr = inp.get("wr")

    K = args.steps
    ms, stage_ms, launches, clk = time_steps(layer, inp, K, args.warmup, world,
                                             ClockSampler(local))
    ms = max_over_ranks(ms, dev)
    ms_step = ms / K
    value = job_throughput(world, cfg.T, K, ms)

    peaks = load_peaks()
    g = gemm_record(cfg, stage_ms, peaks, mx_sel, args.recompute)
    gemm_tflops, peak_t = g["achieved"], g["peak"]
    mem = memory_bytes(cfg, mx_dispatch=g["mx_stage"]["gemm1_swiglu"])
    mem_gbs = {n: {"ms": stage_ms[n], "gbs": mem[n] / (stage_ms[n] / 1000.0) / 1e9}
               for n in mem if n in stage_ms}
    roofline = {"kernel": ("MXFP8 grouped GEMM incl. operand quantisation" if mx else
                           "grouped GEMM") + f" ({len(g['per_gemm'])} launches per step, tcgen05)",
                "bound": "tensor", "achieved": gemm_tflops, "peak": peak_t, "unit": "TFLOP/s",
                "frac": gemm_tflops / peak_t,
                "peak_source": (f"{peaks['source']} sustained bf16 (torch.matmul 8192^3 under power "
                                "cap)" + (" x 2 (nominal fp8/bf16 dense ratio)" if mx else "")),
                "nominal_peak": g["nominal"], "frac_of_nominal": gemm_tflops / g["nominal"],
                "traffic": gemm_traffic(f"{cfg.name}/{cfg.dtype}", mx_sel, args.recompute),
                "traffic_scope": "DRAM bytes per step, sum over the six GEMM launches, from the "
                                 "committed ncu capture totals (null for other workloads or once "
                                 "the kernel sources changed since the capture)",
                "algorithmic_flops_per_step": g["flops"],
                "algorithmic_bytes_per_step": gemm_algorithmic_bytes(cfg, mx)}
    peak_mem = round(torch.cuda.max_memory_allocated(dev) / 2 ** 30, 2)

    # ---------------------------------------------------------- end to end
    e2e = None
    if not args.no_e2e:
        pipe = ops.HostStreamedSteps(layer)
        host_in = [{n: inp[n].cpu().pin_memory() for n in pipe.names}]
        host_out = [{"out": torch.empty(layer.out.shape, dtype=layer.out.dtype).pin_memory(),
                     "dx": torch.empty(layer.dx.shape, dtype=layer.dx.dtype).pin_memory()}]
        h2d, d2h = pipe.bytes_per_step(host_in[0])
        pipe.run(inp["w13"], inp["w2"], host_in, host_out, 2, w_r=wr)  # warm-up
        s0, s1 = ops.make_events(2)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        s0.record()
        pipe.run(inp["w13"], inp["w2"], host_in, host_out, K, w_r=wr)
        s1.record()
        torch.cuda.synchronize()
        ems = s0.elapsed_time(s1)
        ems = max_over_ranks(ems, dev)
        e2e = {"value": job_throughput(world, cfg.T, K, ems), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "api": "routing_grouped_gemm_moe_b200.ops.HostStreamedSteps over MoELayer.forward/"
                      "backward (C ABI moe_layer_fwd / moe_layer_bwd)",
               "copies": "every step: H2D of x, dOut (and logits) from pinned host memory, D2H of "
                         "out and dx into pinned host memory, on two copy streams overlapped with "
                         "the neighbouring steps' compute; all inside the timed region"}
        del pipe, host_in, host_out

    # ---------------------------------------------------------- sub-records
    # (rank 0 at N = 1 only, after the headline; not part of `value`)
    extra = {}
    if rank == 0 and world == 1 and not args.no_extra and cfg.name == "large_bf16" \
            and not (mx or args.recompute):
        del layer, inp
        torch.cuda.empty_cache()
        mxr = sub_record(ops, I, I.CONFIGS["large"], dev, peaks, mx_keep_weights=True)
        mxr["ratio_vs_bf16"] = mxr["tokens_per_s"] / value
        mxr["gemm_peak_source"] = "2 x measured sustained bf16 (nominal fp8/bf16 dense ratio)"
        extra["mxfp8"] = mxr
        cfgs = {}
        for name in ("fine", "pool_e8", "pool_e32", "pool_e128", "skewed"):
            cfgs[name] = sub_record(ops, I, I.CONFIGS[name], dev, peaks, steps=10)
        cfgs["pool_e128_over_e8"] = cfgs["pool_e128"]["tokens_per_s"] / cfgs["pool_e8"]["tokens_per_s"]
        extra["configs"] = cfgs
        extra["recompute"] = model_like_memory(ops, I, I.CONFIGS["large_bf16"], dev)
        extra["router_isolated"] = router_isolated(ops, I.CONFIGS["large_bf16"], dev)
        extra["library_reference"] = library_reference(ops, dev, seconds=args.library_seconds)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(cfg)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "mxfp8" if mx else "bf16",
        "data": "synthetic (seeded counter-based generator; random-init weights)",
        "config": {"workload": describe(cfg), "global_batch_tokens": world * cfg.T,
                   "parallelism": f"{world} independent replica(s), no collective",
                   "activation_recompute": bool(args.recompute),
                   "mxfp8_weights_quantised_once_per_step": bool(mx and not args.mx_requantize_weights),
                   "mxfp8_gemms": (mx_sel or list(ops.MX_GEMM_NAMES)) if mx else [],
                   "l2": l2_note(cfg)},
        "gemm_tflops": gemm_tflops,
        "gemm_frac_of_measured_sustained": gemm_tflops / peak_t,
        "stages_ms": stage_ms, "gemm": g["per_gemm"], "memory_bound_gbs": mem_gbs,
        "roofline": roofline, "gpu_launches": launches, "clocks": clk,
        # device memory of the headline run (torch's allocator: inputs,
        # weights, saved activations, gradients, workspace)
        "peak_memory_gib": peak_mem,
    }
    if e2e:
        line["e2e"] = e2e
    line.update(extra)
    if cpu:
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
