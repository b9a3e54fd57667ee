"""The bench's roofline accounting (CPU): FLOPs and algorithmic bytes per
step, the traffic figure it takes from the committed ncu capture, and the
whole-job throughput."""
import os

import pytest

from routing_grouped_gemm_moe_b200 import inputs as I

bench = pytest.importorskip("bench")


@pytest.mark.parametrize("name", ["tiny", "fine", "pool_e128", "skewed", "large_bf16"])
def test_gemm_flops_total_is_18_T_k_d_f(name):
    """Forward 2 x (2f d + f d) and backward 2 x (f d + f d + 2f d + 2f d)
    multiply-adds per routed row: 18 T k d f FLOPs per step; recompute runs
    GEMM1 (4 T k d f) again."""
    cfg = I.CONFIGS[name]
    T, k, d, f = cfg.T, cfg.k, cfg.d, cfg.f
    assert sum(bench.gemm_flops(cfg).values()) == 18 * T * k * d * f
    assert sum(bench.gemm_flops(cfg, recompute=True).values()) == 22 * T * k * d * f


def test_large_layer_figures():
    cfg = I.CONFIGS["large_bf16"]
    assert sum(bench.gemm_flops(cfg).values()) == 39582418599936
    assert bench.gemm_algorithmic_bytes(cfg) == 46170898432


@pytest.mark.parametrize("name", ["tiny", "fine", "large_bf16"])
@pytest.mark.parametrize("mx", [False, True])
def test_gemm_algorithmic_bytes_enumerated_per_gemm(name, mx):
    """Each GEMM reads its operands once and writes its output once (bf16
    outputs; MXFP8 operands 1 + 1/32 bytes per element; the saved [G | U]
    that the SwiGLU-backward epilogue reads stays bf16)."""
    cfg = I.CONFIGS[name]
    M, d, f, E = cfg.T * cfg.k, cfg.d, cfg.f, cfg.E
    op = 1 + 1 / 32 if mx else 2
    gemms = [  # (operand elements read, bf16 elements read, elements written)
        (M * d + E * 2 * f * d, 0, M * 2 * f + M * f),    # GEMM1 + SwiGLU: x_perm, W13 -> [G|U], A
        (M * f + E * d * f, 0, M * d),                    # GEMM2: A, W2 -> Y
        (M * d + E * d * f, M * 2 * f, M * 2 * f),        # dA + SwiGLU bwd: dY, W2 (+ [G|U]) -> dH
        (M * d + M * f, 0, E * d * f),                    # dW2: dY, A
        (M * 2 * f + E * 2 * f * d, 0, M * d),            # dX: dH, W13
        (M * 2 * f + M * d, 0, E * 2 * f * d),            # dW13: dH, x_perm
    ]
    want = sum(op * r + 2 * rb + 2 * w for r, rb, w in gemms)
    assert bench.gemm_algorithmic_bytes(cfg, mx) == int(want)


def test_memory_bound_stage_bytes():
    cfg = I.CONFIGS["large_bf16"]
    T, d, E, k = cfg.T, cfg.d, cfg.E, cfg.k
    M = T * k
    b = bench.memory_bytes(cfg)
    # dispatch: x read, x_perm written, dest_pos / src_token / ranks, top-k indices
    assert b["dispatch"] == 2 * T * d + 2 * M * d + 12 * M + 4 * T * k
    # combine: Y_perm read, out written, positions + weights
    assert b["combine"] == 2 * M * d + 2 * T * d + 8 * T * k
    # unpermute-sum: dX_perm read, dx written, positions
    assert b["unpermute_sum"] == 2 * M * d + 2 * T * d + 4 * T * k
    # an MXFP8 GEMM1: the dispatch also writes x_perm's codes and scales
    assert bench.memory_bytes(cfg, mx_dispatch=True)["dispatch"] == b["dispatch"] + M * d + M * d // 32


def _source_hash():
    import hashlib
    csrc = os.path.join(os.path.dirname(os.path.abspath(bench.__file__)), "routing_grouped_gemm_moe_b200",
                        "csrc")
    h = hashlib.sha256()
    for f in bench.KERNEL_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def test_traffic_comes_from_the_capture_of_these_sources(tmp_path, monkeypatch):
    """The committed per-step DRAM traffic is reported only while the kernel
    sources still hash to the value recorded beside it."""
    import json
    d = json.load(open(bench.TRAFFIC_FILE))
    want = d["bytes_per_step"]["large_bf16/bf16"]
    assert bench.kernel_source_hash() == _source_hash()
    fresh = d["source_hash"] == _source_hash()
    assert bench.gemm_traffic("large_bf16/bf16", None, False) == (want if fresh else None)
    # not for other variants of the step
    assert bench.gemm_traffic("large_bf16/bf16", ["gemm1"], False) is None
    assert bench.gemm_traffic("large_bf16/bf16", None, True) is None
    assert bench.gemm_traffic("fine/bf16", None, False) is None
    # a capture of these very sources is reported, a stale one is not
    cur = tmp_path / "cur.json"
    cur.write_text(json.dumps(dict(d, source_hash=_source_hash())))
    assert bench.gemm_traffic("large_bf16/bf16", None, False, str(cur)) == want
    stale = tmp_path / "stale.json"
    stale.write_text(json.dumps(dict(d, source_hash="0000" + _source_hash()[4:])))
    assert bench.gemm_traffic("large_bf16/bf16", None, False, str(stale)) is None


def test_job_throughput_counts_every_rank():
    # 4 ranks x 32768 tokens x 20 steps in 800 ms
    assert bench.job_throughput(4, 32768, 20, 800.0) == pytest.approx(4 * 32768 * 20 / 0.8)


@pytest.mark.parametrize("workload", ["pool_e8", "fine"])
def test_reference_arm_line_and_other_ranks(workload):
    """`bench.py --impl reference` prints one JSON line with the oracle's
    rate on rank 0 and exits quietly on the other ranks."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.abspath(bench.__file__))
    cmd = [sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "1",
           "--warmup", "3", "--ref-rows", "64", "--workload", workload]
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.strip() == ""
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0
