"""Multi-process (world size 2, gloo on CPU) checks of the data-parallel
replica path bench.py runs under torchrun: each rank draws its own batch with
the same weights, the timed region is reduced to the slowest rank, and the
job throughput counts every rank's tokens.  No GPU involved."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port):
    sys.path.insert(0, ROOT)
    import bench
    from routing_grouped_gemm_moe_b200 import inputs as I
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        cfg = I.CONFIGS["tiny"]
        inp = bench.replica_inputs(cfg, rank, world, "cpu")
        # the batch differs between ranks, the weights do not
        xs = [torch.empty_like(inp["x"].float()) for _ in range(world)]
        dist.all_gather(xs, inp["x"].float())
        assert not torch.equal(xs[0], xs[1])
        for n in ("w13", "w2", "wr"):
            ws = [torch.empty_like(inp[n].float()) for _ in range(world)]
            dist.all_gather(ws, inp[n].float())
            assert torch.equal(ws[0], ws[1]), n
        # rank 0's batch is the single-replica batch
        if rank == 0:
            single = bench.replica_inputs(cfg, 0, 1, "cpu")
            assert torch.equal(single["x"].view(torch.int16), inp["x"].view(torch.int16))
        # the slowest rank sets the job time; every rank gets the same value
        ms = [3.0, 5.5][rank]
        m = bench.max_over_ranks(ms, "cpu")
        assert m == 5.5
        v = bench.job_throughput(world, cfg.T, 4, m)
        assert abs(v - world * cfg.T * 4 / 5.5e-3) < 1e-6 * v
        vs = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(vs, torch.tensor([v], dtype=torch.float64))
        assert vs[0].item() == vs[1].item()
    finally:
        dist.destroy_process_group()


def test_replicas_two_ranks_gloo():
    mp.spawn(_rank_main, args=(2, _free_port()), nprocs=2, join=True)


def test_single_replica_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert not dist.is_initialized()
    assert bench.max_over_ranks(7.25, "cpu") == 7.25
