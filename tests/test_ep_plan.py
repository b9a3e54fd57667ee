"""Row placement of expert parallelism over W ranks (routing_grouped_gemm_moe_b200.ep),
as world-size-2 and -4 gloo process groups on the CPU (no GPU involved).

Each rank routes its own seeded batch with the oracle, plans its own
single-GPU dispatch, exchanges the per-expert counts with one all-gather,
computes the placement, and sends every routed row to the owner of its
expert (an all-to-all of rows stands in for the peer stores over NVLink).
Each rank's receive buffer must equal the single-GPU dispatch of all ranks'
batches concatenated in rank order, restricted to that rank's experts:
counts, offsets and every row bit for bit."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
T, d, E, k = 96, 16, 8, 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _batch(rank):
    from routing_grouped_gemm_moe_b200 import inputs as I
    lg = I.normal_f32(I.stream_key(500 + rank, 1), (T, E))
    lg[:, E - 1] -= 3.0 * (rank + 1)      # uneven loads, different per rank
    x = I.normal_bf16(I.stream_key(500 + rank, 2), (T, d), 1.0)
    return lg, x


def _rank_main(rank, world, port):
    sys.path.insert(0, ROOT)
    from oracle import moe as om
    from routing_grouped_gemm_moe_b200 import ep
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        lg, x = _batch(rank)
        idx, _ = om.router_topk(lg.numpy(), k)
        counts, offsets, dest, src = om.dispatch_plan(idx, E)
        counts_all = ep.exchange_counts(torch.from_numpy(counts.astype(np.int32)))
        assert counts_all.shape == (world, E) and torch.equal(counts_all[rank], torch.from_numpy(counts))
        pl = ep.plan(counts_all, rank)
        own, pos = ep.destinations(torch.from_numpy(dest), torch.from_numpy(idx),
                                   torch.from_numpy(offsets), pl["send_base"], E, world)
        # send rows: per destination rank, (position, row) pairs
        xv = x.view(torch.int16)
        send_pos, send_rows = [], []
        for r in range(world):
            sel = (own == r).reshape(-1)
            t_of = torch.arange(T).repeat_interleave(k)[sel]
            send_pos.append(pos.reshape(-1)[sel])
            send_rows.append(xv[t_of])
        n_send = torch.tensor([p.numel() for p in send_pos])
        n_recv = torch.empty_like(n_send)
        dist.all_to_all_single(n_recv, n_send)
        ins, outs = n_send.tolist(), n_recv.tolist()
        recv_pos = torch.empty(sum(outs), dtype=torch.int64)
        recv_rows = torch.empty(sum(outs), d // 2, dtype=torch.int32)  # bf16 pairs
        dist.all_to_all_single(recv_pos, torch.cat(send_pos), outs, ins)
        dist.all_to_all_single(recv_rows, torch.cat(send_rows).view(torch.int32), outs, ins)
        recv_rows = recv_rows.view(torch.int16)
        total = int(pl["recv_offsets"][-1])
        buf = torch.full((total, d), -1, dtype=torch.int16)
        seen = torch.zeros(total, dtype=torch.int64)
        buf[recv_pos] = recv_rows
        seen.index_add_(0, recv_pos, torch.ones_like(recv_pos))
        assert torch.all(seen == 1), "every receive row is written exactly once"
        # the single-GPU dispatch of the concatenated batch, restricted to this rank's experts
        lgs, xs = zip(*[_batch(r) for r in range(world)])
        idx_all, _ = om.router_topk(torch.cat(lgs).numpy(), k)
        c_all, off_all, _, src_all = om.dispatch_plan(idx_all, E)
        El = E // world
        e0, e1 = rank * El, (rank + 1) * El
        want_rows = torch.cat(xs).view(torch.int16)[torch.from_numpy(src_all[off_all[e0]:off_all[e1]].astype(np.int64))]
        assert torch.equal(buf, want_rows)
        want_off = off_all[e0:e1 + 1] - off_all[e0]
        assert np.array_equal(pl["recv_offsets"].numpy(), want_off)
        assert np.array_equal(counts_all.sum(0).numpy(), c_all)
        # where each source's rows of each local expert start
        for s in range(world):
            for j in range(El):
                before = int(counts_all[:s, e0 + j].sum())
                assert int(pl["src_base"][s, j]) == want_off[j] + before
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_ep_placement_gloo(world):
    mp.spawn(_rank_main, args=(world, _free_port()), nprocs=world, join=True)


def test_ep_plan_rejects_uneven_split():
    sys.path.insert(0, ROOT)
    from routing_grouped_gemm_moe_b200 import ep
    with pytest.raises(ValueError):
        ep.plan(torch.zeros(3, 8, dtype=torch.int32), 0)
