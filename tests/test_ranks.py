"""The N > 1 path of bench.py on CPU ranks (gloo, world size 2).

bench.py runs one process per GPU. The problems are independent (weak scaling):
each rank draws its own prefill (seed + 1000·rank), and the only collectives
are the timing barrier and the max over ranks of the per-rank times. The
whole-job value is every rank's tokens over that max. The reference arm runs
on rank 0 only. These checks use the same Ranks class with the gloo backend.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import dataclasses
    import bench
    import workloads as W
    ranks = bench.Ranks(world, backend="gloo")
    ranks.barrier()
    # per-rank time: rank r reports 10 + r ms; every rank must see the max
    t_max = ranks.max(10.0 + rank)
    cfg = dataclasses.replace(W.CONFIGS[bench.PREFILL_CFG],
                              seed=W.CONFIGS[bench.PREFILL_CFG].seed + 1000 * ranks.rank)
    ranks.close()
    q.put((rank, ranks.world, t_max, cfg.seed))


def test_two_ranks_barrier_max_and_seeds():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(world))
    assert [r[0] for r in res] == [0, 1]
    assert all(r[1] == world for r in res)
    assert all(r[2] == 11.0 for r in res)            # max over ranks, seen by all
    assert res[1][3] - res[0][3] == 1000               # independent problems per rank
    # whole-job value: all ranks' tokens over the slowest rank's time
    L = 131072
    assert pytest.approx(L * world / (res[0][2] / 1e3)) == 2 * L / 0.011


def _reference_rank(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world)})
    sys.path.insert(0, ROOT)
    import argparse
    import contextlib
    import io
    import bench
    buf = io.StringIO()
    args = argparse.Namespace(gpus=world, steps=1, warmup=0, L=512, impl="reference")
    if rank != 0:
        with contextlib.redirect_stdout(buf):
            bench.run_reference(args)
    q.put((rank, buf.getvalue()))


def test_reference_arm_runs_on_rank_zero_only():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_reference_rank, args=(1, 2, 0, q))
    p.start()
    p.join(timeout=120)
    assert p.exitcode == 0
    rank, out = q.get(timeout=5)
    assert rank == 1 and out == ""


def _plan_rank(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    import bench
    import sparse_attention_long_02_b200 as dsa
    ranks = bench.Ranks(world, backend="gloo")
    L, chunk = 131072, 4096
    mine = dsa.plan_prefill_chunks(L, L, 64, 128, 2048, chunk, ranks.world, ranks.rank)
    # every rank's share, gathered: the plan needs no communication, so the
    # shares must tile the rows without overlap
    buf = torch.full((L // chunk,), -1, dtype=torch.int64)
    buf[:len(mine)] = torch.tensor(mine, dtype=torch.int64)
    parts = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(parts, buf)
    # rows each rank runs, and the whole-job value at a per-rank time of 10 + r ms
    rows = sum(min(chunk, L - c0) for c0 in mine)
    t_max = ranks.max(10.0 + rank)
    ranks.close()
    q.put((rank, [p[p >= 0].tolist() for p in parts], rows, t_max))


def test_row_shards_tile_one_prefill_over_two_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_plan_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(world))
    assert res[0][1] == res[1][1]                       # both ranks see the same plan
    shares = res[0][1]
    assert sorted(c for s in shares for c in s) == list(range(0, 131072, 4096))
    assert res[0][2] + res[1][2] == 131072              # all rows, once
    # strong scaling: one prefill's tokens over the slowest rank's time
    assert res[0][3] == res[1][3] == 11.0
