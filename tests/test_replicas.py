"""The benchmark's replica plumbing on CPU: two gloo ranks, each timing its own
independent replica.  The whole-job value is the tokens of all ranks over the
slowest rank's time, and only rank 0 runs the oracle arm."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    import datetime

    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench

    ws, r, local = bench.dist_env()
    assert (ws, r, local) == (world, rank, rank)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dev = torch.device("cpu")
        # rank r "took" 10 * (r + 1) ms for 30 steps of batch 2
        total_ms = 10.0 * (rank + 1)
        bench.barrier(dev)
        slowest = bench.max_over_ranks(total_ms, dev)
        tokens = bench.sum_over_ranks(30 * 2, dev)
        out.put((rank, slowest, tokens, tokens / (slowest / 1e3)))

        # the reference arm returns at once on every rank but 0 (no work, no
        # collective), so the other ranks exit cleanly
        if rank != 0:
            class Args:
                batch, workload, warmup, steps = 1, "tiny", 3, 1
            assert bench.run_reference(Args()) is None
        bench.barrier(dev)
    finally:
        dist.destroy_process_group()


def test_two_gloo_replicas_report_the_whole_job():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, slowest, tokens, value in res:
        assert slowest == pytest.approx(20.0)       # the max over ranks
        assert tokens == pytest.approx(120.0)       # both ranks' tokens
        assert value == pytest.approx(120.0 / 0.020)


def test_single_process_helpers_are_identities():
    sys.path.insert(0, ROOT)
    import torch

    import bench

    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        os.environ.pop(k, None)
    assert bench.dist_env() == (1, 0, 0)
    dev = torch.device("cpu")
    assert bench.max_over_ranks(3.5, dev) == 3.5
    assert bench.sum_over_ranks(7.0, dev) == 7.0
    bench.barrier(dev)
