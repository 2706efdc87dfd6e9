"""Host logic of the N > 1 bench path on CPU: two gloo ranks.

The path shards by independent batches, so ranks only meet at the barriers
around the timed region and at the reduction of the timings. The step time
reported is the maximum over ranks; the work is the sum over ranks.
"""
import contextlib
import io
import os
import socket

import pytest
import torch
import torch.distributed as tdist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import bench

    tdist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        times = (1.0 + rank, 10.0 - 3 * rank)   # rank 0: (1, 10); rank 1: (2, 7)
        (ms, attn_ms), units = bench.reduce_over_ranks(tdist, torch.device("cpu"), times, 100 * (rank + 1))
        tdist.barrier()
        (e2e,), _ = bench.reduce_over_ranks(tdist, torch.device("cpu"), (5.0 * (rank + 1),), 0)
        results[rank] = (ms, attn_ms, units, e2e)
    finally:
        tdist.destroy_process_group()


def _run_two_ranks(ctx, results, world):
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(60)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    return codes


@pytest.mark.timeout(300)
def test_two_ranks_max_time_sum_units():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        # the free port can be taken between the probe and the rendezvous:
        # a failed start gets a new port (at most three tries)
        for _ in range(3):
            codes = _run_two_ranks(ctx, results, world)
            if codes == [0, 0]:
                break
        assert codes == [0, 0]
        got = dict(results)
    for rank in range(world):
        assert got[rank] == (2.0, 10.0, 300.0, 10.0)


def test_single_process_reduction_is_identity():
    import bench
    (a, b), u = bench.reduce_over_ranks(None, torch.device("cpu"), (1.5, 2.5), 42)
    assert (a, b, u) == (1.5, 2.5, 42.0)


def test_reference_arm_other_ranks_do_nothing(monkeypatch):
    import bench
    import workloads
    monkeypatch.setenv("RANK", "1")
    args = bench.parse(["--impl", "reference", "--steps", "1", "--warmup", "0"])
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args, workloads.get(1))
    assert buf.getvalue() == ""
