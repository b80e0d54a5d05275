"""Failure of one rank in the N > 1 host path, made on the host (no GPU): a rank that exits, or one
that stays alive but never joins the collective, must turn the other rank's next collective (the
timing reduction of bench.py, the all-gather of the cross-GPU split) into an error within the
process group's timeout, never into a hang."""

import os
import socket
import time

import pytest
import torch.multiprocessing as mp

TIMEOUT_S = 5


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, mode, op, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import torch
    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=TIMEOUT_S))
    if rank == 1:
        if mode == "stalls":
            time.sleep(TIMEOUT_S + 3)  # alive past the timeout, never joins
        os._exit(0)  # leaves without its share of the collective
    t0 = time.monotonic()
    try:
        if op == "reduce":
            bench.reduce_max_sum([1.0], [2.0], world)
        else:
            out = [torch.zeros(4) for _ in range(world)]
            dist.all_gather(out, torch.ones(4))
        results[0] = ("no error", time.monotonic() - t0)
    except Exception as e:  # the error the surviving rank must see
        results[0] = (type(e).__name__, time.monotonic() - t0)
    os._exit(0)


@pytest.mark.parametrize("mode", ["exits", "stalls"])
@pytest.mark.parametrize("op", ["reduce", "all_gather"])
def test_surviving_rank_gets_an_error(mode, op):
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, mode, op, results)) for r in range(world)]
        for p in procs:
            p.start()
        deadline = time.monotonic() + 6 * TIMEOUT_S + 60
        for p in procs:
            p.join(timeout=max(1.0, deadline - time.monotonic()))
        alive = [p for p in procs if p.is_alive()]
        for p in alive:
            p.kill()
        assert not alive, "a rank hung"
        kind, elapsed = results[0]
        print(mode, op, kind, round(elapsed, 2))
        assert kind != "no error"
        assert elapsed < 3 * TIMEOUT_S + 30, elapsed
