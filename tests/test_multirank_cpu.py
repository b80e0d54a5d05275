"""The N>1 host logic of bench.py on CPU: two gloo ranks, no GPU.

Requests are independent, so ranks share no data; the only exchange is the
timing reduction (max over ranks) and the byte count (sum over ranks).
"""

import os
import socket

import numpy as np
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import torch.distributed as dist

    import bench
    from variable_length_paged_b200 import workloads as W
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mx, sm = bench.reduce_max_sum([1.5 + rank, 10.0 - rank], [100.0 * (rank + 1)], world)
        gen = W.CONFIGS["mixed"]
        w = gen(seed=gen.__defaults__[0] + 1000 * rank) if rank else gen()
        bench.barrier(world)
        results[rank] = (mx, sm, w.seq_lens.tolist())
    finally:
        dist.destroy_process_group()


def test_two_rank_reduction_and_shards():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=240)
            assert p.exitcode == 0
        res = dict(results)
    for r in range(world):
        mx, sm, _ = res[r]
        assert mx == [2.5, 10.0] and sm == [300.0]
    # each rank draws its own batch of the same shape
    a, b = np.array(res[0][2]), np.array(res[1][2])
    assert a.shape == b.shape and not np.array_equal(a, b)
    assert a.min() >= 1000 and b.max() <= 16000
