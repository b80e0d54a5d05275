"""Context parallelism on CPU: two gloo ranks, each holding half of every request's pages.

Each rank attends over its slice (with the CPU oracle, since there is no GPU
here), the ranks all-gather their (out, lse), and the log-sum-exp merge of the
slices must equal attention over the whole cache.  This checks the slicing of
lengths and block tables and the exchange; the GPU kernels for the same steps
are checked in tests/test_gpu_context_parallel.py.
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist

    import oracle
    from variable_length_paged_b200 import workloads as W
    from variable_length_paged_b200.context_parallel import local_view

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = W.make_workload("cp", [1, 63, 64, 65, 700, 3000, 0, 129], num_q_heads=8, num_kv_heads=2, head_dim=64,
                            page_size=16, seed=9)
        ll, lbt = local_view(w.seq_lens, w.block_table, 16, world, rank)
        o, l, st = oracle.attention(w.q, w.k_cache, w.v_cache, lbt, ll, scale=w.problem.scale)
        parts_o = [torch.empty(o.shape, dtype=torch.float64) for _ in range(world)]
        parts_l = [torch.empty(l.shape, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(parts_o, torch.from_numpy(o))
        dist.all_gather(parts_l, torch.from_numpy(l))
        B, Hq, d = o.shape
        merged = np.zeros((B, Hq, d))
        merged_l = np.zeros((B, Hq))
        for b in range(B):
            for h in range(Hq):
                merged[b, h], merged_l[b, h] = oracle.combine(np.stack([p[b, h].numpy() for p in parts_o]),
                                                              np.array([p[b, h].item() for p in parts_l]))
        ref, ref_l, _ = oracle.attention(w.q, w.k_cache, w.v_cache, w.block_table, w.seq_lens, scale=w.problem.scale)
        results[rank] = (float(np.abs(merged - ref).max()),
                         bool(np.all(np.isneginf(merged_l) == np.isneginf(ref_l))),
                         float(np.nanmax(np.where(np.isneginf(ref_l), 0, np.abs(merged_l - ref_l)))), st,
                         ll.tolist())
    finally:
        dist.destroy_process_group()


def test_two_rank_slices_merge_to_the_whole():
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
    lens = np.array([1, 63, 64, 65, 700, 3000, 0, 129])
    got = np.array(res[0][4]) + np.array(res[1][4])
    assert np.array_equal(got, lens)  # the slices cover every token once
    for r in range(world):
        err, inf_ok, lerr, st, _ = res[r]
        assert st == 0 and inf_ok and err < 1e-12 and lerr < 1e-12


def test_slices_are_page_aligned_and_balanced():
    from variable_length_paged_b200.context_parallel import local_view, slice_pages
    lens = np.array([0, 1, 16, 17, 1000, 4096])
    bt = np.arange(6 * 300, dtype=np.int32).reshape(6, 300)
    for world in (1, 2, 3, 8):
        total = np.zeros_like(lens)
        for r in range(world):
            p0, p1 = slice_pages(lens, 16, world, r)
            ll, lbt = local_view(lens, bt, 16, world, r)
            total += ll
            for b in range(len(lens)):
                assert np.array_equal(lbt[b, :p1[b] - p0[b]], bt[b, p0[b]:p1[b]])
                assert np.all(lbt[b, p1[b] - p0[b]:] == -1)
                if r < world - 1:
                    assert ll[b] % 16 == 0  # only the last slice may end inside a page
        assert np.array_equal(total, lens)
