"""Context parallelism on one GPU: W ranks emulated one after another in one process.

Each emulated rank runs the decode step on its slice of every request's pages;
da_merge_partials then merges the W results.  The merge must match attention
over the whole cache (fp64 oracle), within the tolerance of the other parity
tests.  The exchange itself (an all-gather) is covered on CPU with gloo.
"""

import numpy as np
import pytest
import torch

from gpu_helpers import check_against_oracle
from variable_length_paged_b200 import da
from variable_length_paged_b200 import workloads as W
from variable_length_paged_b200.context_parallel import local_view

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_emulated_ranks_merge_to_the_whole(da_lib, oracle_lib, world):
    w = W.make_workload("cp", [1, 63, 64, 65, 700, 3000, 0, 129, 20000], num_q_heads=16, num_kv_heads=2,
                        head_dim=128, page_size=64, seed=11)
    dw = w.to("cuda")
    prob = da.problem_from(dw.problem)
    desc = da.da_plan_desc_init(prob, da.PLAN_DYNAMIC, 64, 0)
    bufs = da.Buffers(prob, desc, "cuda")
    parts_out = torch.empty((world,) + tuple(bufs.out.shape), dtype=torch.bfloat16, device="cuda")
    parts_lse = torch.empty((world,) + tuple(bufs.lse.shape), dtype=torch.float32, device="cuda")
    for r in range(world):
        ll, lbt = local_view(w.seq_lens, w.block_table, 64, world, r)
        sl = torch.from_numpy(ll).cuda()
        bt = torch.from_numpy(lbt).cuda()
        da.decode_step(prob, desc, dw.q, dw.k_cache, dw.v_cache, bt, sl, bufs)
        parts_out[r].copy_(bufs.out)
        parts_lse[r].copy_(bufs.lse)
    out = torch.full_like(bufs.out, float("nan"))
    lse = torch.full_like(bufs.lse, float("nan"))
    da.da_merge_partials(parts_out, parts_lse, out, lse)
    torch.cuda.synchronize()
    check_against_oracle(w, out, lse)


def test_cp_decode_step_single_rank_group(da_lib, oracle_lib):
    """The distributed entry point end to end in a one-rank NCCL group."""
    import os

    import torch.distributed as dist

    from variable_length_paged_b200.context_parallel import cp_decode_step
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", "29611")
    created = not dist.is_initialized()
    if created:
        dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        w = W.make_workload("cp1", [5, 700, 3000], num_q_heads=8, num_kv_heads=1, head_dim=128, page_size=64, seed=12)
        dw = w.to("cuda")
        prob = da.problem_from(dw.problem)
        desc = da.da_plan_desc_init(prob, da.PLAN_DYNAMIC, 64, 0)
        bufs = da.Buffers(prob, desc, "cuda")
        out = torch.empty_like(bufs.out)
        lse = torch.empty_like(bufs.lse)
        cp_decode_step(prob, desc, dw.q, dw.k_cache, dw.v_cache, dw.block_table, dw.seq_lens, bufs, out, lse)
        torch.cuda.synchronize()
        check_against_oracle(w, out, lse)
        # on a side stream: the gather and the merge follow that stream's decode
        side = torch.cuda.Stream()
        out.fill_(float("nan"))
        lse.fill_(float("nan"))
        cp_decode_step(prob, desc, dw.q, dw.k_cache, dw.v_cache, dw.block_table, dw.seq_lens, bufs, out, lse,
                       stream=side)
        torch.cuda.synchronize()
        check_against_oracle(w, out, lse)
    finally:
        if created:
            dist.destroy_process_group()
