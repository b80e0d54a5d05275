"""The combine's two kernels, on either side of the switch between them.

The lean kernel (128 threads, running max per warp) serves grids of more than 444
(request, query head) blocks; the wide one (256 threads, global max first, eight segments'
loads in flight per warp) serves smaller grids.  The choice depends on the batch and head
counts only.  Both must give the oracle's result; a batch of 111 requests at 4 query heads
(444 blocks) takes the wide kernel and one of 112 (448 blocks) the lean one, each request split
over many segments.
"""

import numpy as np
import pytest

from gpu_helpers import check_against_oracle, run_step
from variable_length_paged_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B", [111, 112])
def test_combine_either_side_of_the_switch(da_lib, oracle_lib, B):
    rng = np.random.default_rng(B)
    lens = rng.integers(200, 3001, size=B)
    lens[::17] = 0  # requests without segments: out 0, lse -inf from the combine
    w = W.make_workload("combine_switch", lens, num_q_heads=4, num_kv_heads=1, head_dim=128, page_size=64, seed=B)
    out, lse, desc, bufs, _ = run_step(w, width=1000)
    assert desc.max_segments >= 1000
    check_against_oracle(w, out, lse)


@pytest.mark.parametrize("B", [111, 112])
def test_combine_either_side_of_the_switch_fp32_out(da_lib, oracle_lib, B):
    """With fp32 output every request goes through the combine, one segment too."""
    import torch
    from variable_length_paged_b200 import da
    rng = np.random.default_rng(B + 7)
    lens = rng.integers(1, 3001, size=B)
    w = W.make_workload("combine_switch_f32", lens, num_q_heads=4, num_kv_heads=1, head_dim=128, page_size=64,
                        seed=B + 7)
    dw = w.to("cuda")
    prob = da.problem_from(dw.problem)
    desc = da.da_plan_desc_init(prob, da.PLAN_DYNAMIC, 64, 300, out_f32=True)
    bufs = da.Buffers(prob, desc, "cuda")
    for t in (bufs.partial_o, bufs.partial_lse, bufs.out, bufs.lse):
        t.fill_(float("nan"))
    da.decode_step(prob, desc, dw.q, dw.k_cache, dw.v_cache, dw.block_table, dw.seq_lens, bufs)
    torch.cuda.synchronize()
    check_against_oracle(w, bufs.out, bufs.lse)
