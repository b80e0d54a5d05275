"""The failure path on the GPU: a decode launch whose pipeline waits run out.

da_test_stall_next_decode makes the next decode launch's load stage send
nothing (a flag that nothing sets), so every consumer wait gives up after a
short limit; the kernel records DA_DEV_TIMEOUT in the workspace status word and
returns.  Nothing traps or faults: the next step, on the same context and
buffers, must be correct again.  Covers the warp-MMA kernel (bf16, with and
without the in-decode merge, and FP8 multi-query) and the tcgen05 kernel (FP8
plain decode), whose teardown frees tensor memory on this path too.
"""

import time

import pytest
import torch

from gpu_helpers import check_against_oracle, check_against_oracle_fp8, check_mq_fp8_against_oracle
from variable_length_paged_b200 import da
from variable_length_paged_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("variant", ["bf16", "bf16_merge", "fp8", "fp8_multi_query"])
def test_stalled_launch_times_out_and_the_next_step_is_correct(da_lib, oracle_lib, variant):
    q_len = 2 if variant == "fp8_multi_query" else 1
    w = W.make_workload("stall", [3000, 17, 640, 1, 129], num_q_heads=16, num_kv_heads=2, head_dim=128,
                        page_size=64, seed=31, q_len=q_len)
    w8 = W.quantize_fp8(w) if variant.startswith("fp8") else None
    dw = (w8 if w8 is not None else w).to("cuda")
    prob = da.problem_from(w.problem)
    desc = da.da_plan_desc_init(prob, da.PLAN_DYNAMIC, 64, 7, merge_in_decode=variant == "bf16_merge")
    bufs = da.Buffers(prob, desc, "cuda")
    kw = dict(k_scale=dw.k_scale, v_scale=dw.v_scale) if w8 is not None else {}

    def step():
        da.decode_step(prob, desc, dw.q, dw.k_cache, dw.v_cache, dw.block_table, dw.seq_lens, bufs, **kw)
        torch.cuda.synchronize()

    step()
    assert da.da_read_status(bufs.ws) == (da.DEV_OK, -1)
    da.da_test_stall_next_decode(20000)  # 20 ms
    t0 = time.perf_counter()
    step()
    elapsed = time.perf_counter() - t0
    status, index = da.da_read_status(bufs.ws)
    assert status == da.DEV_TIMEOUT and index >= 0
    assert elapsed < 2.0, elapsed  # the short limit held, not the 2 s default
    step()  # same context, same buffers: a normal step again
    assert da.da_read_status(bufs.ws) == (da.DEV_OK, -1)
    if w8 is None:
        check_against_oracle(w, bufs.out, bufs.lse)
    elif q_len > 1:
        check_mq_fp8_against_oracle(w8, bufs.out, bufs.lse)
    else:
        check_against_oracle_fp8(w8, bufs.out, bufs.lse)
