"""da_decode_step_noalloc: the decode step for callers that cannot allocate device memory.

Such callers (an op whose per-call hook must not allocate, an engine that gave
nearly all device memory to its KV-cache pool) use the library's own static
16 MiB device scratch instead of a caller workspace.  This file is collected
last on purpose, so that a failure here does not hide any other test's result.
It checks, through the C ABI, that two calls in a row on different batches give
the same result as the allocating entry points (da_plan + da_decode_attention
+ da_combine) within the tolerance of the other parity tests, that a problem
too large for the scratch is refused before anything is enqueued, and that the
device-side status of a step (a bad page id, a wait that ran out) reaches the
caller through da_noalloc_read_status, the step's only status reader.
"""

import ctypes
import time

import numpy as np
import pytest
import torch

from gpu_helpers import LSE_ATOL, OUT_ATOL, OUT_RTOL, run_step
from variable_length_paged_b200 import da
from variable_length_paged_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _noalloc(dw, tile=64, width=0):
    """One step through da_decode_step_noalloc; synchronises."""
    prob = da.problem_from(dw.problem)
    out = torch.full_like(dw.q, float("nan"))
    lse = torch.full(dw.q.shape[:2], float("nan"), dtype=torch.float32, device=dw.q.device)
    rc = da.lib().da_decode_step_noalloc(ctypes.byref(prob), tile, width, dw.q.data_ptr(), dw.k_cache.data_ptr(),
                                        dw.v_cache.data_ptr(), dw.block_table.data_ptr(), dw.seq_lens.data_ptr(),
                                        out.data_ptr(), lse.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == da.OK, da.status_string(rc)
    torch.cuda.synchronize()
    return out, lse


def _assert_close(out, lse, ref_out, ref_lse):
    o, r = out.float().cpu().double(), ref_out.float().cpu().double()
    assert torch.isfinite(o).all()
    assert ((o - r).abs() <= OUT_ATOL + OUT_RTOL * r.abs()).all()
    a, b = lse.cpu().double(), ref_lse.cpu().double()
    both = torch.isneginf(a) & torch.isneginf(b)
    assert (torch.where(both, torch.zeros_like(a), (a - b).abs()) <= LSE_ATOL).all()


def test_two_calls_match_the_allocating_entry_points(da_lib):
    batches = [
        W.make_workload("a", np.random.default_rng(1).integers(1000, 16001, 24), num_q_heads=64, num_kv_heads=8,
                        head_dim=128, page_size=64, seed=11),
        W.make_workload("b", [0, 1, 7000, 65, 300, 129, 4096], num_q_heads=32, num_kv_heads=4, head_dim=128,
                        page_size=64, seed=12),
    ]
    for w in batches:  # two calls in a row, the second on a different batch
        dw = w.to("cuda")
        ref_out, ref_lse, *_ = run_step(None, dw=dw)
        ref_out, ref_lse = ref_out.clone(), ref_lse.clone()
        out, lse = _noalloc(dw)
        _assert_close(out, lse, ref_out, ref_lse)


def test_too_large_for_the_scratch_is_refused(da_lib):
    B = 2048  # (C + B - 1) segments x 64 heads x 128 x 4 bytes of partials is far above 16 MiB
    prob = da.problem(B, 64, 8, 128, 64, 4, 8, 0.088)
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    p = dummy.data_ptr()
    rc = da.lib().da_decode_step_noalloc(ctypes.byref(prob), 64, 37, p, p, p, p, p, p, p, None)
    assert rc == da.ERR_WORKSPACE
    assert da.lib().da_decode_step_noalloc(ctypes.byref(prob), 64, 37, *([None] * 7), None) == da.ERR_WORKSPACE


def _status():
    st, bad = ctypes.c_int32(-7), ctypes.c_int32(-7)
    rc = da.lib().da_noalloc_read_status(ctypes.byref(st), ctypes.byref(bad), torch.cuda.current_stream().cuda_stream)
    assert rc == da.OK, da.status_string(rc)
    return st.value, bad.value


def test_status_of_a_step_reaches_the_caller(da_lib):
    w = W.make_workload("status", [300, 500, 2000], num_q_heads=8, num_kv_heads=1, head_dim=128, page_size=64,
                        seed=21)
    dw = w.to("cuda")
    ref_out, ref_lse, *_ = run_step(None, dw=dw)
    ref_out, ref_lse = ref_out.clone(), ref_lse.clone()
    _noalloc(dw)
    assert _status() == (da.DEV_OK, -1)
    # a block-table entry outside the cache: that chunk is skipped and request 1 is reported
    good = int(dw.block_table[1, 2])
    dw.block_table[1, 2] = w.problem.num_pages + 5
    _noalloc(dw)
    assert _status() == (da.DEV_BAD_PAGE, 1)
    dw.block_table[1, 2] = good
    # a decode launch whose loads never come: every wait runs out after 20 ms
    da.da_test_stall_next_decode(20000)
    t0 = time.perf_counter()
    _noalloc(dw)
    elapsed = time.perf_counter() - t0
    st, bad = _status()
    assert st == da.DEV_TIMEOUT and bad >= 0
    assert elapsed < 2.0, elapsed  # the short limit held, not the 2 s default
    # the next call plans afresh (status reset) and is correct again
    out, lse = _noalloc(dw)
    assert _status() == (da.DEV_OK, -1)
    _assert_close(out, lse, ref_out, ref_lse)
