"""The decode trace (256 steps, batch 256, lengths changing every step) and the append kernel.

The plan is rebuilt on the device every step and checked bit-exactly against
the oracle's plan at every step; attention outputs are checked against the
fp64 oracle on every (request, head) at steps 0, 1, 127 and 255, and the same
two ends of the trace (steps 0 and 255) run once more over an FP8 E4M3 copy of
the cache (the tensor-core kernel) against the FP8 oracle; at the end the device
cache, written step by step by da_append_kv, must equal the host cache bit for
bit at every live token.
"""

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import assert_plan_equal, check_against_oracle, check_against_oracle_fp8, run_step_fp8
from variable_length_paged_b200 import da
from variable_length_paged_b200 import workloads as W
from variable_length_paged_b200.trace import DeviceTrace

pytestmark = pytest.mark.gpu


def test_append_kv_rows_land_in_their_pages(da_lib):
    w = W.make_workload("a", [63, 64, 1, 0, 200], num_q_heads=8, num_kv_heads=2, head_dim=128, page_size=64,
                        seed=3, max_pages_per_req=5, extra_pages=4)
    dw = w.to("cuda")
    prob = da.problem_from(w.problem)
    lens = w.seq_lens.copy()
    bt = w.block_table.copy()
    spare = sorted(set(range(w.problem.num_pages)) - set(bt[bt >= 0].tolist()))
    for b in range(len(lens)):  # grow every live request by one token (new page when full)
        if lens[b] == 0:
            continue
        if lens[b] % 64 == 0:
            bt[b, lens[b] // 64] = spare.pop()
        lens[b] += 1
    dw.block_table.copy_(torch.from_numpy(bt))
    dw.seq_lens.copy_(torch.from_numpy(lens))
    g = torch.Generator().manual_seed(5)
    nk = torch.randn(5, 2, 128, generator=g).to(torch.bfloat16)
    nv = torch.randn(5, 2, 128, generator=g).to(torch.bfloat16)
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    k0, v0 = dw.k_cache.clone(), dw.v_cache.clone()
    da.da_append_kv(prob, nk.cuda(), nv.cuda(), dw.block_table, dw.seq_lens, dw.k_cache, dw.v_cache, status)
    torch.cuda.synchronize()
    assert status.tolist() == [0, 0]
    ek, ev = k0.clone(), v0.clone()
    for b in range(5):
        if lens[b] == 0:
            continue
        pos = lens[b] - 1
        page, slot = bt[b, pos // 64], pos % 64
        ek[page, :, slot] = nk[b].cuda()
        ev[page, :, slot] = nv[b].cuda()
    same = lambda a, b: torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert same(dw.k_cache, ek) and same(dw.v_cache, ev)
    # a bad page id is reported and its row skipped
    dw.block_table[4, (lens[4] - 1) // 64] = w.problem.num_pages + 3
    da.da_append_kv(prob, nk.cuda(), nv.cuda(), dw.block_table, dw.seq_lens, dw.k_cache, dw.v_cache, status)
    torch.cuda.synchronize()
    assert status.tolist() == [da.DEV_BAD_PAGE, 4]


def test_decode_trace_256_steps(da_lib, oracle_lib):
    tr = W.DecodeTrace()
    dt = DeviceTrace(tr)
    prob = dt.prob
    desc = da.da_plan_desc_init(prob, da.PLAN_DYNAMIC, 64, 0)
    bufs = da.Buffers(prob, desc, "cuda")
    cap = prob.max_pages_per_req * prob.page_size
    for t in range(tr.steps):
        if t > 0:
            dt.advance()
        da.decode_step(prob, desc, dt.q, dt.k_cache, dt.v_cache, dt.block_table, dt.seq_lens, bufs)
        torch.cuda.synchronize()
        assert_plan_equal(da.read_plan(desc, bufs.ws), oracle.plan(tr.seq_lens, 64, desc.num_ctas, cap,
                                                                       start_cost=desc.start_cost))
        if t in (0, 1, 127, 255):
            check_against_oracle(tr.workload(), bufs.out, bufs.lse)
        if t in (0, tr.steps - 1):  # the trace's batch at both ends, over an FP8 copy of its cache
            w8 = W.quantize_fp8(tr.workload())
            out8, lse8, _, bufs8, _ = run_step_fp8(w8)
            assert da.da_read_status(bufs8.ws) == (0, -1)
            check_against_oracle_fp8(w8, out8, lse8)
            del out8, lse8, bufs8, w8
    assert dt.status.tolist() == [0, 0]
    assert da.da_read_status(bufs.ws) == (0, -1)
    # the device cache, built step by step by the append kernel, equals the host cache at live tokens
    live = np.zeros((prob.num_pages, prob.page_size), dtype=bool)
    for b in range(prob.batch):
        t = np.arange(int(tr.lens[b]))
        live[tr.block_table[b, t // prob.page_size], t % prob.page_size] = True
    m = torch.from_numpy(live)
    for dev_c, host_c in ((dt.k_cache, tr.k_cache), (dt.v_cache, tr.v_cache)):
        d = dev_c.cpu().permute(0, 2, 1, 3)[m]
        h = host_c.permute(0, 2, 1, 3)[m]
        assert torch.equal(d.view(torch.int16), h.view(torch.int16))


def test_recorded_trace_replays_the_live_trace(da_lib):
    """record + apply (the bench's device-only replay) leaves the device in the same state, bit for
    bit, as live advance steps, and the steps give the same outputs."""
    kw = dict(seed=9, batch=48, steps=40, num_q_heads=16, num_kv_heads=2, median=900.0, max_len=4096,
              p_finish=0.05)
    live, rec = DeviceTrace(W.DecodeTrace(**kw)), DeviceTrace(W.DecodeTrace(**kw))
    prob = live.prob
    desc = da.da_plan_desc_init(prob, da.PLAN_DYNAMIC, 64, 0)
    b1, b2 = da.Buffers(prob, desc, "cuda"), da.Buffers(prob, desc, "cuda")
    ups = rec.record(39)
    same = lambda a, b: torch.equal(a.view(torch.int16), b.view(torch.int16))
    for t in range(40):
        if t > 0:
            live.advance()
            rec.apply(ups[t - 1])
        for dt, b in ((live, b1), (rec, b2)):
            da.decode_step(prob, desc, dt.q, dt.k_cache, dt.v_cache, dt.block_table, dt.seq_lens, b)
        torch.cuda.synchronize()
        assert torch.equal(live.seq_lens, rec.seq_lens) and torch.equal(live.block_table, rec.block_table)
        assert same(b1.out, b2.out) and torch.equal(b1.lse, b2.lse)
    assert same(live.k_cache, rec.k_cache) and same(live.v_cache, rec.v_cache)
    assert live.status.tolist() == rec.status.tolist() == [0, 0]


def test_fused_plan_append_matches_separate_launches(da_lib, oracle_lib):
    """da_plan_append (one launch: block 0 plans, the others append) leaves the caches, the plan and
    the step's outputs bit for bit as da_append_kv followed by da_plan do, step after step; the plan
    also equals the oracle's, and the outputs the fp64 oracle's at the last step."""
    kw = dict(seed=17, batch=300, steps=24, num_q_heads=16, num_kv_heads=2, median=700.0, max_len=4096,
              p_finish=0.08)
    sep, fus = DeviceTrace(W.DecodeTrace(**kw)), DeviceTrace(W.DecodeTrace(**kw))
    host = W.DecodeTrace(**kw)
    prob = sep.prob
    desc = da.da_plan_desc_init(prob, da.PLAN_DYNAMIC, 64, 0)
    b1, b2 = da.Buffers(prob, desc, "cuda"), da.Buffers(prob, desc, "cuda")
    u1, u2 = sep.record(23), fus.record(23)
    same = lambda a, b: torch.equal(a.view(torch.int16), b.view(torch.int16))
    cap = prob.max_pages_per_req * prob.page_size
    for t in range(24):
        if t > 0:
            sep.apply(u1[t - 1])
            fus.apply(u2[t - 1], plan=(desc, b2.ws))
            host.advance()
        da.decode_step(prob, desc, sep.q, sep.k_cache, sep.v_cache, sep.block_table, sep.seq_lens, b1)
        da.decode_step(prob, desc, fus.q, fus.k_cache, fus.v_cache, fus.block_table, fus.seq_lens, b2,
                       planned=t > 0)
        torch.cuda.synchronize()
        assert torch.equal(b1.ws, b2.ws)
        assert_plan_equal(da.read_plan(desc, b2.ws), oracle.plan(host.seq_lens, 64, desc.num_ctas, cap,
                                                                   start_cost=desc.start_cost))
        assert same(b1.out, b2.out) and torch.equal(b1.lse, b2.lse)
        assert same(sep.k_cache, fus.k_cache) and same(sep.v_cache, fus.v_cache)
    check_against_oracle(host.workload(), b2.out, b2.lse)
    assert sep.status.tolist() == fus.status.tolist() == [0, 0]


def test_fused_plan_append_reports_bad_pages_and_lengths(da_lib):
    """Append errors reach the append status pair, plan errors the workspace, as with the two calls."""
    w = W.make_workload("a", [63, 64, 1, 0, 200], num_q_heads=8, num_kv_heads=2, head_dim=128, page_size=64,
                        seed=3, max_pages_per_req=5, extra_pages=4)
    dw = w.to("cuda")
    prob = da.problem_from(w.problem)
    desc = da.da_plan_desc_init(prob, da.PLAN_DYNAMIC, 64, 0)
    bufs = da.Buffers(prob, desc, "cuda")
    nk = torch.zeros(5, 2, 128, dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    dw.block_table[2, 0] = w.problem.num_pages + 1
    da.da_plan_append(prob, desc, dw.seq_lens, bufs.ws, nk, nk, dw.block_table, dw.k_cache, dw.v_cache, status)
    torch.cuda.synchronize()
    assert status.tolist() == [da.DEV_BAD_PAGE, 2]
    assert da.da_read_status(bufs.ws) == (0, -1)  # the planner reads lengths only
    status.zero_()
    dw.seq_lens[3] = -4
    da.da_plan_append(prob, desc, dw.seq_lens, bufs.ws, nk, nk, dw.block_table, dw.k_cache, dw.v_cache, status)
    torch.cuda.synchronize()
    assert status.tolist()[0] != 0
    assert da.da_read_status(bufs.ws) == (da.DEV_BAD_SEQLEN, 3)
