"""da_decode_step_host: the whole step from host inputs to host outputs in one C call.

Checked against the fp64 oracle, and bit for bit against the separate device
calls (the same kernels on the same inputs must give the same bits).
"""

import numpy as np
import pytest
import torch

from gpu_helpers import (check_against_oracle, check_against_oracle_fp8, check_mq_against_oracle, run_step,
                         run_step_fp8)
from variable_length_paged_b200 import da
from variable_length_paged_b200 import workloads as W

pytestmark = pytest.mark.gpu

RAGGED = [0, 1, 15, 63, 64, 65, 1000, 4097, 17, 300]


def ragged(q_len=1, seed=11):
    return W.make_workload("ragged", RAGGED, num_q_heads=16, num_kv_heads=2, head_dim=128, page_size=64, seed=seed,
                           q_len=q_len, recipe="host-step test")


def host_step(w, kind=da.PLAN_DYNAMIC, pinned=True, w8=None, seq_lens=None, state=None):
    """Run da_decode_step_host (FP8 cache when `w8` is given); returns (out_host, lse_host, state),
    with state reusable for later calls."""
    if state is None:
        dw = (w8 if w8 is not None else w).to("cuda")
        prob = da.problem_from(w.problem)
        desc = da.da_plan_desc_init(prob, kind, 64, 0)
        bufs = da.Buffers(prob, desc, "cuda")
        for t in (bufs.partial_o, bufs.partial_lse, bufs.out, bufs.lse):
            t.fill_(float("nan"))
        for t in (dw.q, dw.seq_lens, dw.block_table):  # the call must copy the inputs itself
            t.zero_()
        ks, vs = dw.k_scale, dw.v_scale

        def host(t):
            return t.pin_memory() if pinned else t.clone()

        q_h = host(w.q.contiguous())
        bt_h = host(torch.from_numpy(np.ascontiguousarray(w.block_table)))
        sl_h = host(torch.from_numpy(np.ascontiguousarray(w.seq_lens, dtype=np.int32)))
        out_h = host(torch.full(bufs.out.shape, float("nan"), dtype=torch.bfloat16))
        lse_h = host(torch.full(bufs.lse.shape, float("nan"), dtype=torch.float32))
        state = dict(dw=dw, prob=prob, desc=desc, bufs=bufs, ks=ks, vs=vs, q_h=q_h, bt_h=bt_h, sl_h=sl_h,
                     out_h=out_h, lse_h=lse_h)
    s = state
    if seq_lens is not None:
        s["sl_h"].copy_(torch.from_numpy(np.asarray(seq_lens, dtype=np.int32)))
    dw = s["dw"]
    da.da_decode_step_host(s["prob"], s["desc"], s["q_h"], s["bt_h"], s["sl_h"], dw.k_cache, dw.v_cache, dw.q,
                           dw.block_table, dw.seq_lens, s["bufs"], s["out_h"], s["lse_h"], k_scale=s["ks"],
                           v_scale=s["vs"])
    torch.cuda.synchronize()
    return s["out_h"], s["lse_h"], s


@pytest.mark.parametrize("kind", [da.PLAN_DYNAMIC, da.PLAN_STATIC])
def test_host_step_matches_oracle_and_device_calls(kind):
    w = ragged()
    out_h, lse_h, _ = host_step(w, kind=kind)
    check_against_oracle(w, out_h, lse_h)
    out_d, lse_d, *_ = run_step(w, kind=kind)
    assert torch.equal(out_h.view(torch.int16), out_d.cpu().view(torch.int16))
    assert torch.equal(lse_h, lse_d.cpu())


def test_host_step_tiny():
    w = W.tiny()
    out_h, lse_h, _ = host_step(w)
    check_against_oracle(w, out_h, lse_h)


def test_host_step_pageable_buffers():
    w = ragged(seed=12)
    out_h, lse_h, _ = host_step(w, pinned=False)
    check_against_oracle(w, out_h, lse_h)


def test_host_step_follows_new_lengths():
    """The host lengths are copied every call: the same state serves steps of different lengths."""
    w = ragged(seed=13)
    out_h, lse_h, st = host_step(w)
    check_against_oracle(w, out_h, lse_h)
    shorter = np.array([max(0, l - 7) for l in RAGGED], np.int32)
    shorter[1] = 0  # a request finishes
    out_h, lse_h, _ = host_step(w, seq_lens=shorter, state=st)
    check_against_oracle(w, out_h, lse_h, seq_lens=shorter)


def test_host_step_fp8():
    w8 = W.quantize_fp8(ragged(seed=14))
    out_h, lse_h, _ = host_step(w8.base, w8=w8)
    check_against_oracle_fp8(w8, out_h, lse_h)
    out_d, lse_d, *_ = run_step_fp8(w8)
    assert torch.equal(out_h.view(torch.int16), out_d.cpu().view(torch.int16))
    assert torch.equal(lse_h, lse_d.cpu())


def test_host_step_multi_query():
    w = ragged(q_len=2, seed=15)  # 2 queries x 8 heads per KV head fill the 16 MMA rows
    out_h, lse_h, _ = host_step(w)
    assert out_h.shape == (len(RAGGED), 2, 16, 128)
    check_mq_against_oracle(w, out_h, lse_h)


def test_mapped_host_buffers_skip_the_copies():
    """With pinned (mapped) host buffers the plan launch itself brings lengths, block table and q in,
    and out / lse are written in place: the device outputs stay untouched, and the results equal the
    copy path's (pageable buffers) bit for bit."""
    w = ragged(seed=16)
    out_p, lse_p, st = host_step(w, pinned=True)
    dw, bufs = st["dw"], st["bufs"]
    assert torch.equal(dw.q.cpu().view(torch.int16), w.q.view(torch.int16))  # copied by the plan launch
    assert torch.equal(dw.seq_lens.cpu(), torch.from_numpy(w.seq_lens))
    assert torch.equal(dw.block_table.cpu(), torch.from_numpy(w.block_table))
    assert torch.isnan(bufs.out.float()).all() and torch.isnan(bufs.lse).all()  # never written
    check_against_oracle(w, out_p, lse_p)
    out_c, lse_c, st_c = host_step(w, pinned=False)
    assert not torch.isnan(st_c["bufs"].lse).all()  # the copy path wrote the device outputs
    assert torch.equal(out_p.view(torch.int16), out_c.view(torch.int16)) and torch.equal(lse_p, lse_c)


def test_unaligned_pinned_views():
    """q 8 bytes past a 16-byte boundary is brought in by 4-byte pieces; lse 4 bytes past one is not
    written in place but copied back.  Same results."""
    w = ragged(seed=17)
    out_h, lse_h, st = host_step(w)
    ref_out, ref_lse = out_h.clone(), lse_h.clone()
    s = st
    q_big = torch.empty(w.q.numel() + 8, dtype=torch.bfloat16).pin_memory()
    q_off = q_big[4:4 + w.q.numel()].view(w.q.shape)
    q_off.copy_(w.q)
    lse_big = torch.full((s["lse_h"].numel() + 2,), float("nan")).pin_memory()
    lse_off = lse_big[1:1 + s["lse_h"].numel()].view(s["lse_h"].shape)
    s["q_h"], s["lse_h"] = q_off, lse_off
    s["dw"].q.zero_()
    s["bufs"].lse.fill_(float("nan"))
    out2, lse2, _ = host_step(w, state=s)
    assert torch.equal(s["dw"].q.cpu().view(torch.int16), w.q.view(torch.int16))
    assert not torch.isnan(s["bufs"].lse).all()  # lse went through its device copy
    assert torch.equal(out2.view(torch.int16), ref_out.view(torch.int16)) and torch.equal(lse2, ref_lse)


@pytest.mark.parametrize("kind", [da.PLAN_DYNAMIC, da.PLAN_STATIC])
def test_host_inputs_plan_matches_the_oracle_plan(kind, oracle_lib):
    """The plan built from host lengths inside the input launch is the oracle's plan, for a batch
    larger than one block's pass (600 requests) and with lengths changing between calls."""
    import oracle
    from gpu_helpers import assert_plan_equal
    lens = np.random.default_rng(5).integers(0, 3000, 600).astype(np.int32)
    w = W.make_workload("wide", lens.tolist(), num_q_heads=8, num_kv_heads=1, head_dim=64, page_size=64, seed=18,
                        recipe="host-step plan test")
    _, _, st = host_step(w, kind=kind)
    cap = w.problem.max_pages_per_req * w.problem.page_size
    for t in range(3):
        cur = np.maximum(lens - 100 * t, 0).astype(np.int32)
        out_h, lse_h, st = host_step(w, kind=kind, seq_lens=cur, state=st)
        d = st["desc"]
        got = da.read_plan(d, st["bufs"].ws)
        want = (oracle.plan(cur, 64, d.num_ctas, cap, start_cost=d.start_cost) if kind == da.PLAN_DYNAMIC
                else oracle.static_plan(cur, 64, d.splits, cap))
        assert_plan_equal(got, want)
        assert torch.equal(st["dw"].seq_lens.cpu(), torch.from_numpy(cur))
    check_against_oracle(w, out_h, lse_h, seq_lens=cur)


def test_large_q_is_read_in_place():
    """A q above 1 MiB in mapped memory is read by the decode kernel over the bus (q_dev untouched);
    lengths and block table still come in through the plan launch.  Same bits as the copy path."""
    lens = np.random.default_rng(6).integers(0, 700, 160).astype(np.int32)
    w = W.make_workload("big-q", lens.tolist(), num_q_heads=32, num_kv_heads=4, head_dim=128, page_size=64,
                        seed=19, recipe="host-step large q")
    assert w.q.numel() * 2 > (1 << 20)
    for w8 in (None, W.quantize_fp8(w)):
        base = w if w8 is None else w8.base
        out_p, lse_p, st = host_step(base, w8=w8)
        assert torch.count_nonzero(st["dw"].q) == 0  # never copied in
        assert torch.equal(st["dw"].seq_lens.cpu(), torch.from_numpy(w.seq_lens))
        if w8 is None:
            check_against_oracle(w, out_p, lse_p)
        else:
            check_against_oracle_fp8(w8, out_p, lse_p)
        out_c, lse_c, _ = host_step(base, w8=w8, pinned=False)
        assert torch.equal(out_p.view(torch.int16), out_c.view(torch.int16)) and torch.equal(lse_p, lse_c)


def test_large_multi_query_q_is_read_in_place():
    """Multi-query decode with a q above 1 MiB in mapped memory: the multi-query kernel reads it over
    the bus; causal limits and results as on the copy path."""
    lens = np.random.default_rng(7).integers(2, 600, 160).astype(np.int32)
    w = W.make_workload("big-q-mq", lens.tolist(), num_q_heads=32, num_kv_heads=4, head_dim=128, page_size=64,
                        seed=20, q_len=2, recipe="host-step large multi-query q")
    assert w.q.numel() * 2 > (1 << 20)
    out_p, lse_p, st = host_step(w)
    assert torch.count_nonzero(st["dw"].q) == 0  # never copied in
    check_mq_against_oracle(w, out_p, lse_p)
    out_c, lse_c, _ = host_step(w, pinned=False)
    assert torch.equal(out_p.view(torch.int16), out_c.view(torch.int16)) and torch.equal(lse_p, lse_c)
