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
