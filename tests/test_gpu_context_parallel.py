"""Context parallelism on one GPU: W ranks emulated one after another in one process.

Each emulated rank runs the decode step, with fp32 output, on its slice of every
request's pages; da_merge_partials_f32 then merges the W results.  The merge must match attention
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


def _bf16_ulp(x):
    """Spacing of bf16 values at |x| (8 significant bits)."""
    a = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_emulated_ranks_merge_to_the_whole(da_lib, oracle_lib, world):
    """W slices, each run as an ordinary step with fp32 output, merged by da_merge_partials_f32:
    the result matches attention over the whole cache, and the merge itself is the exact
    log-sum-exp merge of the fp32 parts rounded once to bf16 (no part is rounded before it)."""
    w = W.make_workload("cp", [1, 63, 64, 65, 700, 3000, 0, 129, 20000], num_q_heads=16, num_kv_heads=2,
                        head_dim=128, page_size=64, seed=11)
    dw = w.to("cuda")
    prob = da.problem_from(dw.problem)
    desc = da.da_plan_desc_init(prob, da.PLAN_DYNAMIC, 64, 0, out_f32=True)
    bufs = da.Buffers(prob, desc, "cuda")
    assert bufs.out.dtype == torch.float32
    parts_out = torch.empty((world,) + tuple(bufs.out.shape), dtype=torch.float32, device="cuda")
    parts_lse = torch.empty((world,) + tuple(bufs.lse.shape), dtype=torch.float32, device="cuda")
    for r in range(world):
        ll, lbt = local_view(w.seq_lens, w.block_table, 64, world, r)
        sl = torch.from_numpy(ll).cuda()
        bt = torch.from_numpy(lbt).cuda()
        bufs.out.fill_(float("nan"))
        da.decode_step(prob, desc, dw.q, dw.k_cache, dw.v_cache, bt, sl, bufs)
        parts_out[r].copy_(bufs.out)
        parts_lse[r].copy_(bufs.lse)
    out = torch.full(bufs.out.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full_like(bufs.lse, float("nan"))
    da.da_merge_partials_f32(parts_out, parts_lse, out, lse)
    torch.cuda.synchronize()
    err, _ = check_against_oracle(w, out, lse)

    # the merge alone, against the fp64 log-sum-exp merge of the same fp32 parts
    po = parts_out.cpu().double().numpy()
    pl = parts_lse.cpu().double().numpy()
    M = pl.max(axis=0)
    live = np.isfinite(M)
    Ms = np.where(live, M, 0.0)
    wts = np.exp(pl - Ms[None])  # 0 for empty parts
    L = wts.sum(axis=0)
    ref_lse = np.where(live, Ms + np.log(np.where(live, L, 1.0)), -np.inf)
    ref_out = np.where(live[..., None], (wts[..., None] * po).sum(axis=0) / np.where(live, L, 1.0)[..., None], 0.0)
    got = out.float().cpu().double().numpy()
    # one rounding to bf16 (half a bf16 step) plus fp32 arithmetic over W parts
    assert np.all(np.abs(got - ref_out) <= 0.5 * _bf16_ulp(ref_out) + 4e-6 * world * (np.abs(ref_out) + 1e-3))
    got_lse = lse.cpu().double().numpy()
    assert np.array_equal(np.isneginf(got_lse), ~live)
    assert np.all(np.abs(np.where(live, got_lse - ref_lse, 0.0)) <= 2e-6 * world * (1 + np.abs(ref_lse)))
    if world == 1:
        # one part: the merge returns that part's result rounded once
        assert np.array_equal(out.cpu().view(torch.int16), parts_out[0].to(torch.bfloat16).cpu().view(torch.int16))


def test_fp32_step_output_matches_the_bf16_step(da_lib, oracle_lib):
    """A step with fp32 output: every request (one segment, several, none) is written by the combine,
    and rounding it to bf16 gives the ordinary step's out within one bf16 step."""
    w = W.make_workload("f32", [0, 1, 700, 3000, 20000, 129], num_q_heads=16, num_kv_heads=2, head_dim=128,
                        page_size=64, seed=13)
    dw = w.to("cuda")
    prob = da.problem_from(dw.problem)
    res = {}
    for f32 in (False, True):
        desc = da.da_plan_desc_init(prob, da.PLAN_DYNAMIC, 64, 11, out_f32=f32)
        bufs = da.Buffers(prob, desc, "cuda")
        bufs.out.fill_(float("nan"))
        bufs.lse.fill_(float("nan"))
        da.decode_step(prob, desc, dw.q, dw.k_cache, dw.v_cache, dw.block_table, dw.seq_lens, bufs)
        torch.cuda.synchronize()
        res[f32] = (bufs.out.clone(), bufs.lse.clone())
    o32 = res[True][0]
    assert o32.dtype == torch.float32 and torch.isfinite(o32).all()
    check_against_oracle(w, o32.to(torch.bfloat16), res[True][1])
    o16 = res[False][0].float().cpu().double().numpy()
    d = np.abs(o32.cpu().double().numpy() - o16)
    assert np.all(d <= _bf16_ulp(o16))
    assert torch.equal(torch.isneginf(res[True][1]), torch.isneginf(res[False][1]))
    with pytest.raises(da.DaError):  # the in-decode merge writes bf16 only
        bad = da.da_plan_desc_init(prob, da.PLAN_DYNAMIC, 64, 11, merge_in_decode=True, out_f32=True)
        da.da_workspace_size(prob, bad)


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
        desc = da.da_plan_desc_init(prob, da.PLAN_DYNAMIC, 64, 0, out_f32=True)
        bufs = da.Buffers(prob, desc, "cuda")
        out = torch.empty(bufs.out.shape, dtype=torch.bfloat16, device="cuda")
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
