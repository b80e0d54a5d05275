"""Balance tables: a dynamic plan weighted per CTA, and the decode grid's blocks placed on the
plan's CTAs by a table.

The plan with weights must equal the oracle's weighted plan bit for bit; the table changes who
computes which tiles, never the result, so every step with a table (random or measured) must
still match the fp64 oracle.  A table that does not fit its descriptor is refused on the device
(DA_DEV_BAD_BALANCE) and the step runs with the even split.
"""

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import assert_plan_equal, check_against_oracle, check_against_oracle_fp8
from variable_length_paged_b200 import da
from variable_length_paged_b200 import workloads as W

pytestmark = pytest.mark.gpu


def random_table(desc, rng, spread=65536):
    C, H = desc.num_ctas, desc.num_kv_heads
    w = rng.integers(1, spread + 1, size=C).astype(np.int32)
    p = np.stack([rng.permutation(C) for _ in range(H)]).astype(np.int32)
    return w, p


def install(desc, w, p):
    table = torch.zeros(da.da_balance_words(desc), dtype=torch.int32, device="cuda")
    da.da_balance_set(desc, w, p, table)
    torch.cuda.synchronize()
    desc.balance = table.data_ptr()
    return table


@pytest.mark.parametrize("C", [1, 7, 37, 148, 1000])
@pytest.mark.parametrize("start_cost", [0, 2])
def test_weighted_plan_matches_oracle(da_lib, oracle_lib, C, start_cost):
    rng = np.random.default_rng(C * 10 + start_cost)
    for lens in ([1, 7, 64, 300], [131072, 1000], list(rng.integers(0, 20000, size=200)), [3, 0, 5]):
        lens = np.asarray(lens, np.int32)
        B = len(lens)
        prob = da.problem(B, 8, 2, 128, 64, 2048, 16, 0.1)
        desc = da.da_plan_desc_init(prob, da.PLAN_DYNAMIC, 64, C, start_cost=start_cost)
        w, p = random_table(desc, rng, spread=int(rng.choice([3, 65536])))
        table = install(desc, w, p)
        ws = torch.full((da.da_workspace_size(prob, desc)[0] // 4,), -7, dtype=torch.int32, device="cuda")
        da.da_plan(prob, desc, torch.from_numpy(lens).cuda(), ws)
        torch.cuda.synchronize()
        got = da.read_plan(desc, ws)
        ref = oracle.plan(lens, 64, C, 2048 * 64, start_cost=start_cost, weights=w)
        assert_plan_equal(got, ref)
        assert got["balance"] == 1 and got["status"] == da.DEV_OK
        del table


def test_equal_weights_give_the_even_plan(da_lib, oracle_lib):
    lens = np.random.default_rng(3).integers(0, 9000, size=64).astype(np.int32)
    prob = da.problem(64, 8, 8, 128, 64, 2048, 16, 0.1)
    desc = da.da_plan_desc_init(prob, da.PLAN_DYNAMIC, 64, 37)
    table = install(desc, np.full(37, 4096, np.int32), np.tile(np.arange(37, dtype=np.int32), (8, 1)))
    ws = torch.zeros(da.da_workspace_size(prob, desc)[0] // 4, dtype=torch.int32, device="cuda")
    da.da_plan(prob, desc, torch.from_numpy(lens).cuda(), ws)
    torch.cuda.synchronize()
    assert_plan_equal(da.read_plan(desc, ws), oracle.plan(lens, 64, 37, 2048 * 64, start_cost=2))
    del table


def small(lens, Hq=16, Hkv=2, seed=0):
    return W.make_workload("small", lens, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=128, page_size=64, seed=seed)


def step_with_table(w, desc_kw, table_seed, fp8=False, **step_kw):
    dw = w.to("cuda")
    prob = da.problem_from(dw.problem)
    desc = da.da_plan_desc_init(prob, da.PLAN_DYNAMIC, **desc_kw)
    table = install(desc, *random_table(desc, np.random.default_rng(table_seed)))
    bufs = da.Buffers(prob, desc, "cuda")
    for t in (bufs.partial_o, bufs.partial_lse, bufs.out, bufs.lse):
        t.fill_(float("nan"))
    kw = dict(k_scale=dw.k_scale, v_scale=dw.v_scale) if fp8 else {}
    da.decode_step(prob, desc, dw.q, dw.k_cache, dw.v_cache, dw.block_table, dw.seq_lens, bufs, **kw, **step_kw)
    torch.cuda.synchronize()
    assert da.read_plan(desc, bufs.ws)["balance"] == 1
    assert da.da_read_status(bufs.ws) == (0, -1)
    del table
    return bufs


@pytest.mark.parametrize("C", [7, 37, 148])
def test_decode_with_random_table(da_lib, oracle_lib, C):
    w = small([3000, 70, 1, 512, 2049, 0, 33, 9000], seed=C)
    bufs = step_with_table(w, dict(tile_tokens=64, width=C), C)
    check_against_oracle(w, bufs.out, bufs.lse)


def test_decode_with_random_table_separate_calls_and_merge(da_lib, oracle_lib):
    w = small([3000, 70, 1, 512, 2049, 0, 33, 9000], seed=5)
    bufs = step_with_table(w, dict(tile_tokens=64, width=37), 5, separate=True)
    check_against_oracle(w, bufs.out, bufs.lse)
    dw = w.to("cuda")
    prob = da.problem_from(dw.problem)
    desc = da.da_plan_desc_init(prob, da.PLAN_DYNAMIC, 64, 37, merge_in_decode=True)
    table = install(desc, *random_table(desc, np.random.default_rng(6)))
    b2 = da.Buffers(prob, desc, "cuda")
    da.decode_step(prob, desc, dw.q, dw.k_cache, dw.v_cache, dw.block_table, dw.seq_lens, b2)
    torch.cuda.synchronize()
    check_against_oracle(w, b2.out, b2.lse)
    del table


def test_fp8_decode_with_random_table(da_lib, oracle_lib):
    w8 = W.quantize_fp8(small([3000, 70, 1, 512, 2049, 0, 33, 9000], seed=8))
    bufs = step_with_table(w8, dict(tile_tokens=64, width=37), 8, fp8=True)
    check_against_oracle_fp8(w8, bufs.out, bufs.lse)


def test_refused_table_runs_even(da_lib, oracle_lib):
    """A buffer that is not a table for this descriptor: the plan is the even one, the status says
    so, and the step is still right."""
    w = small([3000, 70, 1, 512, 2049, 0, 33, 9000], seed=9)
    dw = w.to("cuda")
    prob = da.problem_from(dw.problem)
    desc = da.da_plan_desc_init(prob, da.PLAN_DYNAMIC, 64, 37)
    other = da.da_plan_desc_init(prob, da.PLAN_DYNAMIC, 64, 36)  # a table for another C
    table = torch.zeros(max(da.da_balance_words(desc), da.da_balance_words(other)), dtype=torch.int32, device="cuda")
    da.da_balance_set(other, *random_table(other, np.random.default_rng(1)), table)
    desc.balance = table.data_ptr()
    bufs = da.Buffers(prob, desc, "cuda")
    da.decode_step(prob, desc, dw.q, dw.k_cache, dw.v_cache, dw.block_table, dw.seq_lens, bufs)
    torch.cuda.synchronize()
    got = da.read_plan(desc, bufs.ws)
    assert got["balance"] == 0
    assert da.da_read_status(bufs.ws)[0] == da.DEV_BAD_BALANCE
    assert_plan_equal(got, oracle.plan(dw.seq_lens.cpu().numpy(), 64, 37, prob.max_pages_per_req * 64, start_cost=2))
    check_against_oracle(w, bufs.out, bufs.lse)


@pytest.mark.parametrize("fp8", [False, True])
def test_block_times_and_calibration(da_lib, oracle_lib, fp8):
    """Every block of the decode grid writes its start and end; a table measured from them
    (two rounds) is valid, the plan takes it, and the full-size mixed step stays right."""
    w = W.mixed()
    w = W.quantize_fp8(w) if fp8 else w
    dw = w.to("cuda")
    prob = da.problem_from(dw.problem)
    desc = da.da_plan_desc_init(prob, da.PLAN_DYNAMIC, 64, 0)
    bufs = da.Buffers(prob, desc, "cuda")
    kw = dict(k_scale=dw.k_scale, v_scale=dw.v_scale) if fp8 else {}

    def run(d):
        da.decode_step(prob, d, dw.q, dw.k_cache, dw.v_cache, dw.block_table, dw.seq_lens, bufs, **kw)

    times = torch.zeros((prob.num_kv_heads, desc.num_ctas, 2), dtype=torch.int64, device="cuda")
    desc.block_times = times.data_ptr()
    run(desc)
    torch.cuda.synchronize()
    desc.block_times = None
    t = times.cpu().numpy()
    assert np.all(t[:, :, 0] > 0) and np.all(t[:, :, 1] >= t[:, :, 0])
    assert (t[:, :, 1] - t[:, :, 0]).max() < 10_000_000  # ns: well under the 2 s wait limit

    table = da.calibrate_balance(desc, run, "cuda", rounds=2, steps=5)
    words = table.cpu().numpy()
    C, H = desc.num_ctas, desc.num_kv_heads
    weights, perm = words[4:4 + C], words[4 + C:].reshape(H, C)
    assert np.all((weights >= 1) & (weights <= 65536))
    assert all(sorted(row) == list(range(C)) for row in perm)
    for t_ in (bufs.out, bufs.lse):
        t_.fill_(float("nan"))
    run(desc)
    torch.cuda.synchronize()
    assert da.read_plan(desc, bufs.ws)["balance"] == 1
    pairs = (np.repeat(np.arange(prob.batch), 4), np.tile([0, 21, 42, 63], prob.batch))
    if fp8:
        check_against_oracle_fp8(w, bufs.out, bufs.lse, pairs=pairs)
    else:
        check_against_oracle(w, bufs.out, bufs.lse, pairs=pairs)
    ref = oracle.plan(dw.seq_lens.cpu().numpy(), 64, C, prob.max_pages_per_req * 64, start_cost=2, weights=weights)
    assert_plan_equal(da.read_plan(desc, bufs.ws), ref)
