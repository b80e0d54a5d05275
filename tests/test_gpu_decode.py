"""Decode attention on the GPU against the fp64 oracle, element by element.

Tolerance (both sides see the same bf16 inputs): |out - ref| <= 1e-2 + 1e-2*|ref|
on the bf16 output and |lse - ref| <= 1e-3 on the fp32 log-sum-exp.
"""

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import check_against_oracle, run_step
from variable_length_paged_b200 import da
from variable_length_paged_b200 import workloads as W

pytestmark = pytest.mark.gpu


def small(lens, Hq=8, Hkv=1, d=128, P=64, seed=0, **kw):
    return W.make_workload("small", lens, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=d, page_size=P, seed=seed, **kw)


def test_tiny_config(da_lib, oracle_lib):
    w = W.tiny()
    out, lse, desc, bufs, _ = run_step(w)
    check_against_oracle(w, out, lse)
    assert da.da_read_status(bufs.ws) == (0, -1)


def test_several_tiles_and_ragged_tail(da_lib, oracle_lib):
    w = small([1, 15, 16, 17, 63, 64, 65, 127, 128, 129, 1000, 4097], Hq=16, Hkv=2, seed=1)
    for C in (1, 3, 7, 37, 148):
        out, lse, *_ = run_step(w, width=C)
        check_against_oracle(w, out, lse)


@pytest.mark.parametrize("T", [16, 32, 48, 64, 128, 256])
@pytest.mark.parametrize("C", [1, 7, 37, 148, 1000])
def test_tile_and_cta_count_do_not_change_the_result(da_lib, oracle_lib, T, C):
    w = small([3000, 70, 1, 512, 2049, 0, 33], Hq=16, Hkv=2, seed=2)
    out, lse, *_ = run_step(w, tile=T, width=C)
    check_against_oracle(w, out, lse)


@pytest.mark.parametrize("kind,width", [(da.PLAN_DYNAMIC, 1), (da.PLAN_DYNAMIC, 37), (da.PLAN_DYNAMIC, 1000),
                                        (da.PLAN_STATIC, 1), (da.PLAN_STATIC, 7)])
def test_merge_in_decode(da_lib, oracle_lib, kind, width):
    """merge_in_decode = 1: the decode kernel's last CTA per split request merges it, and
    requests without segments are written by the decode kernel too (no combine launch)."""
    w = small([3000, 70, 1, 512, 2049, 0, 33], Hq=16, Hkv=2, seed=13)
    out, lse, desc, *_ = run_step(w, kind=kind, width=width, merge_in_decode=True)
    assert desc.merge_in_decode == 1
    check_against_oracle(w, out, lse)


@pytest.mark.parametrize("name", ["mixed", "low_conc"])
def test_merge_in_decode_full_size(da_lib, oracle_lib, name):
    w = W.CONFIGS[name]()
    out, lse, desc, *_ = run_step(w, merge_in_decode=True)
    check_against_oracle(w, out, lse)


def test_merge_in_decode_counts_reset_every_step(da_lib, oracle_lib):
    """The per-request segment counters live in the workspace and are reset by each plan."""
    w = small([3000, 70, 1, 512, 2049, 0, 33], Hq=16, Hkv=2, seed=14)
    out, lse, desc, bufs, dw = run_step(w, width=37, merge_in_decode=True)
    for _ in range(3):
        out, lse, *_ = run_step(None, dw=dw, bufs=bufs, width=37, merge_in_decode=True)
        check_against_oracle(w, out, lse)


@pytest.mark.parametrize("S", [1, 2, 4, 7, 16, 64])
def test_static_split_k(da_lib, oracle_lib, S):
    w = small([3000, 70, 1, 512, 2049, 0, 33], Hq=16, Hkv=2, seed=3)
    out, lse, desc, *_ = run_step(w, kind=da.PLAN_STATIC, width=S)
    assert desc.num_ctas == 7 * S
    check_against_oracle(w, out, lse)


@pytest.mark.parametrize("P", [16, 32, 64, 128])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_page_size_head_dim_group(da_lib, oracle_lib, P, d, G):
    w = small([1, 200, 37, 1500], Hq=2 * G, Hkv=2, d=d, P=P, seed=P + d + G)
    out, lse, *_ = run_step(w, width=11)
    check_against_oracle(w, out, lse)


def test_empty_and_full_capacity(da_lib, oracle_lib):
    w = small([0, 0, 640, 1], Hq=8, Hkv=1, seed=4, max_pages_per_req=10)
    out, lse, *_ = run_step(w, width=5)
    check_against_oracle(w, out, lse)
    assert not out[0].float().abs().sum() and torch.isneginf(lse[:2]).all()
    # the whole batch empty
    w0 = small([0, 0], Hq=8, Hkv=1, seed=5)
    out, lse, *_ = run_step(w0)
    assert not out.float().abs().sum() and torch.isneginf(lse).all()


def test_bad_lengths_are_reported_and_skipped(da_lib, oracle_lib):
    w = small([300, 50, 700], Hq=8, Hkv=1, seed=6, max_pages_per_req=12)
    dw = w.to("cuda")
    dw.seq_lens[1] = 12 * 64 + 1  # beyond capacity
    out, lse, desc, bufs, _ = run_step(None, dw=dw)
    assert da.da_read_status(bufs.ws) == (da.DEV_BAD_SEQLEN, 1)
    sl = w.seq_lens.copy()
    sl[1] = 0
    pairs = (np.array([0, 0, 2, 2], np.int32), np.array([0, 7, 3, 5], np.int32))
    check_against_oracle(w, out, lse, pairs=pairs, seq_lens=sl)
    assert torch.isneginf(lse[1]).all() and not out[1].float().abs().sum()


def test_bad_page_id_is_reported_without_fault(da_lib, oracle_lib):
    w = small([300, 500], Hq=8, Hkv=1, seed=7)
    dw = w.to("cuda")
    dw.block_table[1, 2] = w.problem.num_pages + 5
    out, lse, desc, bufs, _ = run_step(None, dw=dw)
    st, bad = da.da_read_status(bufs.ws)
    assert st == da.DEV_BAD_PAGE and bad == 1
    check_against_oracle(w, out, lse, pairs=(np.zeros(8, np.int32), np.arange(8, dtype=np.int32)))


def test_shared_prefix_pages(da_lib, oracle_lib):
    w = small([900, 900, 300], Hq=8, Hkv=1, seed=8)
    bt = w.block_table.copy()
    bt[1, :10] = bt[0, :10]  # request 1 shares the first 640 tokens of request 0
    w.block_table = bt
    out, lse, *_ = run_step(w, width=7)
    check_against_oracle(w, out, lse)


def test_deterministic(da_lib):
    w = small([5000, 300, 17], Hq=16, Hkv=2, seed=9)
    a = run_step(w, width=37)
    b = run_step(None, dw=a[4], width=37)
    assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16))
    assert torch.equal(a[1], b[1])


def test_lengths_change_between_steps_inside_one_graph(da_lib, oracle_lib):
    """The plan is rebuilt on the device: one captured graph serves every step while
    requests grow, finish and are cancelled (seq_lens edited in device memory only)."""
    lens0 = np.array([2000, 10, 3000, 640], np.int32)
    # every request owns pages for 3800 tokens, so its length can move anywhere below that
    w = small([3800, 3800, 3800, 3800], Hq=16, Hkv=2, seed=10, max_pages_per_req=60)
    dw = w.to("cuda")
    prob = da.problem_from(dw.problem)
    desc = da.da_plan_desc_init(prob, da.PLAN_DYNAMIC, 64, 37)
    bufs = da.Buffers(prob, desc, "cuda")
    dw.seq_lens.copy_(torch.from_numpy(lens0))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        da.decode_step(prob, desc, dw.q, dw.k_cache, dw.v_cache, dw.block_table, dw.seq_lens, bufs)  # warm up
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        da.decode_step(prob, desc, dw.q, dw.k_cache, dw.v_cache, dw.block_table, dw.seq_lens, bufs)
    schedule = [[2000, 10, 3000, 640], [2001, 11, 3001, 641], [2002, 0, 3002, 642], [2003, 0, 1, 3800],
                [0, 0, 0, 0], [17, 3700, 64, 65]]
    for lens in schedule:
        dw.seq_lens.copy_(torch.tensor(lens, dtype=torch.int32))
        g.replay()
        torch.cuda.synchronize()
        check_against_oracle(w, bufs.out, bufs.lse, seq_lens=np.array(lens, np.int32))


@pytest.mark.parametrize("name", ["mixed", "skewed", "low_conc", "uniform"])
def test_full_size_configs(da_lib, oracle_lib, name):
    w = W.CONFIGS[name]()
    out, lse, desc, bufs, _ = run_step(w)
    assert da.da_read_status(bufs.ws) == (0, -1)
    check_against_oracle(w, out, lse)  # every (request, head) of the full-size batch
    # the static comparator on the same inputs
    out_s, lse_s, *_ = run_step(w, kind=da.PLAN_STATIC)
    check_against_oracle(w, out_s, lse_s)


def test_batch_past_the_planner_shared_memory_copy(da_lib, oracle_lib):
    """5000 short requests (empty ones included): the planner's global-memory path, a combine
    grid of 5000 x Hq blocks, and the decode kernel walking thousands of one-tile segments."""
    rng = np.random.default_rng(77)
    lens = rng.integers(0, 400, size=5000)
    lens[rng.random(5000) < 0.1] = 0
    w = W.make_workload("many", lens, num_q_heads=8, num_kv_heads=2, head_dim=64, page_size=32, seed=77)
    out, lse, desc, bufs, _ = run_step(w)
    assert da.da_read_status(bufs.ws) == (0, -1)
    check_against_oracle(w, out, lse)


def test_two_million_token_request(da_lib, oracle_lib):
    """One 2^21-token request next to short ones (32768 pages of the first request, 1 GB of
    K/V): long segments on every CTA; sampled heads against the oracle."""
    lens = [2 ** 21, 1, 777]
    w = W.make_workload("long", lens, num_q_heads=8, num_kv_heads=1, head_dim=128, page_size=64, seed=41,
                        spare_frac=0.0)
    out, lse, desc, bufs, _ = run_step(w)
    assert da.da_read_status(bufs.ws) == (0, -1)
    pairs = (np.array([0, 0, 0, 1, 2], np.int32), np.array([0, 3, 7, 5, 2], np.int32))
    check_against_oracle(w, out, lse, pairs=pairs)
