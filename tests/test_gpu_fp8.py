"""Decode attention over an FP8 (E4M3, per-KV-head scale) cache against the fp64 oracle.

Both sides read the same codes and scales; the tolerance is the one of the bf16
path (|out - ref| <= 1e-2 + 1e-2*|ref|, |lse - ref| <= 1e-3).
"""

import numpy as np
import pytest
import torch

from gpu_helpers import check_against_oracle_fp8, run_step_fp8
from variable_length_paged_b200 import da
from variable_length_paged_b200 import workloads as W

pytestmark = pytest.mark.gpu


def small8(lens, Hq=16, Hkv=2, P=64, seed=0, **kw):
    return W.quantize_fp8(W.make_workload("small", lens, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=128,
                                          page_size=P, seed=seed, **kw))


def test_fp8_tiles_ctas_and_tails(da_lib, oracle_lib):
    w8 = small8([1, 15, 16, 17, 63, 64, 65, 127, 1000, 4097, 0], seed=1)
    for T, C in [(64, 37), (16, 7), (128, 1), (32, 148), (48, 1000)]:
        out, lse, *_ = run_step_fp8(w8, tile=T, width=C)
        check_against_oracle_fp8(w8, out, lse)


@pytest.mark.parametrize("P", [16, 32, 64, 128])
@pytest.mark.parametrize("G", [1, 4, 8])
def test_fp8_page_size_and_group(da_lib, oracle_lib, P, G):
    w8 = small8([1, 200, 37, 1500], Hq=2 * G, Hkv=2, P=P, seed=P + G)
    out, lse, *_ = run_step_fp8(w8, width=11)
    check_against_oracle_fp8(w8, out, lse)


@pytest.mark.parametrize("S", [1, 3, 16])
def test_fp8_static_split_k(da_lib, oracle_lib, S):
    w8 = small8([3000, 70, 1, 512, 2049, 0, 33], seed=3)
    out, lse, *_ = run_step_fp8(w8, kind=da.PLAN_STATIC, width=S)
    check_against_oracle_fp8(w8, out, lse)


def test_fp8_head_dim_64_is_refused(da_lib):
    prob = da.problem(2, 8, 1, 64, 64, 4, 8, 0.125)
    desc = da.da_plan_desc_init(prob, da.PLAN_DYNAMIC, 64, 4)
    with pytest.raises(da.DaError) as e:
        da.da_decode_attention_fp8(prob, desc, *([1 << 12] * 12))
    assert e.value.code == da.ERR_UNSUPPORTED


@pytest.mark.parametrize("name", ["mixed", "skewed", "low_conc", "uniform"])
def test_fp8_full_size(da_lib, oracle_lib, name):
    w8 = W.quantize_fp8(W.CONFIGS[name]())
    out, lse, desc, bufs, _ = run_step_fp8(w8)
    assert da.da_read_status(bufs.ws) == (0, -1)
    check_against_oracle_fp8(w8, out, lse)


def _set_key(w, b, t, g, row):
    """Write K row `row` (float tensor [d]) for token t of request b, KV head g."""
    P = w.problem.page_size
    page = int(w.block_table[b, t // P])
    w.k_cache[page, g, t % P] = row.to(torch.bfloat16)


def test_fp8_query_magnitudes(da_lib, oracle_lib):
    """Query rows from 1e-4 to 30 in size, and a row whose entries span three decades."""
    w = W.make_workload("small", [700, 33, 2048, 1, 5000], num_q_heads=16, num_kv_heads=2, head_dim=128,
                        page_size=64, seed=21)
    f = torch.tensor([1e-4, 1e-2, 0.3, 1.0, 3.0, 10.0, 30.0, 0.05] * 2, dtype=torch.float32)
    q = w.q.float() * f[None, :, None]
    q[:, 3, :64] *= 1e-3
    w.q = q.to(torch.bfloat16)
    w8 = W.quantize_fp8(w)
    out, lse, *_ = run_step_fp8(w8, width=7)
    check_against_oracle_fp8(w8, out, lse)


@pytest.mark.parametrize("spike", [12.0, 20.0])
def test_fp8_spike_over_a_flat_tail(da_lib, oracle_lib, spike):
    """One key far above thousands of equal ones: the tail's total weight (about 20000 e^-12
    against 1 at spike 12) must survive the rounding of the small weights."""
    L = [20000, 5000, 3000]
    w = W.make_workload("small", L, num_q_heads=16, num_kv_heads=2, head_dim=128, page_size=64, seed=22)
    d = w.problem.head_dim
    w.k_cache.zero_()  # every key 0 (score 0), then one spike per (request, KV head)
    e1 = torch.zeros(d)
    e1[5] = 1.0
    a = spike * float(np.sqrt(d))  # score of the spike for a query e1: a * 1/sqrt(d) = spike
    for b, t0 in [(0, 7777), (1, 100), (2, 2999)]:
        for g in range(2):
            _set_key(w, b, t0, g, a * e1)
    s = torch.tensor([1.0, 0.5, -1.0, 0.9, 1.0, 0.25, 0.75, 1.0] * 2)  # per-head spike strength
    w.q = (s[None, :, None] * e1[None, None, :]).expand(3, 16, d).contiguous().to(torch.bfloat16)
    w8 = W.quantize_fp8(w)
    for T, C in [(64, 37), (64, 3), (128, 1)]:
        out, lse, *_ = run_step_fp8(w8, tile=T, width=C)
        check_against_oracle_fp8(w8, out, lse)


def test_fp8_zero_query_long_request(da_lib, oracle_lib):
    """q = 0: every weight equal over 30000 tokens; out is the mean of V, lse = ln L."""
    w = W.make_workload("small", [30000, 17], num_q_heads=8, num_kv_heads=1, head_dim=128, page_size=64, seed=23)
    w.q.zero_()
    w8 = W.quantize_fp8(w)
    out, lse, *_ = run_step_fp8(w8, width=5)
    check_against_oracle_fp8(w8, out, lse)
    assert np.allclose(lse.cpu().numpy(), np.log(np.array([30000, 17], np.float64))[:, None], atol=1e-4)


def test_fp8_shared_prefix_pages(da_lib, oracle_lib):
    """Two requests whose block tables name the same pages (a shared prefix) on the tensor-core path."""
    w = W.make_workload("small", [900, 900, 300], num_q_heads=8, num_kv_heads=1, head_dim=128, page_size=64,
                        seed=8)
    bt = w.block_table.copy()
    bt[1, :10] = bt[0, :10]  # request 1 shares the first 640 tokens of request 0
    w.block_table = bt
    w8 = W.quantize_fp8(w)
    out, lse, *_ = run_step_fp8(w8, width=7)
    check_against_oracle_fp8(w8, out, lse)


def test_fp8_lengths_change_inside_one_graph(da_lib, oracle_lib):
    """One captured FP8 step serves requests that grow, finish and restart (lengths edited in device
    memory only); every replay matches the oracle at its lengths."""
    import dataclasses
    w = W.make_workload("small", [3800, 3800, 3800, 3800], num_q_heads=16, num_kv_heads=2, head_dim=128,
                        page_size=64, seed=21, max_pages_per_req=60)
    w8 = W.quantize_fp8(w)
    dw = w8.to("cuda")
    prob = da.problem_from(dw.problem)
    desc = da.da_plan_desc_init(prob, da.PLAN_DYNAMIC, 64, 37)
    bufs = da.Buffers(prob, desc, "cuda")
    step = lambda: da.decode_step(prob, desc, dw.q, dw.k_cache, dw.v_cache, dw.block_table, dw.seq_lens, bufs,
                                  k_scale=dw.k_scale, v_scale=dw.v_scale)
    dw.seq_lens.copy_(torch.tensor([2000, 10, 3000, 640], dtype=torch.int32))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        step()  # warm up
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step()
    for lens in [[2000, 10, 3000, 640], [2001, 0, 3001, 1], [0, 0, 0, 0], [17, 3800, 128, 129], [1, 2, 3, 3799]]:
        dw.seq_lens.copy_(torch.tensor(lens, dtype=torch.int32))
        g.replay()
        torch.cuda.synchronize()
        cur = dataclasses.replace(w8, base=dataclasses.replace(w, seq_lens=np.array(lens, np.int32)))
        check_against_oracle_fp8(cur, bufs.out, bufs.lse)
    assert da.da_read_status(bufs.ws) == (0, -1)
