"""The one-call step (da_decode_step) against the three separate calls.

da_decode_step enqueues da_plan (or da_static_plan), the decode and da_combine in one
call, with every check of the three made before the first launch.  Its results must
equal the separate calls' bit for bit, with the same plan in the workspace and the
same status word, on batches with CTAs that have no tile (fewer tiles than CTAs),
segments shorter than the stage ring, empty static splits, bad lengths and a large
batch, for both cache formats.
"""

import numpy as np
import pytest
import torch

from gpu_helpers import check_against_oracle
from variable_length_paged_b200 import da
from variable_length_paged_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _both(w, kind, tile, width, fp8=False):
    dw = (W.quantize_fp8(w) if fp8 else w).to("cuda")
    prob = da.problem_from(dw.problem)
    desc = da.da_plan_desc_init(prob, kind, tile, width)
    kw = dict(k_scale=dw.k_scale, v_scale=dw.v_scale) if fp8 else {}
    res = []
    for separate in (False, True):
        bufs = da.Buffers(prob, desc, "cuda")
        for t in (bufs.partial_o, bufs.partial_lse, bufs.out, bufs.lse):
            t.fill_(float("nan"))
        da.decode_step(prob, desc, dw.q, dw.k_cache, dw.v_cache, dw.block_table, dw.seq_lens, bufs,
                       separate=separate, **kw)
        torch.cuda.synchronize()
        res.append((bufs.out.clone(), bufs.lse.clone(), da.read_plan(desc, bufs.ws), da.da_read_status(bufs.ws)))
    (o1, l1, p1, s1), (o2, l2, p2, s2) = res
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1, l2)
    for key in ("seg_req", "seg_tile_begin", "seg_tile_end", "cta_seg_begin", "req_seg_begin"):
        assert np.array_equal(p1[key], p2[key]), key
    assert s1 == s2
    return o1, l1, s1


@pytest.mark.parametrize("kind,tile,width", [(da.PLAN_DYNAMIC, 64, 0), (da.PLAN_DYNAMIC, 16, 7),
                                             (da.PLAN_DYNAMIC, 64, 1000), (da.PLAN_DYNAMIC, 128, 148),
                                             (da.PLAN_STATIC, 64, 3), (da.PLAN_STATIC, 32, 16)])
@pytest.mark.parametrize("fp8", [False, True])
def test_one_call_step_equals_separate_calls(da_lib, oracle_lib, kind, tile, width, fp8):
    w = W.make_workload("one_call", [1, 0, 17, 64, 65, 200, 1000, 4097, 33, 20000, 0, 129], num_q_heads=16,
                        num_kv_heads=2, head_dim=128, page_size=64, seed=41)
    out, lse, st = _both(w, kind, tile, width, fp8)
    assert st == (da.DEV_OK, -1)
    if not fp8:
        check_against_oracle(w, out, lse)


def test_one_call_step_with_bad_lengths(da_lib, oracle_lib):
    w = W.make_workload("one_call_bad", [300, 5000, 70], num_q_heads=8, num_kv_heads=1, head_dim=128, page_size=64,
                        seed=42)
    w.seq_lens = w.seq_lens.copy()
    w.seq_lens[1] = -5  # a bad length: the request gets 0 tiles and is reported
    out, lse, st = _both(w, da.PLAN_DYNAMIC, 64, 5)
    assert st == (da.DEV_BAD_SEQLEN, 1)


def test_one_call_step_large_batch(da_lib, oracle_lib):
    lens = np.random.default_rng(43).integers(0, 200, 1100)
    w = W.make_workload("one_call_big", lens, num_q_heads=8, num_kv_heads=1, head_dim=64, page_size=16, seed=43)
    out, lse, st = _both(w, da.PLAN_DYNAMIC, 64, 0)
    assert st == (da.DEV_OK, -1)
    check_against_oracle(w, out, lse)
