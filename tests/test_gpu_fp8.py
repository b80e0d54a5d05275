"""Decode attention over an FP8 (E4M3, per-KV-head scale) cache against the fp64 oracle.

Both sides read the same codes and scales; the tolerance is the one of the bf16
path (|out - ref| <= 1e-2 + 1e-2*|ref|, |lse - ref| <= 1e-3).
"""

import numpy as np
import pytest

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


@pytest.mark.parametrize("name", ["mixed", "skewed"])
def test_fp8_full_size(da_lib, oracle_lib, name):
    w8 = W.quantize_fp8(W.CONFIGS[name]())
    out, lse, desc, bufs, _ = run_step_fp8(w8)
    assert da.da_read_status(bufs.ws) == (0, -1)
    check_against_oracle_fp8(w8, out, lse)
