"""Multi-query decode (q_len new tokens per request, causal within the cache) and 16-row groups.

The G query heads x q_len queries of a request share the 16 MMA rows, so each
K/V tile is read once for all queries.  Checked against the fp64 oracle with
the tolerance of the other parity tests.
"""

import numpy as np
import pytest

from gpu_helpers import (check_against_oracle, check_mq_against_oracle, check_mq_fp8_against_oracle, run_step,
                         run_step_fp8)
from variable_length_paged_b200 import da
from variable_length_paged_b200 import workloads as W

pytestmark = pytest.mark.gpu


def mq(lens, G, Q, Hkv=2, d=128, P=64, seed=0, **kw):
    return W.make_workload("mq", lens, num_q_heads=G * Hkv, num_kv_heads=Hkv, head_dim=d, page_size=P, seed=seed,
                           q_len=Q, **kw)


@pytest.mark.parametrize("G,Q", [(8, 2), (4, 4), (2, 8), (1, 16), (1, 3), (4, 2), (2, 5), (16, 1)])
def test_mq_rows(da_lib, oracle_lib, G, Q):
    w = mq([1, 2, 15, 16, 17, 64, 65, 300, 2049], G, Q, seed=G * 31 + Q)
    out, lse, *_ = run_step(w, width=7)
    if Q == 1:
        check_against_oracle(w, out, lse)
    else:
        check_mq_against_oracle(w, out, lse)


@pytest.mark.parametrize("T,C", [(16, 1), (64, 37), (128, 148), (48, 1000)])
def test_mq_tiles_and_ctas(da_lib, oracle_lib, T, C):
    w = mq([3000, 70, 1, 512, 2049, 0, 33], 8, 2, seed=3)
    out, lse, *_ = run_step(w, tile=T, width=C)
    check_mq_against_oracle(w, out, lse)


@pytest.mark.parametrize("d,P", [(64, 16), (64, 64), (128, 32)])
def test_mq_head_dim_and_pages(da_lib, oracle_lib, d, P):
    w = mq([1, 200, 37, 1500], 4, 3, d=d, P=P, seed=d + P)
    out, lse, *_ = run_step(w, width=11)
    check_mq_against_oracle(w, out, lse)


def test_mq_static_split_k(da_lib, oracle_lib):
    w = mq([3000, 70, 1, 512, 2049, 0, 33], 8, 2, seed=4)
    out, lse, *_ = run_step(w, kind=da.PLAN_STATIC, width=5)
    check_mq_against_oracle(w, out, lse)


@pytest.mark.parametrize("G,Q", [(8, 2), (2, 6)])
def test_mq_fp8(da_lib, oracle_lib, G, Q):
    w8 = W.quantize_fp8(mq([1, 3, 17, 64, 65, 300, 2049, 4000], G, Q, seed=5))
    out, lse, *_ = run_step_fp8(w8, width=13)
    check_mq_fp8_against_oracle(w8, out, lse)


def test_mq_full_size_mixed(da_lib, oracle_lib):
    w = W.mixed(q_len=2)
    out, lse, desc, bufs, _ = run_step(w)
    assert da.da_read_status(bufs.ws) == (0, -1)
    check_mq_against_oracle(w, out, lse)
