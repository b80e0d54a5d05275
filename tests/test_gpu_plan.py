"""The on-device planners against the oracle's plans: bit-exact work lists."""

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import assert_plan_equal
from variable_length_paged_b200 import da

pytestmark = pytest.mark.gpu


def plan_on_device(lens, T, width, kind, cap_pages=2048, P=64, start_cost=None):
    lens = np.asarray(lens, np.int32)
    B = len(lens)
    prob = da.problem(B, 8, 1, 128, P, cap_pages, 16, 0.1)
    desc = da.da_plan_desc_init(prob, kind, T, width, start_cost=start_cost)
    ws_bytes, _, _ = da.da_workspace_size(prob, desc)
    ws = torch.full((ws_bytes // 4,), -7, dtype=torch.int32, device="cuda")
    sl = torch.from_numpy(lens).cuda()
    if kind == da.PLAN_DYNAMIC:
        da.da_plan(prob, desc, sl, ws)
    else:
        da.da_static_plan(prob, desc, sl, ws)
    torch.cuda.synchronize()
    return da.read_plan(desc, ws), cap_pages * P


DEFAULT_START_COST = 2  # da_plan_desc_init's start cost of a dynamic plan

CASES = [
    [],
    [0],
    [0, 0, 0],
    [1],
    [1, 7, 64, 300],
    [131072, 1000],
    [4096] * 64,
    [5, 0, 2],
]


def random_lens(seed):
    rng = np.random.default_rng(seed)
    B = int(rng.choice([1, 3, 32, 128, 256, 1500, 3000]))
    lens = rng.integers(0, 20000, size=B)
    lens[rng.random(B) < 0.15] = 0
    short = rng.random(B) < 0.1
    lens[short] = rng.integers(1, 70, size=int(short.sum()))
    return lens


@pytest.mark.parametrize("T", [16, 64, 256])
@pytest.mark.parametrize("C", [1, 7, 37, 148, 1000])
def test_dynamic_plan_fixed_cases(da_lib, oracle_lib, T, C):
    for lens in CASES:
        if not lens:
            continue
        got, cap = plan_on_device(lens, T, C, da.PLAN_DYNAMIC)
        assert_plan_equal(got, oracle.plan(lens, T, C, cap, start_cost=DEFAULT_START_COST))
        assert got["status"] == 0


@pytest.mark.parametrize("seed", range(12))
def test_dynamic_plan_random(da_lib, oracle_lib, seed):
    rng = np.random.default_rng(100 + seed)
    lens = random_lens(seed)
    T = int(rng.choice([16, 32, 64, 128]))
    C = int(rng.choice([1, 5, 37, 74, 296, 999]))
    got, cap = plan_on_device(lens, T, C, da.PLAN_DYNAMIC)
    assert_plan_equal(got, oracle.plan(lens, T, C, cap, start_cost=DEFAULT_START_COST))


def test_dynamic_plan_bad_lengths(da_lib, oracle_lib):
    lens = [100, -5, 7000, 2048 * 64 + 1, 3, -1]
    got, cap = plan_on_device(lens, 64, 37, da.PLAN_DYNAMIC)
    ref = oracle.plan(lens, 64, 37, cap, start_cost=DEFAULT_START_COST)
    assert ref["bad_index"] == 1
    assert_plan_equal(got, ref)
    assert got["status"] == da.DEV_BAD_SEQLEN


@pytest.mark.parametrize("S", [1, 2, 3, 8, 64])
def test_static_plan(da_lib, oracle_lib, S):
    for lens in CASES[1:] + [list(random_lens(7)), list(random_lens(8))]:
        got, cap = plan_on_device(lens, 64, S, da.PLAN_STATIC)
        assert_plan_equal(got, oracle.static_plan(lens, 64, S, cap))
        assert got["splits"] == S and got["kind"] == da.PLAN_STATIC


@pytest.mark.parametrize("B,C", [(4097, 37), (6000, 296), (20000, 1000)])
def test_dynamic_plan_batches_past_the_shared_memory_copy(da_lib, oracle_lib, B, C):
    """Above 4096 requests the planner reads its prefix arrays back from global memory."""
    rng = np.random.default_rng(B)
    lens = rng.integers(0, 3000, size=B)
    lens[rng.random(B) < 0.2] = 0
    got, cap = plan_on_device(lens, 64, C, da.PLAN_DYNAMIC)
    assert_plan_equal(got, oracle.plan(lens, 64, C, cap, start_cost=DEFAULT_START_COST))
    assert got["status"] == 0


def test_static_plan_large_batch(da_lib, oracle_lib):
    rng = np.random.default_rng(5)
    lens = rng.integers(0, 2000, size=5000)
    got, cap = plan_on_device(lens, 64, 2, da.PLAN_STATIC)
    assert_plan_equal(got, oracle.static_plan(lens, 64, 2, cap))


def test_static_plan_launches_empty_splits(da_lib, oracle_lib):
    """The comparator's weakness the article names: with lengths that differ, a static split
    count sized by the longest request leaves the short requests' later splits empty (their
    CTAs are launched and find nothing), while the dynamic plan gives every CTA work."""
    lens = [100, 5000, 70, 16000]
    got, cap = plan_on_device(lens, 64, 8, da.PLAN_STATIC)
    empty = int(np.sum(np.asarray(got["seg_tile_end"]) == np.asarray(got["seg_tile_begin"])))
    # chunk = ceil(ceil(16000/64)/8) = 32 tiles: 100 -> 1 busy split, 5000 -> 3, 70 -> 1, 16000 -> 8
    assert empty == 8 * 4 - (1 + 3 + 1 + 8)
    dyn, _ = plan_on_device(lens, 64, 32, da.PLAN_DYNAMIC, start_cost=0)  # tiles only: loads within one tile
    loads = np.bincount(np.asarray(dyn["seg_cta"]),
                        weights=np.asarray(dyn["seg_tile_end"]) - np.asarray(dyn["seg_tile_begin"]), minlength=32)
    U = sum(-(-L // 64) for L in lens)
    assert loads.min() >= U // 32 and loads.max() <= -(-U // 32)


def test_dynamic_plan_wide_division_path(da_lib, oracle_lib):
    """C * (U + 1) >= 2^31: the planner's owner/first-tile formulas take their 64-bit form."""
    rng = np.random.default_rng(9)
    lens = rng.integers(2000, 6000, size=20000)
    T, C = 16, 1000
    U = int(sum(-(-int(L) // T) for L in lens))
    assert C * (U + 1) >= 2 ** 31
    got, cap = plan_on_device(lens, T, C, da.PLAN_DYNAMIC)
    assert_plan_equal(got, oracle.plan(lens, T, C, cap, start_cost=DEFAULT_START_COST))


@pytest.mark.parametrize("sc", [0, 1, 3, 7])
@pytest.mark.parametrize("C", [1, 7, 37, 296, 1000])
def test_dynamic_plan_start_cost(da_lib, oracle_lib, sc, C):
    """Start units: every fixed case (tiny ones make the plan sparse at large C) and a random
    batch, for several start costs, bit-exact against the oracle's plan."""
    for lens in CASES + [list(random_lens(31)), list(random_lens(32))]:
        if not lens:
            continue
        got, cap = plan_on_device(lens, 64, C, da.PLAN_DYNAMIC, start_cost=sc)
        assert_plan_equal(got, oracle.plan(lens, 64, C, cap, start_cost=sc))
