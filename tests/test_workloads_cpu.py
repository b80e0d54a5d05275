"""The seeded input generator against its recipe, on CPU: lengths, page layout, poison and the trace's
step dynamics are what the workloads are said to be (at reduced batch where the full caches would be
large)."""

import math

import numpy as np
import torch

from variable_length_paged_b200 import workloads as W


def check_layout(w: W.Workload, poisoned: bool = True):
    """Block table rows name distinct in-range pages, -1 past the request; live slots are finite and,
    for the named configs, every other slot is NaN (the trace refills whole pages with fresh values
    and keeps freed pages as they were, so there only the live slots are checked)."""
    p = w.problem
    B, P = p.batch, p.page_size
    assert w.block_table.shape == (B, p.max_pages_per_req) and w.block_table.dtype == np.int32
    assert w.k_cache.shape == (p.num_pages, p.num_kv_heads, P, p.head_dim) == w.v_cache.shape
    assert w.q.shape == (B, p.num_q_heads, p.head_dim) and w.q.dtype == torch.bfloat16
    live = np.zeros((p.num_pages, P), dtype=bool)
    seen = set()
    for b in range(B):
        L = int(w.seq_lens[b])
        n = -(-L // P)
        pages = w.block_table[b, :n]
        assert np.all((pages >= 0) & (pages < p.num_pages)) and np.all(w.block_table[b, n:] == -1)
        assert not (set(pages.tolist()) & seen), "pages shared between requests"
        seen |= set(pages.tolist())
        t = np.arange(L)
        live[pages[t // P], t % P] = True
    m = torch.from_numpy(live)
    for c in (w.k_cache, w.v_cache):
        rows = c.permute(0, 2, 1, 3)  # [page, slot, head, d]
        assert torch.isfinite(rows[m].float()).all(), "a live slot is not finite"
        if poisoned:
            assert torch.isnan(rows[~m].float()).all(), "an unused slot is not poisoned"


def test_tiny_recipe():
    w = W.tiny()
    assert w.seq_lens.tolist() == [1, 7, 64, 300]
    p = w.problem
    assert (p.num_q_heads, p.num_kv_heads, p.head_dim, p.page_size) == (4, 1, 64, 16) and p.scale == 0.125
    check_layout(w)
    assert np.any(np.diff(w.block_table[3, :19]) != 1), "page ids are shuffled"


def test_same_seed_same_workload():
    a, b = W.tiny(seed=9), W.tiny(seed=9)
    assert np.array_equal(a.block_table, b.block_table)
    assert torch.equal(a.q.view(torch.int16), b.q.view(torch.int16))
    assert torch.equal(a.k_cache.view(torch.int16), b.k_cache.view(torch.int16))
    c = W.tiny(seed=10)
    assert not torch.equal(a.q.view(torch.int16), c.q.view(torch.int16))


def test_mixed_lengths_and_layout():
    w = W.mixed(batch=6)
    assert np.all((w.seq_lens >= 1000) & (w.seq_lens <= 16000))
    p = w.problem
    assert (p.num_q_heads, p.num_kv_heads, p.head_dim, p.page_size) == (64, 8, 128, 64)
    assert p.scale == np.float32(1 / math.sqrt(128))
    check_layout(w)


def test_skewed_split_and_outliers():
    w = W.skewed(batch=20)
    lens = w.seq_lens
    long = lens >= 16384
    assert long.sum() == 2 and np.all(lens[long] <= 65536) and np.all((lens[~long] >= 256) & (lens[~long] <= 2048))
    check_layout(w)
    # about 1 % of the K rows are scaled by 8: their norm stands far above the N(0,1) rows' sqrt(d)
    P, d = w.problem.page_size, w.problem.head_dim
    norms = []
    for b in range(w.problem.batch):
        t = np.arange(int(lens[b]))
        pages = w.block_table[b, t // P]
        norms.append(w.k_cache[torch.from_numpy(pages.astype(np.int64)), 0, torch.from_numpy(t % P)].float().norm(dim=-1))
    n = torch.cat(norms)
    frac = float((n > 4 * math.sqrt(d)).float().mean())
    assert 0.007 < frac < 0.013, frac


def test_low_conc_lengths():
    w = W.low_conc()
    assert w.seq_lens.tolist() == [131072, 1000]
    assert w.problem.max_pages_per_req * w.problem.page_size >= 131072


def test_trace_steps_grow_finish_and_restart():
    tr = W.DecodeTrace(seed=3, batch=16, steps=20, num_q_heads=8, num_kv_heads=2, median=300.0, max_len=2000,
                       p_finish=0.2, new_len=(500, 2000), spare_pages=2000)
    lens0 = tr.seq_lens.copy()
    assert np.all((lens0 >= 1) & (lens0 <= 2000))
    check_layout(tr.workload(), poisoned=False)
    restarts = 0
    for _ in range(20):
        before = tr.seq_lens.copy()
        upd = tr.advance()
        after = tr.seq_lens
        r = np.zeros(16, dtype=bool)
        r[upd["restarted"]] = True
        restarts += int(r.sum())
        assert np.all(after[~r] == before[~r] + 1)  # every other slot grows by one token
        assert np.all((after[r] >= 501) & (after[r] <= 2001))  # restarted: U[500, 2000], then + 1
        assert upd["new_k"].shape == (16, 2, 128) and upd["q"].shape == (16, 8, 128)
        live = sum(-(-int(L) // 64) for L in after)
        assert live + len(tr.free) == tr.problem.num_pages  # no page lost or handed out twice
    assert restarts > 0
    check_layout(tr.workload(), poisoned=False)


def test_fp8_quantiser_recipe():
    """scale = max |x| / 448 per KV head; every live value comes back within half an E4M3 step of its
    exponent (3 mantissa bits: |x/scale - e4m3| <= 2^-4 |x/scale|, or an absolute 2^-10 in the
    subnormal range); the largest |x| of each head maps to the largest finite code 448."""
    w = W.make_workload("q8", [1, 17, 300, 64], num_q_heads=4, num_kv_heads=2, head_dim=128, page_size=16, seed=4)
    w8 = W.quantize_fp8(w)
    P = w.problem.page_size
    for cache, code, scale in ((w.k_cache, w8.k_code, w8.k_scale), (w.v_cache, w8.v_code, w8.v_scale)):
        assert code.dtype == torch.uint8 and code.shape == cache.shape and scale.dtype == np.float32
        vals, decs = [], []
        for b in range(w.problem.batch):
            t = np.arange(int(w.seq_lens[b]))
            pages = torch.from_numpy(w.block_table[b, t // P].astype(np.int64))
            slots = torch.from_numpy(t % P)
            vals.append(cache[pages, :, slots].float())  # [L, Hkv, d]
            decs.append(code[pages, :, slots].view(torch.float8_e4m3fn).float())
        x, c = torch.cat(vals), torch.cat(decs)
        for g in range(w.problem.num_kv_heads):
            amax = float(x[:, g].abs().max())
            assert scale[g] == np.float32(amax / 448.0)
            y = x[:, g] / float(scale[g])
            err = (y - c[:, g]).abs()
            assert torch.all(err <= torch.maximum(y.abs() * 2.0 ** -4, torch.full_like(y, 2.0 ** -10)))
            assert float(c[:, g].abs().max()) == 448.0
