"""Pins for the CPU oracle: checks that tie it to something other than itself.

Each ``pin_*`` function raises AssertionError when the oracle library passed in
(``lib``; None = the real one) breaks a fact fixed by the definition of
decode attention or of the tile plan: closed forms, invariants, special cases
that reduce to a library routine (torch's scaled_dot_product_attention and
logsumexp in float64), hand-derived worked examples, and brute force on tiny
inputs.  The same battery is run against deliberately broken copies of the
oracle (tests/test_oracle_mutants.py) to show that each plausible mistake is
caught by at least one pin.

Operation source: "Tencent HPC lands in SGLang, challenging default inference
kernels", section "Why Tencent HPC matters for online model serving".
"""

from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ---------------------------------------------------------------------------------------------
# Small case construction: dense per-request K/V -> pages, in a chosen page order.


def bf16(x) -> torch.Tensor:
    return torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)


def pack(dense_k, dense_v, page_size: int, rng: np.random.Generator | None = None, spare: int = 1,
         max_pages: int | None = None):
    """Lay out per-request dense K/V ([L_b, Hkv, d] bf16) as [pages, Hkv, P, d] with a block table."""
    Hkv, d = dense_k[0].shape[1], dense_k[0].shape[2]
    P = page_size
    used = [-(-k.shape[0] // P) for k in dense_k]
    n_pages = sum(used) + spare
    order = rng.permutation(n_pages) if rng is not None else np.arange(n_pages)
    mp = max_pages or max(1, max(used))
    bt = np.full((len(dense_k), mp), -1, dtype=np.int32)
    kc = torch.full((n_pages, Hkv, P, d), float("nan"), dtype=torch.bfloat16)
    vc = kc.clone()
    o = 0
    for b, (k, v) in enumerate(zip(dense_k, dense_v)):
        for j in range(used[b]):
            page = int(order[o]); o += 1
            bt[b, j] = page
            rows = slice(j * P, min((j + 1) * P, k.shape[0]))
            n = rows.stop - rows.start
            kc[page, :, :n, :] = k[rows].permute(1, 0, 2)
            vc[page, :, :n, :] = v[rows].permute(1, 0, 2)
    lens = np.array([k.shape[0] for k in dense_k], dtype=np.int32)
    return kc, vc, bt, lens


def random_case(rng, B, Hq, Hkv, d, P, lens, scale=None):
    q = bf16(rng.standard_normal((B, Hq, d)))
    dk = [bf16(rng.standard_normal((L, Hkv, d))) for L in lens]
    dv = [bf16(rng.standard_normal((L, Hkv, d))) for L in lens]
    kc, vc, bt, sl = pack(dk, dv, P, rng)
    scale = float(np.float32(1.0 / math.sqrt(d))) if scale is None else scale
    return q, dk, dv, kc, vc, bt, sl, scale


def run(lib, q, kc, vc, bt, sl, scale, **kw):
    return oracle.attention(q, kc, vc, bt, sl, scale=scale, lib=lib, **kw)


# ---------------------------------------------------------------------------------------------
# Attention pins.


def pin_golden_attention(lib=None):
    with open(os.path.join(GOLDEN, "attention_hand.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        d = len(c["q"])
        q = bf16(c["q"]).reshape(1, 1, d)
        k = bf16(c["k"]).reshape(-1, 1, d)
        v = bf16(c["v"]).reshape(-1, 1, d)
        assert torch.equal(q.float(), torch.tensor(c["q"]).reshape(1, 1, d)), "fixture not bf16-exact"
        kc, vc, bt, sl = pack([k], [v], c["page_size"], np.random.default_rng(7))
        out, lse, st = run(lib, q, kc, vc, bt, sl, c["scale"])
        assert st == oracle.OK
        want = np.array([eval(e, {"math": math}) for e in c["out"]])
        np.testing.assert_allclose(out[0, 0], want, rtol=1e-13, atol=1e-13, err_msg=c["name"])
        assert abs(lse[0, 0] - eval(c["lse"], {"math": math})) < 1e-13, c["name"]


def pin_length_one(lib=None):
    """One cached token: the softmax weight is 1, so out is that V row and lse is its score."""
    rng = np.random.default_rng(11)
    for (Hq, Hkv, d, P) in [(4, 1, 64, 16), (8, 2, 32, 4), (6, 3, 16, 1)]:
        q, dk, dv, kc, vc, bt, sl, scale = random_case(rng, 3, Hq, Hkv, d, P, [1, 1, 1])
        out, lse, st = run(lib, q, kc, vc, bt, sl, scale)
        assert st == oracle.OK
        G = Hq // Hkv
        for b in range(3):
            for h in range(Hq):
                g = h // G
                assert np.array_equal(out[b, h], dv[b][0, g].double().numpy())
                s0 = scale * float(torch.dot(q[b, h].double(), dk[b][0, g].double()))
                assert abs(lse[b, h] - s0) <= 1e-12 * max(1.0, abs(s0))


def pin_constant_v(lib=None):
    """If every V row equals c, every convex combination of them is c."""
    rng = np.random.default_rng(12)
    B, Hq, Hkv, d, P = 3, 8, 2, 16, 4
    lens = [5, 17, 33]
    q = bf16(rng.standard_normal((B, Hq, d)) * 3)
    dk = [bf16(rng.standard_normal((L, Hkv, d)) * 3) for L in lens]
    c = bf16(rng.standard_normal((Hkv, d)))
    dv = [c.unsqueeze(0).expand(L, Hkv, d).contiguous() for L in lens]
    kc, vc, bt, sl = pack(dk, dv, P, rng)
    out, lse, st = run(lib, q, kc, vc, bt, sl, 0.3)
    assert st == oracle.OK
    for b in range(B):
        for h in range(Hq):
            np.testing.assert_allclose(out[b, h], c[h // (Hq // Hkv)].double().numpy(), rtol=1e-13, atol=1e-14)


def pin_uniform_scores(lib=None):
    """q = 0 (or scale = 0): all scores are 0, so out is the mean of the V rows and lse = ln L."""
    rng = np.random.default_rng(13)
    B, Hq, Hkv, d, P = 3, 4, 2, 8, 3
    lens = [1, 10, 29]
    _, dk, dv, kc, vc, bt, sl, _ = random_case(rng, B, Hq, Hkv, d, P, lens)
    for qv, sc in [(torch.zeros(B, Hq, d, dtype=torch.bfloat16), 0.7),
                   (bf16(rng.standard_normal((B, Hq, d))), 0.0)]:
        out, lse, st = run(lib, qv, kc, vc, bt, sl, sc)
        assert st == oracle.OK
        for b, L in enumerate(lens):
            for h in range(Hq):
                g = h // (Hq // Hkv)
                np.testing.assert_allclose(out[b, h], dv[b][:, g].double().mean(0).numpy(), rtol=1e-12, atol=1e-13)
                assert abs(lse[b, h] - math.log(L)) < 1e-13


def pin_dominant_key(lib=None):
    """One key far ahead of the rest: the output tends to its V row, lse to its score."""
    rng = np.random.default_rng(14)
    d, L, P = 16, 40, 8
    q = bf16(np.ones((1, 1, d)))
    k = torch.zeros(L, 1, d, dtype=torch.bfloat16)
    k[23, 0, :] = 4.0  # score 64 * scale vs 0 elsewhere
    v = bf16(rng.standard_normal((L, 1, d)))
    kc, vc, bt, sl = pack([k], [v], P, rng)
    out, lse, st = run(lib, q, kc, vc, bt, sl, 1.0)
    assert st == oracle.OK
    # exact answer: weight w = e^64 / (e^64 + 39) on row 23, (1 - w)/39 on each other row
    np.testing.assert_allclose(out[0, 0], v[23, 0].double().numpy(), rtol=1e-15, atol=40 * math.exp(-64) * 4)
    assert abs(lse[0, 0] - 64.0) < 1e-20 + 39 * math.exp(-64)


def pin_page_order_invariance(lib=None):
    """Moving pages around while rewriting the block table must not change a single bit."""
    rng = np.random.default_rng(15)
    B, Hq, Hkv, d, P = 4, 8, 2, 32, 4
    lens = [3, 4, 9, 30]
    q = bf16(rng.standard_normal((B, Hq, d)))
    dk = [bf16(rng.standard_normal((L, Hkv, d))) for L in lens]
    dv = [bf16(rng.standard_normal((L, Hkv, d))) for L in lens]
    a = run(lib, q, *pack(dk, dv, P, np.random.default_rng(1)), 0.25)
    b = run(lib, q, *pack(dk, dv, P, np.random.default_rng(2), spare=5), 0.25)
    c = run(lib, q, *pack(dk, dv, P, None), 0.25)
    assert a[2] == b[2] == c[2] == oracle.OK
    for x in (b, c):
        assert np.array_equal(a[0], x[0]) and np.array_equal(a[1], x[1])


def pin_prefix_sharing(lib=None):
    """Two requests whose block tables name the same pages (a shared prefix) see the same tokens."""
    rng = np.random.default_rng(16)
    Hq, Hkv, d, P = 4, 2, 16, 4
    q1 = bf16(rng.standard_normal((1, Hq, d)))
    k = bf16(rng.standard_normal((12, Hkv, d)))
    v = bf16(rng.standard_normal((12, Hkv, d)))
    kc, vc, bt, sl = pack([k], [v], P, rng)
    bt2 = np.concatenate([bt, bt], 0)
    q2 = torch.cat([q1, q1], 0)
    out, lse, st = run(lib, q2, kc, vc, bt2, np.array([12, 8], np.int32), 0.25)
    ref8, lse8, _ = run(lib, q1, *pack([k[:8]], [v[:8]], P, None), 0.25)
    ref12, lse12, _ = run(lib, q1, *pack([k], [v], P, None), 0.25)
    assert st == oracle.OK
    assert np.array_equal(out[0], ref12[0]) and np.array_equal(out[1], ref8[0])
    assert np.array_equal(lse[1], lse8[0]) and np.array_equal(lse[0], lse12[0])


def pin_matches_sdpa(lib=None):
    """Brute force by a library routine: torch SDPA (float64, GQA) and logsumexp over the gathered cache."""
    rng = np.random.default_rng(17)
    for (B, Hq, Hkv, d, P, lens) in [(3, 4, 1, 64, 16, [1, 7, 40]), (2, 8, 2, 8, 3, [13, 26]),
                                     (2, 6, 3, 16, 1, [5, 9]), (4, 16, 2, 128, 64, [64, 65, 130, 1])]:
        q, dk, dv, kc, vc, bt, sl, scale = random_case(rng, B, Hq, Hkv, d, P, lens)
        out, lse, st = run(lib, q, kc, vc, bt, sl, scale)
        assert st == oracle.OK
        for b in range(B):
            qb = q[b].double().unsqueeze(0).unsqueeze(2)  # [1, Hq, 1, d]
            kb = dk[b].double().permute(1, 0, 2).unsqueeze(0)  # [1, Hkv, L, d]
            vb = dv[b].double().permute(1, 0, 2).unsqueeze(0)
            ref = torch.nn.functional.scaled_dot_product_attention(qb, kb, vb, scale=scale, enable_gqa=True)
            np.testing.assert_allclose(out[b], ref[0, :, 0].numpy(), rtol=1e-11, atol=1e-12)
            kx = kb.repeat_interleave(Hq // Hkv, dim=1)  # torch's GQA convention
            s = torch.einsum("hd,htd->ht", qb[0, :, 0], kx[0]) * scale
            np.testing.assert_allclose(lse[b], torch.logsumexp(s, dim=1).numpy(), rtol=1e-12, atol=1e-12)


def pin_split_merge_identity(lib=None):
    """Attention over [0, a) and [a, L) merged by log-sum-exp equals attention over [0, L).

    The second piece is taken by starting the block table at page a / P.  The
    merged result is checked both with the oracle's combine and with a
    weighting written here from the two partial normalisers.
    """
    rng = np.random.default_rng(18)
    Hq, Hkv, d, P = 4, 2, 16, 4
    L = 37
    q = bf16(rng.standard_normal((1, Hq, d)))
    k = bf16(rng.standard_normal((L, Hkv, d)))
    v = bf16(rng.standard_normal((L, Hkv, d)))
    kc, vc, bt, sl = pack([k], [v], P, rng)
    full, full_lse, _ = run(lib, q, kc, vc, bt, sl, 0.4)
    for a in (4, 8, 20, 36):
        pieces = [(bt, a), (bt[:, a // P:], L - a)]
        parts = [run(lib, q, kc, vc, np.ascontiguousarray(t), np.array([n], np.int32), 0.4) for t, n in pieces]
        for h in range(Hq):
            o = np.stack([p[0][0, h] for p in parts])
            l = np.array([p[1][0, h] for p in parts])
            merged, merged_lse = oracle.combine(o, l, lib=lib)
            np.testing.assert_allclose(merged, full[0, h], rtol=1e-12, atol=1e-13)
            assert abs(merged_lse - full_lse[0, h]) < 1e-12
            # a second, separately written merge: weights e^{lse_i} / e^{lse_full}
            w = np.exp(l - full_lse[0, h])
            assert abs(w.sum() - 1.0) < 1e-12
            np.testing.assert_allclose((w[:, None] * o).sum(0), full[0, h], rtol=1e-12, atol=1e-13)
    # merging with an empty piece (lse = -inf) changes nothing
    m, ml = oracle.combine(np.stack([full[0, 0], np.zeros(d)]), np.array([full_lse[0, 0], -np.inf]), lib=lib)
    assert np.array_equal(m, full[0, 0]) or np.allclose(m, full[0, 0], rtol=1e-15)
    assert ml == full_lse[0, 0]
    m, ml = oracle.combine(np.zeros((2, d)), np.array([-np.inf, -np.inf]), lib=lib)
    assert ml == -np.inf and not m.any()


def pin_degenerate_lengths(lib=None):
    """Length 0 gives out = 0, lse = -inf; out-of-range lengths are reported and count as 0."""
    rng = np.random.default_rng(19)
    Hq, Hkv, d, P = 2, 1, 8, 4
    q, dk, dv, kc, vc, bt, sl, scale = random_case(rng, 2, Hq, Hkv, d, P, [0, 6])
    out, lse, st = run(lib, q, kc, vc, bt, sl, scale)
    assert st == oracle.OK
    assert not out[0].any() and np.all(lse[0] == -np.inf) and np.all(np.isfinite(lse[1]))
    for bad in (-1, bt.shape[1] * P + 1):
        out, lse, st = run(lib, q, kc, vc, bt, np.array([bad, 6], np.int32), scale)
        assert st == oracle.ERR_BAD_SEQLEN
        assert not out[0].any() and np.all(lse[0] == -np.inf)
    bt2 = bt.copy()
    bt2[1, 0] = kc.shape[0]  # page id out of range
    _, _, st = run(lib, q, kc, vc, bt2, sl, scale)
    assert st == oracle.ERR_BAD_PAGE


def pin_pairs_match_full(lib=None):
    rng = np.random.default_rng(20)
    q, dk, dv, kc, vc, bt, sl, scale = random_case(rng, 3, 8, 2, 16, 4, [3, 11, 20])
    full, full_lse, _ = run(lib, q, kc, vc, bt, sl, scale)
    pb = np.array([2, 0, 1, 2], np.int32)
    ph = np.array([7, 0, 3, 4], np.int32)
    sub, sub_lse, st = run(lib, q, kc, vc, bt, sl, scale, pairs=(pb, ph))
    assert st == oracle.OK
    assert np.array_equal(sub, full[pb, ph]) and np.array_equal(sub_lse, full_lse[pb, ph])


# ---------------------------------------------------------------------------------------------
# FP8 (E4M3) cache pins.


def random_fp8_case(rng, B, Hq, Hkv, d, P, lens, k_scale, v_scale):
    """Random E4M3 codes (NaN codes excluded) laid out in shuffled pages, plus the dequantised dense K/V."""
    n_pages = sum(-(-L // P) for L in lens) + 2
    codes = rng.integers(0, 256, size=(2, n_pages, Hkv, P, d), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x3C  # avoid the NaN codes
    perm = rng.permutation(n_pages)
    mp = max(1, max(-(-L // P) for L in lens))
    bt = np.full((B, mp), -1, np.int32)
    o = 0
    for b, L in enumerate(lens):
        n = -(-L // P)
        bt[b, :n] = perm[o:o + n]
        o += n
    deq = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64)
    deq[0] *= torch.tensor(k_scale, dtype=torch.float64)[None, :, None, None]
    deq[1] *= torch.tensor(v_scale, dtype=torch.float64)[None, :, None, None]
    dense = []
    for b, L in enumerate(lens):
        t = np.arange(L)
        pages, slots = bt[b, t // P], t % P
        dense.append((deq[0][pages, :, slots, :], deq[1][pages, :, slots, :]))  # [L, Hkv, d]
    q = bf16(rng.standard_normal((B, Hq, d)))
    return q, codes[0], codes[1], bt, np.array(lens, np.int32), dense


def pin_e4m3_decoding(lib=None):
    """All 256 E4M3 codes against torch's float8_e4m3fn conversion."""
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    for c in range(256):
        v = oracle.e4m3_value(c, lib=lib)
        r = float(ref[c])
        assert (math.isnan(v) and math.isnan(r)) or v == r, (c, v, r)


def pin_fp8_matches_sdpa(lib=None):
    rng = np.random.default_rng(22)
    B, Hq, Hkv, d, P, lens = 3, 8, 2, 64, 16, [1, 40, 97]
    ks, vs = [0.013, 0.002], [0.5, 0.07]
    q, kc, vc, bt, sl, dense = random_fp8_case(rng, B, Hq, Hkv, d, P, lens, ks, vs)
    scale = 0.125
    out, lse, st = oracle.attention_fp8(q, kc, vc, ks, vs, bt, sl, scale=scale, lib=lib)
    assert st == oracle.OK
    for b in range(B):
        kb = dense[b][0].permute(1, 0, 2).unsqueeze(0)
        vb = dense[b][1].permute(1, 0, 2).unsqueeze(0)
        qb = q[b].double().unsqueeze(0).unsqueeze(2)
        ref = torch.nn.functional.scaled_dot_product_attention(qb, kb, vb, scale=scale, enable_gqa=True)
        np.testing.assert_allclose(out[b], ref[0, :, 0].numpy(), rtol=1e-11, atol=1e-12)
        s = torch.einsum("hd,htd->ht", qb[0, :, 0], kb.repeat_interleave(Hq // Hkv, dim=1)[0]) * scale
        np.testing.assert_allclose(lse[b], torch.logsumexp(s, dim=1).numpy(), rtol=1e-12, atol=1e-12)


def pin_fp8_equals_bf16_when_exact(lib=None):
    """With power-of-two scales every dequantised value is exact in bf16: both formats give the same bits."""
    rng = np.random.default_rng(23)
    B, Hq, Hkv, d, P, lens = 2, 4, 2, 32, 8, [9, 30]
    ks, vs = [0.125, 4.0], [2.0 ** -6, 1.0]
    q, kc, vc, bt, sl, _ = random_fp8_case(rng, B, Hq, Hkv, d, P, lens, ks, vs)
    deq = lambda c, sc: (torch.from_numpy(c).view(torch.float8_e4m3fn).to(torch.float64)
                         * torch.tensor(sc, dtype=torch.float64)[None, :, None, None])
    kb, vb = deq(kc, ks).to(torch.bfloat16), deq(vc, vs).to(torch.bfloat16)
    assert torch.equal(kb.double(), deq(kc, ks)) and torch.equal(vb.double(), deq(vc, vs))
    a = oracle.attention_fp8(q, kc, vc, ks, vs, bt, sl, scale=0.3, lib=lib)
    b = oracle.attention(q, kb, vb, bt, sl, scale=0.3, lib=lib)
    assert a[2] == b[2] == oracle.OK
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


# ---------------------------------------------------------------------------------------------
# Multi-query decode pins.


def pin_mq_matches_sdpa_with_causal_mask(lib=None):
    """Q new tokens at the end of each cache; torch SDPA (float64) with an explicit position mask."""
    rng = np.random.default_rng(24)
    for (B, Q, Hq, Hkv, d, P, lens) in [(3, 2, 8, 2, 16, 4, [2, 9, 30]), (2, 4, 4, 1, 8, 3, [1, 13]),
                                        (1, 3, 6, 3, 32, 8, [5])]:
        _, dk, dv, kc, vc, bt, sl, scale = random_case(rng, B, Hq, Hkv, d, P, lens)
        q = bf16(rng.standard_normal((B, Q, Hq, d)))
        out, lse, st = oracle.attention_mq(q, kc, vc, bt, sl, scale=scale, lib=lib)
        assert st == oracle.OK
        for b, L in enumerate(lens):
            pos = torch.arange(L)
            for i in range(Q):
                qpos = L - Q + i
                if qpos < 0:
                    assert not out[b, i].any() and np.all(lse[b, i] == -np.inf)
                    continue
                mask = (pos <= qpos).view(1, 1, 1, L)
                qb = q[b, i].double().unsqueeze(0).unsqueeze(2)
                kb = dk[b].double().permute(1, 0, 2).unsqueeze(0)
                vb = dv[b].double().permute(1, 0, 2).unsqueeze(0)
                ref = torch.nn.functional.scaled_dot_product_attention(qb, kb, vb, attn_mask=mask, scale=scale,
                                                                       enable_gqa=True)
                np.testing.assert_allclose(out[b, i], ref[0, :, 0].numpy(), rtol=1e-11, atol=1e-12)
                s_ = torch.einsum("hd,htd->ht", qb[0, :, 0], kb.repeat_interleave(Hq // Hkv, dim=1)[0]) * scale
                s_ = s_.masked_fill(~mask.view(1, L), float("-inf"))
                np.testing.assert_allclose(lse[b, i], torch.logsumexp(s_, dim=1).numpy(), rtol=1e-12, atol=1e-12)


def pin_mq_single_query_is_decode(lib=None):
    """With one query per request, multi-query decode is plain decode, bit for bit."""
    rng = np.random.default_rng(25)
    q, dk, dv, kc, vc, bt, sl, scale = random_case(rng, 3, 8, 2, 16, 4, [1, 7, 33])
    a = oracle.attention(q, kc, vc, bt, sl, scale=scale, lib=lib)
    b = oracle.attention_mq(q.unsqueeze(1).contiguous(), kc, vc, bt, sl, scale=scale, lib=lib)
    assert a[2] == b[2] == oracle.OK
    assert np.array_equal(a[0], b[0][:, 0]) and np.array_equal(a[1], b[1][:, 0])


ATTENTION_PINS = [pin_golden_attention, pin_length_one, pin_constant_v, pin_uniform_scores, pin_dominant_key,
                  pin_page_order_invariance, pin_prefix_sharing, pin_matches_sdpa, pin_split_merge_identity,
                  pin_degenerate_lengths, pin_pairs_match_full, pin_e4m3_decoding, pin_fp8_matches_sdpa,
                  pin_fp8_equals_bf16_when_exact, pin_mq_matches_sdpa_with_causal_mask,
                  pin_mq_single_query_is_decode]


# ---------------------------------------------------------------------------------------------
# Plan pins.


def cta_starts(U, C, weights=None):
    """First unit of each CTA's range (and U at the end): the even split floor(c*U/C), or with
    weights (and U >= C) one unit per CTA plus the other U - C units dealt out in proportion."""
    if weights is None or U < C:
        return [c * U // C for c in range(C + 1)]
    W = sum(weights)
    acc = [sum(weights[:c]) for c in range(C + 1)]
    return [c + (U - C) * acc[c] // W for c in range(C + 1)]


def brute_force_plan(seq_lens, T, C, capacity, start_cost=0, weights=None):
    """The dynamic plan by scanning: lay out every unit (a request's start units, then its tiles),
    and for each tile unit search the CTA whose range holds it."""
    n = [(-(-L // T) if 0 <= L <= capacity else 0) for L in seq_lens]
    units = []  # (request, tile or None for a start unit)
    for r, nr in enumerate(n):
        if nr:
            units += [(r, None)] * start_cost + [(r, t) for t in range(nr)]
    U = len(units)
    starts = cta_starts(U, C, weights)
    segs = []  # [req, cta, tile_begin, tile_end]
    for u, (r, t) in enumerate(units):
        if t is None:
            continue
        cta = next(c for c in range(C) if starts[c] <= u < starts[c + 1])
        if segs and segs[-1][0] == r and segs[-1][1] == cta:
            segs[-1][3] = t + 1
        else:
            segs.append([r, cta, t, t + 1])
    return n, U, segs


def check_plan_invariants(p, seq_lens, T, C, capacity, start_cost=0, weights=None):
    n = [(-(-L // T) if 0 <= L <= capacity else 0) for L in seq_lens]
    w = [nr + start_cost if nr else 0 for nr in n]  # units per request, start units included
    B, U, S = len(seq_lens), sum(w), p["num_segments"]
    assert p["num_units"] == U
    assert list(p["req_tile_prefix"]) == list(np.concatenate([[0], np.cumsum(w)]))
    assert S <= C + max(B, 1) - 1
    req, cta, tb, te = p["seg_req"], p["seg_cta"], p["seg_tile_begin"], p["seg_tile_end"]
    assert np.all(te > tb)  # no empty segment in a dynamic plan
    # segments of each request tile [0, n_b) in order, without gap or overlap
    for b in range(B):
        s0, s1 = p["req_seg_begin"][b], p["req_seg_begin"][b + 1]
        assert np.all(req[s0:s1] == b)
        cover = [t for s in range(s0, s1) for t in range(tb[s], te[s])]
        assert cover == list(range(n[b]))
    # each CTA's load (its tiles plus the start units in its range) is floor or ceil of U / C,
    # its segments are contiguous, in unit order, and inside its range of units
    prefix = p["req_tile_prefix"]
    first = cta_starts(U, C, weights)
    start_units = np.zeros(C, np.int64)
    for b in range(B):
        for u in range(int(prefix[b]), int(prefix[b]) + (start_cost if n[b] else 0)):
            start_units[next(c for c in range(C) if first[c] <= u < first[c + 1])] += 1
    loads = np.zeros(C, np.int64)
    for c in range(C):
        s0, s1 = p["cta_seg_begin"][c], p["cta_seg_begin"][c + 1]
        assert np.all(cta[s0:s1] == c)
        loads[c] = int((te[s0:s1] - tb[s0:s1]).sum()) + start_units[c]
        for s in range(s0, s1):
            u0 = int(prefix[req[s]]) + start_cost + int(tb[s])
            assert first[c] <= u0 and u0 + int(te[s] - tb[s]) <= first[c + 1]
    assert loads.sum() == U
    if U and (weights is None or U < C):
        assert loads.min() >= U // C and loads.max() <= -(-U // C)
    elif U:
        # every CTA holds one unit plus, within one unit, its weight's share of the other U - C
        share = (U - C) * np.asarray(weights, np.float64) / float(sum(weights))
        assert np.all(loads >= 1) and np.all(np.abs(loads - 1 - share) < 1.0 + 1e-9)
    units = [prefix[req[s]] + start_cost + tb[s] for s in range(S)]
    assert units == sorted(units)


def compare_plan(p, want: dict):
    for key in ("num_units", "num_segments"):
        assert p[key] == want[key], key
    for key in ("req_tile_prefix", "req_seg_begin", "cta_seg_begin", "seg_req", "seg_cta", "seg_tile_begin",
                "seg_tile_end"):
        assert list(p[key]) == list(want[key]), key


def pin_golden_plans(lib=None):
    with open(os.path.join(GOLDEN, "plan_hand.json")) as f:
        g = json.load(f)
    for c in g["dynamic"]:
        p = oracle.plan(c["seq_lens"], c["tile_tokens"], c["num_ctas"], 1 << 20, lib=lib,
                        start_cost=c.get("start_cost", 0), weights=c.get("weights"))
        compare_plan(p, c)
    for c in g["static"]:
        p = oracle.static_plan(c["seq_lens"], c["tile_tokens"], c["splits"], 1 << 20, lib=lib)
        compare_plan(p, c)


def pin_plan_brute_force(lib=None, exhaustive_batch: int = 3, max_len: int = 5):
    import itertools
    for B in range(0, exhaustive_batch + 1):
        for lens in itertools.product(range(max_len + 1), repeat=B):
            for T in (1, 2, 3):
                for C in range(1, 7):
                    p = oracle.plan(list(lens), T, C, 1 << 20, lib=lib)
                    n, U, segs = brute_force_plan(list(lens), T, C, 1 << 20)
                    got = list(zip(p["seg_req"], p["seg_cta"], p["seg_tile_begin"], p["seg_tile_end"]))
                    assert got == [tuple(s) for s in segs], (lens, T, C)
                    check_plan_invariants(p, list(lens), T, C, 1 << 20)


def pin_plan_random(lib=None):
    rng = np.random.default_rng(21)
    for _ in range(60):
        B = int(rng.integers(1, 300))
        C = int(rng.choice([1, 7, 37, 148, 296, 1000]))
        T = int(rng.choice([16, 32, 64, 128]))
        lens = rng.integers(0, 5000, size=B)
        lens[rng.random(B) < 0.2] = 0
        p = oracle.plan(lens, T, C, 1 << 20, lib=lib)
        check_plan_invariants(p, list(lens), T, C, 1 << 20)
        if B * C < 20000:
            _, _, segs = brute_force_plan(list(lens), T, C, 1 << 20)
            got = list(zip(p["seg_req"], p["seg_cta"], p["seg_tile_begin"], p["seg_tile_end"]))
            assert got == [tuple(s) for s in segs]


def pin_plan_start_cost_brute_force(lib=None):
    """Start units: every small case against the explicit unit walk, sigma = 1, 2, 3."""
    import itertools
    for B in range(0, 4):
        for lens in itertools.product(range(5), repeat=B):
            for T in (1, 2):
                for C in range(1, 7):
                    for sc in (1, 2, 3):
                        p = oracle.plan(list(lens), T, C, 1 << 20, lib=lib, start_cost=sc)
                        _, _, segs = brute_force_plan(list(lens), T, C, 1 << 20, start_cost=sc)
                        got = list(zip(p["seg_req"], p["seg_cta"], p["seg_tile_begin"], p["seg_tile_end"]))
                        assert got == [tuple(s) for s in segs], (lens, T, C, sc)
                        check_plan_invariants(p, list(lens), T, C, 1 << 20, start_cost=sc)


def pin_plan_start_cost_random(lib=None):
    """Start units at serving sizes: invariants always, the explicit walk where it is cheap;
    sigma = 0 through the start-cost entry point is the plain plan."""
    rng = np.random.default_rng(23)
    lib = lib or oracle._load()
    for _ in range(40):
        B = int(rng.integers(1, 300))
        C = int(rng.choice([1, 7, 37, 148, 296, 1000]))
        T = int(rng.choice([16, 64, 128]))
        sc = int(rng.choice([1, 2, 5]))
        lens = rng.integers(0, 5000, size=B)
        lens[rng.random(B) < 0.2] = 0
        p = oracle.plan(lens, T, C, 1 << 20, lib=lib, start_cost=sc)
        check_plan_invariants(p, list(lens), T, C, 1 << 20, start_cost=sc)
        if B * C < 20000:
            _, _, segs = brute_force_plan(list(lens), T, C, 1 << 20, start_cost=sc)
            got = list(zip(p["seg_req"], p["seg_cta"], p["seg_tile_begin"], p["seg_tile_end"]))
            assert got == [tuple(s) for s in segs]
        plain = oracle.plan(lens, T, C, 1 << 20, lib=lib)
        zero = oracle._run_plan(lib.dao_plan_start_cost, lens, T, C, 1 << 20, C + B - 1, C, 0)
        compare_plan(zero, plain)


def pin_plan_weighted_brute_force(lib=None):
    """Weighted ranges: every small case against the explicit unit walk, with weights from
    equal to skewed by 65536 : 1, sigma = 0 and 2."""
    import itertools
    rng = np.random.default_rng(27)
    for B in range(0, 4):
        for lens in itertools.product(range(5), repeat=B):
            for T in (1, 2):
                for C in range(1, 6):
                    for wv in ([1] * C, list(rng.integers(1, 10, size=C)), [65536] + [1] * (C - 1),
                               [1] * (C - 1) + [65536]):
                        for sc in (0, 2):
                            p = oracle.plan(list(lens), T, C, 1 << 20, lib=lib, start_cost=sc, weights=wv)
                            _, _, segs = brute_force_plan(list(lens), T, C, 1 << 20, start_cost=sc, weights=wv)
                            got = list(zip(p["seg_req"], p["seg_cta"], p["seg_tile_begin"], p["seg_tile_end"]))
                            assert got == [tuple(s) for s in segs], (lens, T, C, wv, sc)
                            check_plan_invariants(p, list(lens), T, C, 1 << 20, start_cost=sc, weights=wv)


def pin_plan_weighted_random(lib=None):
    """Weighted ranges at serving sizes: invariants (each CTA within one unit of its weight's
    share), the explicit walk where cheap, and equal weights give the even split exactly."""
    rng = np.random.default_rng(29)
    lib = lib or oracle._load()
    for _ in range(30):
        B = int(rng.integers(1, 300))
        C = int(rng.choice([1, 7, 37, 148, 296, 1000]))
        T = int(rng.choice([16, 64, 128]))
        sc = int(rng.choice([0, 2]))
        lens = rng.integers(0, 5000, size=B)
        lens[rng.random(B) < 0.2] = 0
        wv = rng.integers(1, 65537, size=C) if rng.random() < 0.5 else rng.integers(900, 1200, size=C)
        p = oracle.plan(lens, T, C, 1 << 20, lib=lib, start_cost=sc, weights=wv)
        check_plan_invariants(p, list(lens), T, C, 1 << 20, start_cost=sc, weights=list(wv))
        if B * C < 20000:
            _, _, segs = brute_force_plan(list(lens), T, C, 1 << 20, start_cost=sc, weights=list(wv))
            got = list(zip(p["seg_req"], p["seg_cta"], p["seg_tile_begin"], p["seg_tile_end"]))
            assert got == [tuple(s) for s in segs]
        even = oracle.plan(lens, T, C, 1 << 20, lib=lib, start_cost=sc, weights=np.full(C, int(rng.integers(1, 65537))))
        compare_plan(even, oracle.plan(lens, T, C, 1 << 20, lib=lib, start_cost=sc))


def pin_plan_bad_lengths(lib=None):
    p = oracle.plan([5, -3, 7, 99, 2], 2, 3, 10, lib=lib)
    assert p["status"] == oracle.ERR_BAD_SEQLEN and p["bad_index"] == 1
    check_plan_invariants(p, [5, 0, 7, 0, 2], 2, 3, 10)
    p = oracle.plan([5, 3], 2, 3, 10, lib=lib)
    assert p["status"] == oracle.OK and p["bad_index"] == -1


def brute_force_static(seq_lens, T, S, capacity):
    n = [(-(-L // T) if 0 <= L <= capacity else 0) for L in seq_lens]
    maxT = max(n, default=0)
    chunk = -(-maxT // S)
    # split s of request b takes the tiles t < n_b with t // chunk == s
    segs = []
    for b, nb in enumerate(n):
        for s in range(S):
            tiles = [t for t in range(nb) if chunk and t // chunk == s]
            lo = tiles[0] if tiles else min(s * chunk, nb)
            hi = tiles[-1] + 1 if tiles else lo
            segs.append((b, b * S + s, lo, hi))
    return n, segs


def pin_static_brute_force(lib=None):
    import itertools
    for B in range(0, 4):
        for lens in itertools.product([0, 1, 3, 8, 17], repeat=B):
            for T in (1, 4):
                for S in (1, 2, 3, 5):
                    p = oracle.static_plan(list(lens), T, S, 1 << 20, lib=lib)
                    n, segs = brute_force_static(list(lens), T, S, 1 << 20)
                    got = list(zip(p["seg_req"], p["seg_cta"], p["seg_tile_begin"], p["seg_tile_end"]))
                    assert got == segs, (lens, T, S)
                    assert p["num_units"] == sum(n)
                    assert list(p["req_seg_begin"]) == [b * S for b in range(B + 1)]
                    assert list(p["cta_seg_begin"]) == list(range(B * S + 1))
                    # the longest request's splits are non-empty up to ceil(maxT / chunk) of them
                    if n and max(n):
                        chunk = -(-max(n) // S)
                        assert sum(1 for s in segs if s[3] > s[2]) == sum(-(-x // chunk) for x in n)


def pin_static_empty_splits(lib=None):
    """Static split-k sized by the longest request leaves the short ones' later splits empty
    (counted by hand: chunk = ceil(250 / 8) = 32 tiles; busy splits 1 + 3 + 1 + 8 of 32)."""
    p = oracle.static_plan([100, 5000, 70, 16000], 64, 8, 2048 * 64, lib=lib)
    empty = int(np.sum(np.asarray(p["seg_tile_end"]) == np.asarray(p["seg_tile_begin"])))
    assert p["num_segments"] == 32 and empty == 19


PLAN_PINS = [pin_golden_plans, pin_plan_brute_force, pin_plan_random, pin_plan_start_cost_brute_force,
             pin_plan_start_cost_random, pin_plan_weighted_brute_force, pin_plan_weighted_random,
             pin_plan_bad_lengths, pin_static_brute_force, pin_static_empty_splits]
