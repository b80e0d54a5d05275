"""The C ABI seen from the host, without a GPU: exports, sizes, layout and argument checks.

Every call here returns before any CUDA call is made (argument checks come
first), so nothing is launched.
"""

import re
import subprocess

import pytest

from conftest import ROOT, cuda_available

HEADER = f"{ROOT}/include/da.h"


def header_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"DA_API\s+[\w\s\*]+?\b(da_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported(da_lib):
    declared = header_functions()
    assert len(declared) >= 10
    out = subprocess.run(["nm", "-D", "--defined-only", da_lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (da_\w+)", out))
    assert set(declared) <= exported, set(declared) - exported
    assert exported <= set(declared), f"undeclared exports: {exported - set(declared)}"
    assert sorted(da_lib.EXPORTS) == declared
    for name in declared:
        getattr(da_lib.lib(), name)


def prob(da, **kw):
    base = dict(batch=32, num_q_heads=64, num_kv_heads=8, head_dim=128, page_size=64, max_pages_per_req=250,
                num_pages=8400, scale=0.08838834764831845)
    base.update(kw)
    return da.problem(**base)


def test_plan_descriptor_and_sizes(da_lib):
    da = da_lib
    p = prob(da)
    d = da.da_plan_desc_init(p, da.PLAN_DYNAMIC, 64, 37)
    assert (d.kind, d.batch, d.tile_tokens, d.num_ctas, d.splits, d.max_segments) == (0, 32, 64, 37, 0, 37 + 32 - 1)
    assert (d.num_kv_heads, d.merge_in_decode) == (8, 0)
    ws, po, pl = da.da_workspace_size(p, d)
    off = da.da_workspace_offsets(d)
    assert off[0] == 0 and off[1] == 16 and off[2] == 16 + 4 * d.max_segments
    assert off[3] == off[2] + 33 and off[4] == off[3] + 33 and off[5] == off[4] + 38
    assert off[6] >= off[5] + 32 * 8 and off[6] % 4 == 0
    assert ws == off[6] * 4 and ws % 16 == 0
    assert po == d.max_segments * 64 * 128 * 4 and pl == d.max_segments * 64 * 4
    s = da.da_plan_desc_init(p, da.PLAN_STATIC, 32, 3)
    assert (s.kind, s.num_ctas, s.splits, s.max_segments, s.tile_tokens) == (1, 96, 3, 96, 32)
    d0 = da.da_plan_desc_init(p, da.PLAN_DYNAMIC, 0, 5)
    assert d0.tile_tokens == 64
    # the one-call size query is the descriptor's sizes
    assert da.da_plan_workspace_size(p, 64, 37) == (ws, po, pl)
    assert da.da_plan_workspace_size(p, 32, 5) == da.da_workspace_size(p, da.da_plan_desc_init(p, da.PLAN_DYNAMIC,
                                                                                                 32, 5))
    with pytest.raises(da.DaError) as e:
        da.da_plan_workspace_size(prob(da, head_dim=96), 64, 37)
    assert e.value.code == da.ERR_UNSUPPORTED


def test_noalloc_scratch_limit_boundary(da_lib):
    """The documented limit of the no-allocation step at 64 query heads, d 128, C = 37: 471 requests
    fit the 16 MiB scratch, 472 do not.  With null buffers the first passes the size check and stops
    at the pointer check; the second is refused for size first."""
    import ctypes
    da = da_lib
    sizes = {}
    for B in (471, 472):
        p = prob(da, batch=B)
        ws, po, pl = da.da_plan_workspace_size(p, 64, 37)
        sizes[B] = sum((x + 255) // 256 * 256 for x in (ws, po, pl))
        rc = da.lib().da_decode_step_noalloc(ctypes.byref(p), 64, 37, *([None] * 7), None)
        assert rc == (da.ERR_INVALID_ARG if B == 471 else da.ERR_WORKSPACE), (B, rc)
    assert sizes[471] <= da.NOALLOC_SCRATCH_BYTES < sizes[472]


@pytest.mark.parametrize("kw,code", [
    (dict(num_q_heads=60), -1),          # Hq % Hkv != 0
    (dict(head_dim=96), -2),             # only 64 / 128 are built
    (dict(page_size=8), -2),             # pages must be multiples of 16 rows
    (dict(num_q_heads=256, num_kv_heads=8), -2),  # 32 query heads per KV head do not fit one MMA tile
    (dict(q_len=3), -2),                 # 8 heads x 3 queries > 16 rows
    (dict(q_len=-1), -1),
    (dict(batch=-1), -1),
    (dict(num_pages=0), -1),
    (dict(num_pages=1 << 30), -2),       # row index would overflow int32
])
def test_problem_checks(da_lib, kw, code):
    da = da_lib
    with pytest.raises(da.DaError) as e:
        da.da_plan_desc_init(prob(da, **kw), da.PLAN_DYNAMIC, 64, 37)
    assert e.value.code == code


def test_descriptor_checks(da_lib):
    da = da_lib
    p = prob(da)
    for kind, T, w, code in [(0, 24, 37, -2), (0, -16, 37, -1), (0, 64, -1, -1), (7, 64, 37, -1)]:
        with pytest.raises(da.DaError) as e:
            da.da_plan_desc_init(p, kind, T, w)
        assert e.value.code == code
    lib = da.lib()
    import ctypes
    d = da.da_plan_desc_init(p, da.PLAN_DYNAMIC, 64, 37)
    bad = da.DaPlanDesc(d.kind, d.batch, d.tile_tokens, d.num_ctas, d.splits, d.max_segments - 1, 8, 1)
    assert lib.da_workspace_size(ctypes.byref(p), ctypes.byref(bad), None, None, None) == -1
    # a dynamic call given a static descriptor, and a workspace that is too small
    s = da.da_plan_desc_init(p, da.PLAN_STATIC, 64, 2)
    assert lib.da_plan(ctypes.byref(p), ctypes.byref(s), 16, 256, 1 << 20, None) == -1
    assert lib.da_plan(ctypes.byref(p), ctypes.byref(d), 16, 256, 64, None) == -4
    assert lib.da_plan(ctypes.byref(p), ctypes.byref(d), None, 256, 1 << 20, None) == -1
    assert lib.da_plan(ctypes.byref(p), ctypes.byref(d), 16, 8, 1 << 20, None) == -1  # misaligned workspace
    assert lib.da_decode_attention(ctypes.byref(p), ctypes.byref(d), *([None] * 10), None) == -1
    assert lib.da_combine(None, ctypes.byref(d), *([None] * 5), None) == -1
    assert lib.da_read_status(None, None, None, None) == -1
    assert lib.da_workspace_offsets(None, None) == -1
    # output format: bf16 by default; fp32 is allowed with the combine kernel only
    assert d.out_format == da.OUT_BF16
    f = da.da_plan_desc_init(p, da.PLAN_DYNAMIC, 64, 37, out_f32=True)
    assert da.da_workspace_size(p, f) == da.da_workspace_size(p, d)
    for merge, fmt in ((1, da.OUT_F32), (0, 2), (0, -1)):
        bad = da.da_plan_desc_init(p, da.PLAN_DYNAMIC, 64, 37)
        bad.merge_in_decode, bad.out_format = merge, fmt
        assert lib.da_workspace_size(ctypes.byref(p), ctypes.byref(bad), None, None, None) == -1
    # fp32 output must be 16-byte aligned (the combine stores four floats at a time)
    A = 1 << 12
    assert lib.da_combine(ctypes.byref(p), ctypes.byref(f), A, A, A, A + 8, A, None) == -1
    assert lib.da_decode_attention(ctypes.byref(p), ctypes.byref(f), A, A, A, A, A, A, A, A, A + 8, A, None) == -1
    assert lib.da_merge_partials_f32(2, 10, 128, A + 8, A, A, A, None) == -1
    assert lib.da_merge_partials_f32(2, 10, 96, A, A, A, A, None) == -2
    assert lib.da_merge_partials_f32(2, 0, 128, None, None, None, None, None) == 0


def test_host_step_checks(da_lib):
    """da_decode_step_host rejects bad arguments before it enqueues a copy (no pointer is dereferenced)."""
    import ctypes
    da = da_lib
    lib = da.lib()
    p = prob(da)
    d = da.da_plan_desc_init(p, da.PLAN_DYNAMIC, 64, 37)
    A = 1 << 12  # a 16-byte-aligned stand-in address, never touched: every case fails a check first

    def call(prob_=p, desc=d, ws_bytes=1 << 24, **kw):
        a = dict(q_host=A, bt_host=A, sl_host=A, k=A, v=A, ks=None, vs=None, q_dev=A, bt_dev=A, sl_dev=A, ws=A,
                 po=A, pl=A, out_dev=A, lse_dev=A, out_host=A, lse_host=A)
        a.update(kw)
        return lib.da_decode_step_host(ctypes.byref(prob_), ctypes.byref(desc), a["q_host"], a["bt_host"],
                                       a["sl_host"], a["k"], a["v"], a["ks"], a["vs"], a["q_dev"], a["bt_dev"],
                                       a["sl_dev"], a["ws"], ws_bytes, a["po"], a["pl"], a["out_dev"], a["lse_dev"],
                                       a["out_host"], a["lse_host"], None)

    for name in ("q_host", "bt_host", "sl_host", "out_host", "lse_host", "sl_dev", "ws", "q_dev", "bt_dev", "k",
                 "po", "pl", "out_dev", "lse_dev"):
        assert call(**{name: None}) == da.ERR_INVALID_ARG, name
    assert call(ks=A) == da.ERR_INVALID_ARG  # one scale without the other
    assert call(ws_bytes=64) == da.ERR_WORKSPACE
    assert call(ws=A + 8) == da.ERR_INVALID_ARG  # misaligned workspace
    assert call(k=A + 4) == da.ERR_INVALID_ARG  # misaligned cache
    p64 = prob(da, head_dim=64)
    d64 = da.da_plan_desc_init(p64, da.PLAN_DYNAMIC, 64, 37)
    assert call(prob_=p64, desc=d64, ks=A, vs=A) == da.ERR_UNSUPPORTED  # FP8 needs head_dim 128
    s = da.da_plan_desc_init(p, da.PLAN_STATIC, 64, 2)
    assert call(desc=s, ws_bytes=64) == da.ERR_WORKSPACE  # the static descriptor is checked the same way
    p0 = prob(da, batch=0)
    d0 = da.da_plan_desc_init(p0, da.PLAN_DYNAMIC, 64, 37)
    assert call(prob_=p0, desc=d0, q_host=None) == da.OK  # an empty batch enqueues nothing


def test_plan_append_checks(da_lib):
    """da_plan_append checks the plan's arguments and the append's before it launches anything."""
    import ctypes
    da = da_lib
    lib = da.lib()
    p = prob(da)
    d = da.da_plan_desc_init(p, da.PLAN_DYNAMIC, 64, 37)
    A = 1 << 12  # never dereferenced: every case below fails a check first

    def call(prob_=p, desc=d, ws_bytes=1 << 24, **kw):
        a = dict(sl=A, ws=A, nk=A, nv=A, bt=A, kc=A, vc=A, st=None)
        a.update(kw)
        return lib.da_plan_append(ctypes.byref(prob_), ctypes.byref(desc), a["sl"], a["ws"], ws_bytes, a["nk"],
                                  a["nv"], a["bt"], a["kc"], a["vc"], a["st"], None)

    for name in ("sl", "ws", "nk", "nv", "bt", "kc", "vc"):
        assert call(**{name: None}) == da.ERR_INVALID_ARG, name
    assert call(nk=A + 8) == da.ERR_INVALID_ARG  # rows are moved in 16-byte pieces
    assert call(st=A + 2) == da.ERR_INVALID_ARG
    assert call(ws_bytes=64) == da.ERR_WORKSPACE
    s = da.da_plan_desc_init(p, da.PLAN_STATIC, 64, 2)
    assert call(desc=s) == da.ERR_INVALID_ARG  # the fused launch builds the dynamic plan only
    assert call(prob_=prob(da, num_q_heads=60)) == da.ERR_INVALID_ARG


def test_every_launching_call_checks_before_it_enqueues(da_lib):
    """Null and misaligned arguments of each launching entry point come back as DA_ERR_INVALID_ARG
    (shapes it does not build as DA_ERR_UNSUPPORTED) before any CUDA call; an empty batch is a no-op."""
    import ctypes
    da = da_lib
    lib = da.lib()
    p = prob(da)
    d = da.da_plan_desc_init(p, da.PLAN_DYNAMIC, 64, 37)
    A = 1 << 12  # a 16-byte-aligned stand-in address that no check dereferences
    P, D = ctypes.byref(p), ctypes.byref(d)

    def decode(fp8=False, **kw):
        a = dict(q=A, k=A, v=A, ks=A, vs=A, bt=A, sl=A, ws=A, po=A, pl=A, out=A, lse=A)
        a.update(kw)
        if fp8:
            return lib.da_decode_attention_fp8(P, D, a["q"], a["k"], a["v"], a["ks"], a["vs"], a["bt"], a["sl"],
                                               a["ws"], a["po"], a["pl"], a["out"], a["lse"], None)
        return lib.da_decode_attention(P, D, a["q"], a["k"], a["v"], a["bt"], a["sl"], a["ws"], a["po"], a["pl"],
                                       a["out"], a["lse"], None)

    for name in ("q", "k", "v", "bt", "sl", "ws", "po", "pl", "out", "lse"):
        assert decode(**{name: None}) == da.ERR_INVALID_ARG, name
    for name, off in (("k", 8), ("v", 8), ("q", 2), ("out", 4), ("po", 8), ("ws", 8)):
        assert decode(**{name: A + off}) == da.ERR_INVALID_ARG, name
    assert decode(fp8=True, ks=None) == da.ERR_INVALID_ARG and decode(fp8=True, vs=None) == da.ERR_INVALID_ARG
    assert decode(fp8=True, q=A + 4) == da.ERR_INVALID_ARG  # the FP8 kernels read q in 8-byte pieces
    s = da.da_plan_desc_init(p, da.PLAN_STATIC, 64, 2)
    assert lib.da_static_plan(P, D, A, A, 1 << 24, None) == da.ERR_INVALID_ARG  # a dynamic descriptor
    assert lib.da_static_plan(P, ctypes.byref(s), A, A, 64, None) == da.ERR_WORKSPACE
    # append
    assert lib.da_append_kv(P, None, A, A, A, A, A, None, None) == da.ERR_INVALID_ARG
    assert lib.da_append_kv(P, A + 8, A, A, A, A, A, None, None) == da.ERR_INVALID_ARG
    assert lib.da_append_kv(P, A, A, A, A, A + 8, A, None, None) == da.ERR_INVALID_ARG
    p0 = prob(da, batch=0)
    assert lib.da_append_kv(ctypes.byref(p0), None, None, None, None, None, None, None, None) == da.OK
    # cross-GPU merge
    assert lib.da_merge_partials(0, 10, 128, A, A, A, A, None) == da.ERR_INVALID_ARG
    assert lib.da_merge_partials(2, -1, 128, A, A, A, A, None) == da.ERR_INVALID_ARG
    assert lib.da_merge_partials(2, 10, 96, A, A, A, A, None) == da.ERR_UNSUPPORTED
    assert lib.da_merge_partials(2, 0, 128, None, None, None, None, None) == da.OK
    assert lib.da_merge_partials(2, 10, 128, A, A, None, A, None) == da.ERR_INVALID_ARG
    assert lib.da_merge_partials(2, 10, 128, A + 4, A, A, A, None) == da.ERR_INVALID_ARG
    # the no-allocation step: shape, scratch size, pointers and alignment, all before the plan is enqueued
    def noalloc(prob_=p, width=37, **kw):
        a = dict(q=A, k=A, v=A, bt=A, sl=A, out=A, lse=A)
        a.update(kw)
        return lib.da_decode_step_noalloc(ctypes.byref(prob_), 64, width, a["q"], a["k"], a["v"], a["bt"], a["sl"],
                                          a["out"], a["lse"], None)
    assert noalloc(prob_=prob(da, head_dim=96)) == da.ERR_UNSUPPORTED
    assert noalloc(prob_=prob(da, batch=2000, num_pages=60000)) == da.ERR_WORKSPACE  # past the 16 MiB scratch
    for name in ("q", "k", "v", "bt", "sl", "out", "lse"):
        assert noalloc(**{name: None}) == da.ERR_INVALID_ARG, name
    for name, off in (("k", 8), ("v", 8), ("q", 2), ("out", 4)):
        assert noalloc(**{name: A + off}) == da.ERR_INVALID_ARG, name


def test_stall_switch_checks_its_limit(da_lib):
    """Only the argument check is exercised here: a valid call would arm the next decode launch."""
    da = da_lib
    for bad in (0, 2000001):
        with pytest.raises(da.DaError) as e:
            da.da_test_stall_next_decode(bad)
        assert e.value.code == da.ERR_INVALID_ARG


def test_status_strings(da_lib):
    da = da_lib
    assert da.status_string(0) == "ok" and "workspace" in da.status_string(-4)
    assert "length" in da.dev_status_string(1) and "page" in da.dev_status_string(2)
    assert "timed out" in da.dev_status_string(3) and "plan" in da.dev_status_string(4)
    assert "balance" in da.dev_status_string(5)


def test_balance_table_host_checks(da_lib):
    """Sizes and the checks of da_balance_set that come before any copy."""
    import ctypes
    import numpy as np
    da = da_lib
    d = da.da_plan_desc_init(prob(da), da.PLAN_DYNAMIC, 64, 37)
    assert d.balance is None and d.block_times is None
    assert da.da_balance_words(d) == 4 + 37 + 8 * 37
    good_w = np.full(37, 4096, np.int32)
    good_p = np.tile(np.arange(37, dtype=np.int32), (8, 1))
    fake = ctypes.c_void_p(1 << 20)  # never written: every call below is refused first
    L = da.lib()
    cases = [(np.zeros(37, np.int32), good_p), (np.full(37, 65537, np.int32), good_p)]
    dup = good_p.copy(); dup[3, 5] = dup[3, 6]
    neg = good_p.copy(); neg[0, 0] = -1
    cases += [(good_w, dup), (good_w, neg)]
    for w, p in cases:
        assert L.da_balance_set(ctypes.byref(d), w.ctypes.data, p.ctypes.data, fake, None) == da.ERR_INVALID_ARG
    s = da.da_plan_desc_init(prob(da), da.PLAN_STATIC, 64, 4)
    n = ctypes.c_size_t()
    assert L.da_balance_words(ctypes.byref(s), ctypes.byref(n)) == da.ERR_INVALID_ARG
    big = da.da_plan_desc_init(prob(da), da.PLAN_DYNAMIC, 64, 2049)
    assert L.da_balance_words(ctypes.byref(big), ctypes.byref(n)) == da.ERR_UNSUPPORTED
    # descriptors carrying a table: dynamic only, aligned, at most 2048 CTAs; block times 8-byte aligned
    for desc, field, val, code in [(s, "balance", 1 << 20, da.ERR_INVALID_ARG), (d, "balance", (1 << 20) + 2, da.ERR_INVALID_ARG),
                                   (big, "balance", 1 << 20, da.ERR_UNSUPPORTED),
                                   (d, "block_times", (1 << 20) + 4, da.ERR_INVALID_ARG)]:
        setattr(desc, field, val)
        sizes = (ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t())
        rc = L.da_workspace_size(ctypes.byref(prob(da)), ctypes.byref(desc), *map(ctypes.byref, sizes))
        assert rc == code, (field, val, rc)
        setattr(desc, field, None)


def test_balance_from_times(da_lib):
    """The table measured from block times: in each KV head's row the slowest block runs CTA 0;
    a CTA's weight follows the speed of its blocks; a block with no time counts at its row's
    median; the previous table's weights divide back out."""
    import numpy as np
    da = da_lib
    d = da.da_plan_desc_init(prob(da), da.PLAN_DYNAMIC, 64, 37)
    rng = np.random.default_rng(4)
    dur = rng.uniform(90, 110, size=(8, 37))
    t = np.zeros((8, 37, 2), np.int64)
    t[:, :, 0] = 1000
    t[:, :, 1] = 1000 + np.round(dur * 1000).astype(np.int64)
    w, p = da.da_balance_from_times(d, t)
    for g in range(8):
        assert sorted(p[g]) == list(range(37))
        ns = t[g, :, 1] - t[g, :, 0]
        assert list(np.argsort(p[g])) == list(np.argsort(-ns, kind="stable"))  # slowest first
    assert np.all(np.diff(w) >= 0)  # CTA c runs on the c-th slowest blocks: weights rise with c
    speed = np.sort(1.0 / dur, axis=1).mean(axis=0)
    np.testing.assert_allclose(w / w.mean(), speed / speed.mean(), rtol=2e-3)
    assert abs(w.mean() - 4096) < 2
    # a block without a usable time: the row's median speed
    t2 = t.copy()
    t2[2, 5, 1] = t2[2, 5, 0]
    w2, p2 = da.da_balance_from_times(d, t2)
    assert sorted(p2[2]) == list(range(37))
    # measured with a table in use: the same times under twice the work per CTA give twice the speed
    w3, p3 = da.da_balance_from_times(d, t, np.full(37, 2, np.int32), np.tile(np.arange(37, dtype=np.int32), (8, 1)))
    assert np.array_equal(p3, p) and np.allclose(w3, w, atol=1)
    # a previous table must be whole and valid
    import ctypes
    L = da.lib()
    out_w, out_p = np.zeros(37, np.int32), np.zeros((8, 37), np.int32)
    ident = np.tile(np.arange(37, dtype=np.int32), (8, 1))
    bad = ident.copy(); bad[4, 0] = 36
    for pw, pp in [(np.full(37, 2, np.int32), None), (np.full(37, 0, np.int32), ident), (np.full(37, 2, np.int32), bad)]:
        rc = L.da_balance_from_times(ctypes.byref(d), t.ctypes.data, None if pw is None else pw.ctypes.data,
                                     None if pp is None else pp.ctypes.data, out_w.ctypes.data, out_p.ctypes.data)
        assert rc == da.ERR_INVALID_ARG


@pytest.mark.skipif(cuda_available(), reason="checks the no-device error path")
def test_default_width_needs_a_device(da_lib):
    da = da_lib
    with pytest.raises(da.DaError) as e:
        da.da_plan_desc_init(prob(da), da.PLAN_DYNAMIC, 64, 0)
    assert e.value.code == da.ERR_CUDA and e.value.cuda_error != 0


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    from variable_length_paged_b200 import da
    monkeypatch.setattr(da, "_lib", None)
    monkeypatch.setattr(da, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="libda.so not found"):
        da.lib()
