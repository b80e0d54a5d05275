"""CPU oracle for split-KV decode attention over a paged, variable-length KV cache.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package.  The product path (the
CUDA library in ``variable_length_paged_b200``) never imports, links or runs it,
and the two share no code.

The arithmetic lives in ``dao.c`` (plain C, fp64, one loop per definition);
this module only builds it with gcc and marshals numpy arrays through ctypes.
Source of the method: "Tencent HPC lands in SGLang, challenging default
inference kernels", section "Why Tencent HPC matters for online model
serving" (uneven decode work over the KV cache, uniform tiles handed to CTAs by
the current workload, a static split-k schedule as the baseline).  Every
function here is pinned by tests that do not reuse its formula (closed forms,
invariants, brute force, library routines); see ``tests/test_oracle_*.py``.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dao.c")
_LIB = os.path.join(_HERE, "libdao.so")
_lock = threading.Lock()
_lib = None

OK = 0
ERR_ARG = -1
ERR_BAD_SEQLEN = -2
ERR_BAD_PAGE = -3
ERR_CAPACITY = -4

_i32p = ctypes.POINTER(ctypes.c_int32)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_f64p = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile ``dao.c`` into ``libdao.so`` next to it (gcc, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-shared", "-fPIC",
             "-std=c11", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _bind(path: str):
    """Open a compiled copy of dao.c and declare its signatures."""
    lib = ctypes.CDLL(path)
    lib.dao_attention.restype = ctypes.c_int
    lib.dao_attention.argtypes = [
        ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
        ctypes.c_int32, ctypes.c_int64, ctypes.c_double, _u16p, _u16p, _u16p, _i32p, _i32p,
        ctypes.c_int64, _i32p, _i32p, _f64p, _f64p, ctypes.c_int32]
    lib.dao_combine.restype = ctypes.c_int
    lib.dao_combine.argtypes = [ctypes.c_int32, ctypes.c_int32, _f64p, _f64p, _f64p, _f64p]
    plan_args = [ctypes.c_int32, _i32p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int64,
                 ctypes.c_int32, _i32p, _i32p, _i32p, _i32p, _i32p, _i32p, _i32p, _i32p,
                 _i32p, _i32p]
    lib.dao_plan.restype = ctypes.c_int
    lib.dao_plan.argtypes = plan_args
    lib.dao_plan_start_cost.restype = ctypes.c_int
    lib.dao_plan_start_cost.argtypes = plan_args + [ctypes.c_int32]
    lib.dao_plan_weighted.restype = ctypes.c_int
    lib.dao_plan_weighted.argtypes = plan_args + [ctypes.c_int32, ctypes.POINTER(ctypes.c_int32)]
    lib.dao_static_plan.restype = ctypes.c_int
    lib.dao_static_plan.argtypes = plan_args
    lib.dao_num_threads.restype = ctypes.c_int
    lib.dao_num_threads.argtypes = []
    lib.dao_attention_fp8.restype = ctypes.c_int
    lib.dao_attention_fp8.argtypes = [
        ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
        ctypes.c_int32, ctypes.c_int64, ctypes.c_double, _u16p, _u8p, _u8p, _f64p, _f64p, _i32p, _i32p,
        ctypes.c_int64, _i32p, _i32p, _f64p, _f64p, ctypes.c_int32]
    lib.dao_attention_mq.restype = ctypes.c_int
    lib.dao_attention_mq.argtypes = [
        ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
        ctypes.c_int32, ctypes.c_int64, ctypes.c_double, _u16p, _u16p, _u16p, _i32p, _i32p, _f64p, _f64p,
        ctypes.c_int32]
    lib.dao_e4m3_value.restype = ctypes.c_double
    lib.dao_e4m3_value.argtypes = [ctypes.c_uint8]
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(build())
    return _lib


def compile_variant(src_text: str, path: str) -> str:
    """Compile a modified copy of dao.c (used by the tests that check the pins catch planted mistakes)."""
    c_path = path[:-3] + ".c"
    with open(c_path, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-shared", "-fPIC",
                           "-std=c11", c_path, "-o", path, "-lm"])
    return path


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _u16(a) -> np.ndarray:
    """bf16 data as its raw 16-bit patterns (numpy uint16, C-contiguous)."""
    if hasattr(a, "view") and hasattr(a, "dtype") and str(a.dtype) == "torch.bfloat16":
        import torch  # only for the dtype reinterpretation of CPU tensors
        a = a.contiguous().view(torch.int16).numpy()
    a = np.ascontiguousarray(a)
    if a.dtype == np.int16:
        a = a.view(np.uint16)
    if a.dtype != np.uint16:
        raise TypeError("bf16 inputs must be torch.bfloat16 CPU tensors or uint16 bit arrays")
    return a


def num_threads(lib=None) -> int:
    return int((lib or _load()).dao_num_threads())


def attention(q, k_cache, v_cache, block_table, seq_lens, *, scale: float, num_pages: int | None = None,
              pairs=None, threads: int = 0, lib=None):
    """fp64 decode attention.

    q: bf16 [B, Hq, d]; k_cache, v_cache: bf16 [num_pages, Hkv, P, d];
    block_table: int32 [B, max_pages]; seq_lens: int32 [B].
    pairs: optional (b_idx, h_idx) int arrays selecting (request, head) pairs.
    Returns (out fp64 [n, d], lse fp64 [n], status) with n = len(pairs) or B*Hq
    (then out is reshaped to [B, Hq, d] and lse to [B, Hq]).
    """
    lib = lib or _load()
    q16, k16, v16 = _u16(q), _u16(k_cache), _u16(v_cache)
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B, Hq, d = q16.shape
    n_pages, Hkv, P, d2 = k16.shape
    assert d2 == d and v16.shape == k16.shape and bt.shape[0] == B and sl.shape == (B,)
    max_pages = bt.shape[1] if bt.ndim == 2 else 0
    if num_pages is None:
        num_pages = n_pages
    if pairs is None:
        n = B * Hq
        pb = ph = None
    else:
        pb = np.ascontiguousarray(pairs[0], dtype=np.int32)
        ph = np.ascontiguousarray(pairs[1], dtype=np.int32)
        n = pb.shape[0]
    out = np.empty((n, d), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    st = lib.dao_attention(B, Hq, Hkv, d, P, max_pages, num_pages, float(scale), _ptr(q16, ctypes.c_uint16),
                           _ptr(k16, ctypes.c_uint16), _ptr(v16, ctypes.c_uint16), _ptr(bt, ctypes.c_int32),
                           _ptr(sl, ctypes.c_int32), n,
                           None if pb is None else _ptr(pb, ctypes.c_int32),
                           None if ph is None else _ptr(ph, ctypes.c_int32),
                           _ptr(out, ctypes.c_double), _ptr(lse, ctypes.c_double), int(threads))
    if pairs is None:
        out = out.reshape(B, Hq, d)
        lse = lse.reshape(B, Hq)
    return out, lse, int(st)


def attention_mq(q, k_cache, v_cache, block_table, seq_lens, *, scale: float, threads: int = 0, lib=None):
    """fp64 multi-query decode: q bf16 [B, Q, Hq, d], the Q queries being the last Q cached tokens;
    query i attends causally to tokens [0, L_b - Q + i].  Returns (out [B, Q, Hq, d], lse [B, Q, Hq], status)."""
    lib = lib or _load()
    q16, k16, v16 = _u16(q), _u16(k_cache), _u16(v_cache)
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B, Q, Hq, d = q16.shape
    n_pages, Hkv, P, d2 = k16.shape
    assert d2 == d and v16.shape == k16.shape and bt.shape[0] == B and sl.shape == (B,)
    out = np.empty((B, Q, Hq, d), dtype=np.float64)
    lse = np.empty((B, Q, Hq), dtype=np.float64)
    st = lib.dao_attention_mq(B, Q, Hq, Hkv, d, P, bt.shape[1], n_pages, float(scale), _ptr(q16, ctypes.c_uint16),
                              _ptr(k16, ctypes.c_uint16), _ptr(v16, ctypes.c_uint16), _ptr(bt, ctypes.c_int32),
                              _ptr(sl, ctypes.c_int32), _ptr(out, ctypes.c_double), _ptr(lse, ctypes.c_double),
                              int(threads))
    return out, lse, int(st)


def _u8(a) -> np.ndarray:
    """FP8 codes as raw bytes (numpy uint8, C-contiguous)."""
    if hasattr(a, "dtype") and str(a.dtype).startswith("torch."):
        import torch  # only for the dtype reinterpretation of CPU tensors
        a = a.contiguous().view(torch.uint8).numpy()
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint8:
        raise TypeError("fp8 caches must be torch.float8_e4m3fn / uint8 CPU tensors or uint8 arrays")
    return a


def e4m3_value(code: int, lib=None) -> float:
    """The real number an FP8 E4M3 code stands for (NaN for the NaN codes)."""
    return float((lib or _load()).dao_e4m3_value(int(code)))


def attention_fp8(q, k_code, v_code, k_scale, v_scale, block_table, seq_lens, *, scale: float, pairs=None,
                  threads: int = 0, lib=None):
    """fp64 decode attention over an FP8 E4M3 cache with per-KV-head scales (k = k_scale[g] * e4m3(code)).

    Same shapes and results as ``attention``; k_code, v_code are [num_pages, Hkv, P, d] bytes and
    k_scale, v_scale fp64 [Hkv].
    """
    lib = lib or _load()
    q16, k8, v8 = _u16(q), _u8(k_code), _u8(v_code)
    ks = np.ascontiguousarray(k_scale, dtype=np.float64)
    vs = np.ascontiguousarray(v_scale, dtype=np.float64)
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B, Hq, d = q16.shape
    n_pages, Hkv, P, d2 = k8.shape
    assert d2 == d and v8.shape == k8.shape and ks.shape == (Hkv,) and vs.shape == (Hkv,)
    if pairs is None:
        n, pb, ph = B * Hq, None, None
    else:
        pb = np.ascontiguousarray(pairs[0], dtype=np.int32)
        ph = np.ascontiguousarray(pairs[1], dtype=np.int32)
        n = pb.shape[0]
    out = np.empty((n, d), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    st = lib.dao_attention_fp8(B, Hq, Hkv, d, P, bt.shape[1], n_pages, float(scale), _ptr(q16, ctypes.c_uint16),
                               _ptr(k8, ctypes.c_uint8), _ptr(v8, ctypes.c_uint8), _ptr(ks, ctypes.c_double),
                               _ptr(vs, ctypes.c_double), _ptr(bt, ctypes.c_int32), _ptr(sl, ctypes.c_int32), n,
                               None if pb is None else _ptr(pb, ctypes.c_int32),
                               None if ph is None else _ptr(ph, ctypes.c_int32),
                               _ptr(out, ctypes.c_double), _ptr(lse, ctypes.c_double), int(threads))
    if pairs is None:
        out = out.reshape(B, Hq, d)
        lse = lse.reshape(B, Hq)
    return out, lse, int(st)


def combine(o_parts, lse_parts, lib=None):
    """fp64 log-sum-exp merge of n partials o_parts [n, d], lse_parts [n] -> (out [d], lse)."""
    lib = lib or _load()
    o = np.ascontiguousarray(o_parts, dtype=np.float64)
    l = np.ascontiguousarray(lse_parts, dtype=np.float64)
    n, d = o.shape
    out = np.empty((d,), dtype=np.float64)
    lse = np.empty((1,), dtype=np.float64)
    st = lib.dao_combine(n, d, _ptr(o, ctypes.c_double), _ptr(l, ctypes.c_double),
                         _ptr(out, ctypes.c_double), _ptr(lse, ctypes.c_double))
    assert st == OK
    return out, float(lse[0])


def _run_plan(fn, seq_lens, tile_tokens, width, capacity_tokens, max_segments, num_ctas, *extra):
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B = sl.shape[0]
    arr = lambda n: np.zeros((n,), dtype=np.int32)
    res = dict(req_tile_prefix=arr(B + 1), req_seg_begin=arr(B + 1), cta_seg_begin=arr(num_ctas + 1),
               seg_req=arr(max_segments), seg_cta=arr(max_segments), seg_tile_begin=arr(max_segments),
               seg_tile_end=arr(max_segments))
    nu, ns, bad = (ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32())
    st = fn(B, _ptr(sl, ctypes.c_int32), int(tile_tokens), int(width), int(capacity_tokens), int(max_segments),
            ctypes.byref(nu), ctypes.byref(ns), *[_ptr(res[k], ctypes.c_int32) for k in
                                                   ("req_tile_prefix", "req_seg_begin", "cta_seg_begin", "seg_req",
                                                    "seg_cta", "seg_tile_begin", "seg_tile_end")],
            ctypes.byref(bad), *extra)
    if st not in (OK, ERR_BAD_SEQLEN):
        raise ValueError(f"oracle plan failed with status {st}")
    S = ns.value
    for k in ("seg_req", "seg_cta", "seg_tile_begin", "seg_tile_end"):
        res[k] = res[k][:S].copy()
    res.update(num_units=nu.value, num_segments=S, num_ctas=num_ctas, tile_tokens=int(tile_tokens),
               bad_index=bad.value, status=st)
    return res


def plan(seq_lens, tile_tokens: int, num_ctas: int, capacity_tokens: int, lib=None, start_cost: int = 0,
         weights=None):
    """Dynamic plan (dict of int32 arrays; see ``dao_plan_weighted`` in dao.c).

    start_cost: start units charged to every non-empty request (0: every unit is a tile).
    weights: per-CTA weights in [1, 65536] (None: the even split)."""
    B = len(seq_lens)
    lib = lib or _load()
    if weights is not None:
        w = np.ascontiguousarray(weights, dtype=np.int32)
        assert w.shape == (num_ctas,)
        return _run_plan(lib.dao_plan_weighted, seq_lens, tile_tokens, num_ctas, capacity_tokens,
                         num_ctas + max(B, 1) - 1, num_ctas, int(start_cost), _ptr(w, ctypes.c_int32))
    if start_cost == 0:
        return _run_plan(lib.dao_plan, seq_lens, tile_tokens, num_ctas, capacity_tokens, num_ctas + max(B, 1) - 1,
                         num_ctas)
    return _run_plan(lib.dao_plan_start_cost, seq_lens, tile_tokens, num_ctas, capacity_tokens,
                     num_ctas + max(B, 1) - 1, num_ctas, int(start_cost))


def static_plan(seq_lens, tile_tokens: int, splits: int, capacity_tokens: int, lib=None):
    """Static split-k plan (same dict layout; num_ctas = B * splits)."""
    B = len(seq_lens)
    return _run_plan((lib or _load()).dao_static_plan, seq_lens, tile_tokens, splits, capacity_tokens,
                     max(B * splits, 1), B * splits)
