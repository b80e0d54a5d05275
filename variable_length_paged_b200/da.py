"""Thin ctypes binding of libda.so (C ABI in include/da.h).

Functions keep the C names and only marshal arguments: torch tensors (device
memory) become raw pointers, the current torch CUDA stream becomes the
cudaStream_t.  Every step of the computation runs in the library's kernels;
there is no Python or CPU fallback, and a missing library raises.
"""

from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# DA_LIB_PATH selects another build of the library (one made with `build --define ... --out`)
LIB_PATH = os.environ.get("DA_LIB_PATH") or os.path.join(HERE, "libda.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_WORKSPACE = 0, -1, -2, -3, -4
DEV_OK, DEV_BAD_SEQLEN, DEV_BAD_PAGE, DEV_TIMEOUT, DEV_BAD_PLAN, DEV_BAD_BALANCE = 0, 1, 2, 3, 4, 5
PLAN_DYNAMIC, PLAN_STATIC = 0, 1
OUT_BF16, OUT_F32 = 0, 1

# Every symbol include/da.h declares.
EXPORTS = ("da_plan_desc_init", "da_workspace_size", "da_workspace_offsets", "da_plan", "da_static_plan",
           "da_decode_attention", "da_combine", "da_read_status", "da_status_string", "da_dev_status_string",
           "da_last_cuda_error", "da_device_num_sms", "da_decode_step_noalloc", "da_append_kv",
           "da_decode_attention_fp8", "da_merge_partials", "da_decode_step_host", "da_test_stall_next_decode",
           "da_plan_append", "da_plan_workspace_size", "da_noalloc_read_status",
           "da_merge_partials_f32", "da_decode_step", "da_balance_words", "da_balance_set",
           "da_balance_from_times")

NOALLOC_SCRATCH_BYTES = 16 << 20  # DA_NOALLOC_SCRATCH_BYTES


class DaProblem(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("page_size", ctypes.c_int32), ("max_pages_per_req", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("scale", ctypes.c_float), ("q_len", ctypes.c_int32)]


class DaPlanDesc(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("batch", ctypes.c_int32), ("tile_tokens", ctypes.c_int32),
                ("num_ctas", ctypes.c_int32), ("splits", ctypes.c_int32), ("max_segments", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("merge_in_decode", ctypes.c_int32),
                ("out_format", ctypes.c_int32), ("start_cost", ctypes.c_int32),
                ("balance", ctypes.c_void_p), ("block_times", ctypes.c_void_p)]


class DaError(RuntimeError):
    def __init__(self, fn: str, code: int, cuda_error: int = 0):
        self.code = code
        self.cuda_error = cuda_error
        msg = f"{fn} returned {code} ({status_string(code)})"
        if code == ERR_CUDA:
            msg += f", cudaError {cuda_error}"
        super().__init__(msg)


_lib = None
_vp = ctypes.c_void_p
_sz = ctypes.c_size_t


def lib():
    """Load libda.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libda.so not found at {LIB_PATH}; build it with "
                               "`python -m variable_length_paged_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, D = ctypes.POINTER(DaProblem), ctypes.POINTER(DaPlanDesc)
        sig = {
            "da_plan_desc_init": [P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, D],
            "da_workspace_size": [P, D, ctypes.POINTER(_sz), ctypes.POINTER(_sz), ctypes.POINTER(_sz)],
            "da_workspace_offsets": [D, ctypes.POINTER(ctypes.c_int64)],
            "da_plan_workspace_size": [P, ctypes.c_int32, ctypes.c_int32, ctypes.POINTER(_sz), ctypes.POINTER(_sz),
                                       ctypes.POINTER(_sz)],
            "da_noalloc_read_status": [ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32), _vp],
            "da_plan": [P, D, _vp, _vp, _sz, _vp],
            "da_static_plan": [P, D, _vp, _vp, _sz, _vp],
            "da_decode_attention": [P, D, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp],
            "da_combine": [P, D, _vp, _vp, _vp, _vp, _vp, _vp],
            "da_read_status": [_vp, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32), _vp],
            "da_last_cuda_error": [],
            "da_device_num_sms": [ctypes.POINTER(ctypes.c_int32)],
            "da_decode_step_noalloc": [P, ctypes.c_int32, ctypes.c_int32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp],
            "da_append_kv": [P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp],
            "da_merge_partials": [ctypes.c_int32, ctypes.c_int64, ctypes.c_int32, _vp, _vp, _vp, _vp, _vp],
            "da_merge_partials_f32": [ctypes.c_int32, ctypes.c_int64, ctypes.c_int32, _vp, _vp, _vp, _vp, _vp],
            "da_decode_attention_fp8": [P, D, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp],
            "da_decode_step": [P, D, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp, _vp, _vp, _vp, _vp],
            "da_test_stall_next_decode": [ctypes.c_uint32],
            "da_plan_append": [P, D, _vp, _vp, _sz, _vp, _vp, _vp, _vp, _vp, _vp, _vp],
            "da_decode_step_host": [P, D, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp, _vp, _vp,
                                    _vp, _vp, _vp, _vp],
            "da_balance_words": [D, ctypes.POINTER(_sz)],
            "da_balance_set": [D, _vp, _vp, _vp, _vp],
            "da_balance_from_times": [D, _vp, _vp, _vp, _vp, _vp],
        }
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int32
        for name in ("da_status_string", "da_dev_status_string"):
            fn = getattr(L, name)
            fn.argtypes = [ctypes.c_int32]
            fn.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().da_status_string(int(code)).decode()


def dev_status_string(code: int) -> str:
    return lib().da_dev_status_string(int(code)).decode()


def _check(fn: str, rc: int):
    if rc != OK:
        raise DaError(fn, rc, lib().da_last_cuda_error() if rc == ERR_CUDA else 0)


def problem(batch, num_q_heads, num_kv_heads, head_dim, page_size, max_pages_per_req, num_pages, scale,
            q_len: int = 1) -> DaProblem:
    return DaProblem(int(batch), int(num_q_heads), int(num_kv_heads), int(head_dim), int(page_size),
                     int(max_pages_per_req), int(num_pages), float(scale), int(q_len))


def problem_from(p) -> DaProblem:
    """From any object with the da_problem field names (e.g. workloads.Problem)."""
    return problem(p.batch, p.num_q_heads, p.num_kv_heads, p.head_dim, p.page_size, p.max_pages_per_req,
                   p.num_pages, p.scale, getattr(p, "q_len", 1))


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


# ---- the C calls -------------------------------------------------------------------------------

def da_plan_desc_init(prob: DaProblem, kind: int, tile_tokens: int = 0, width: int = 0,
                      merge_in_decode: bool = False, out_f32: bool = False,
                      start_cost: int | None = None) -> DaPlanDesc:
    """The C call, then the descriptor's switches set as asked: in-decode merge, fp32 output and
    the dynamic plan's start cost (None keeps the C default)."""
    d = DaPlanDesc()
    _check("da_plan_desc_init", lib().da_plan_desc_init(ctypes.byref(prob), int(kind), int(tile_tokens), int(width),
                                                         ctypes.byref(d)))
    d.merge_in_decode = 1 if merge_in_decode else 0
    d.out_format = OUT_F32 if out_f32 else OUT_BF16
    if start_cost is not None:
        d.start_cost = int(start_cost)
    return d


def da_workspace_size(prob: DaProblem, desc: DaPlanDesc) -> tuple[int, int, int]:
    a, b, c = _sz(), _sz(), _sz()
    _check("da_workspace_size", lib().da_workspace_size(ctypes.byref(prob), ctypes.byref(desc), ctypes.byref(a),
                                                         ctypes.byref(b), ctypes.byref(c)))
    return a.value, b.value, c.value


def da_plan_workspace_size(prob: DaProblem, tile_tokens: int = 0, num_ctas: int = 0) -> tuple[int, int, int]:
    a, b, c = _sz(), _sz(), _sz()
    _check("da_plan_workspace_size", lib().da_plan_workspace_size(
        ctypes.byref(prob), int(tile_tokens), int(num_ctas), ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)))
    return a.value, b.value, c.value


def da_workspace_offsets(desc: DaPlanDesc) -> list[int]:
    off = (ctypes.c_int64 * 7)()
    _check("da_workspace_offsets", lib().da_workspace_offsets(ctypes.byref(desc), off))
    return list(off)


def da_plan(prob, desc, seq_lens, ws, ws_bytes: int | None = None, stream=None):
    nbytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    _check("da_plan", lib().da_plan(ctypes.byref(prob), ctypes.byref(desc), _ptr(seq_lens), _ptr(ws), nbytes,
                                    _stream(stream)))


def da_static_plan(prob, desc, seq_lens, ws, ws_bytes: int | None = None, stream=None):
    nbytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    _check("da_static_plan", lib().da_static_plan(ctypes.byref(prob), ctypes.byref(desc), _ptr(seq_lens), _ptr(ws),
                                                  nbytes, _stream(stream)))


def da_decode_attention(prob, desc, q, k_cache, v_cache, block_table, seq_lens, ws, partial_o, partial_lse, out, lse,
                        stream=None):
    _check("da_decode_attention", lib().da_decode_attention(
        ctypes.byref(prob), ctypes.byref(desc), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
        _ptr(seq_lens), _ptr(ws), _ptr(partial_o), _ptr(partial_lse), _ptr(out), _ptr(lse), _stream(stream)))


def da_decode_attention_fp8(prob, desc, q, k_cache, v_cache, k_scale, v_scale, block_table, seq_lens, ws, partial_o,
                            partial_lse, out, lse, stream=None):
    _check("da_decode_attention_fp8", lib().da_decode_attention_fp8(
        ctypes.byref(prob), ctypes.byref(desc), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale),
        _ptr(block_table), _ptr(seq_lens), _ptr(ws), _ptr(partial_o), _ptr(partial_lse), _ptr(out), _ptr(lse),
        _stream(stream)))


def da_decode_step(prob, desc, q, k_cache, v_cache, block_table, seq_lens, bufs: "Buffers", k_scale=None, v_scale=None,
                   stream=None):
    """Plan + decode + combine in one C call (the decode may start on its first chunks before the plan lands)."""
    _check("da_decode_step", lib().da_decode_step(
        ctypes.byref(prob), ctypes.byref(desc), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale),
        _ptr(block_table), _ptr(seq_lens), _ptr(bufs.ws), bufs.ws.numel() * bufs.ws.element_size(),
        _ptr(bufs.partial_o), _ptr(bufs.partial_lse), _ptr(bufs.out), _ptr(bufs.lse), _stream(stream)))


def da_combine(prob, desc, ws, partial_o, partial_lse, out, lse, stream=None):
    _check("da_combine", lib().da_combine(ctypes.byref(prob), ctypes.byref(desc), _ptr(ws), _ptr(partial_o),
                                          _ptr(partial_lse), _ptr(out), _ptr(lse), _stream(stream)))


def da_decode_step_host(prob, desc, q_host, block_table_host, seq_lens_host, k_cache, v_cache, q_dev,
                        block_table_dev, seq_lens_dev, bufs: "Buffers", out_host, lse_host, k_scale=None, v_scale=None,
                        stream=None):
    """Whole step from host inputs to host outputs in one C call (copies in, plan, decode, combine, copies out).

    Asynchronous: `out_host` / `lse_host` are valid after the stream is synchronised."""
    _check("da_decode_step_host", lib().da_decode_step_host(
        ctypes.byref(prob), ctypes.byref(desc), _ptr(q_host), _ptr(block_table_host), _ptr(seq_lens_host),
        _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale), _ptr(q_dev), _ptr(block_table_dev),
        _ptr(seq_lens_dev), _ptr(bufs.ws), bufs.ws.numel() * bufs.ws.element_size(), _ptr(bufs.partial_o),
        _ptr(bufs.partial_lse), _ptr(bufs.out), _ptr(bufs.lse), _ptr(out_host), _ptr(lse_host), _stream(stream)))


def da_append_kv(prob, new_k, new_v, block_table, seq_lens, k_cache, v_cache, status=None, stream=None):
    _check("da_append_kv", lib().da_append_kv(ctypes.byref(prob), _ptr(new_k), _ptr(new_v), _ptr(block_table),
                                              _ptr(seq_lens), _ptr(k_cache), _ptr(v_cache), _ptr(status),
                                              _stream(stream)))


def da_plan_append(prob, desc, seq_lens, ws, new_k, new_v, block_table, k_cache, v_cache, status=None,
                   ws_bytes: int | None = None, stream=None):
    """da_append_kv + da_plan in one launch (block 0 plans, the other blocks append)."""
    nbytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    _check("da_plan_append", lib().da_plan_append(
        ctypes.byref(prob), ctypes.byref(desc), _ptr(seq_lens), _ptr(ws), nbytes, _ptr(new_k), _ptr(new_v),
        _ptr(block_table), _ptr(k_cache), _ptr(v_cache), _ptr(status), _stream(stream)))


def da_merge_partials(part_out, part_lse, out, lse, stream=None):
    """part_out [n, ..., d] bf16 and part_lse [n, ...] fp32 -> out [..., d], lse [...]."""
    n = part_out.shape[0]
    rows = lse.numel()
    _check("da_merge_partials", lib().da_merge_partials(int(n), int(rows), int(part_out.shape[-1]), _ptr(part_out),
                                                        _ptr(part_lse), _ptr(out), _ptr(lse), _stream(stream)))


def da_merge_partials_f32(part_out, part_lse, out, lse, stream=None):
    """part_out [n, ..., d] fp32 (steps run with fp32 output) and part_lse [n, ...] -> out bf16, lse."""
    n = part_out.shape[0]
    rows = lse.numel()
    _check("da_merge_partials_f32", lib().da_merge_partials_f32(int(n), int(rows), int(part_out.shape[-1]),
                                                                _ptr(part_out), _ptr(part_lse), _ptr(out), _ptr(lse),
                                                                _stream(stream)))


def da_read_status(ws, stream=None) -> tuple[int, int]:
    st, bad = ctypes.c_int32(), ctypes.c_int32()
    _check("da_read_status", lib().da_read_status(_ptr(ws), ctypes.byref(st), ctypes.byref(bad), _stream(stream)))
    return st.value, bad.value


def da_test_stall_next_decode(wait_limit_us: int):
    """Failure-path test: the next decode launch on this thread waits for K/V that never come
    and gives up after `wait_limit_us` (status DA_DEV_TIMEOUT); see include/da.h."""
    _check("da_test_stall_next_decode", lib().da_test_stall_next_decode(int(wait_limit_us)))


def da_device_num_sms() -> int:
    n = ctypes.c_int32()
    _check("da_device_num_sms", lib().da_device_num_sms(ctypes.byref(n)))
    return n.value


def da_decode_step_noalloc(prob, q, k_cache, v_cache, block_table, seq_lens, out, lse, tile_tokens: int = 0,
                           num_ctas: int = 0, stream=None):
    """Whole step on the library's static scratch (for callers that cannot allocate; see include/da.h)."""
    _check("da_decode_step_noalloc", lib().da_decode_step_noalloc(
        ctypes.byref(prob), int(tile_tokens), int(num_ctas), _ptr(q), _ptr(k_cache), _ptr(v_cache),
        _ptr(block_table), _ptr(seq_lens), _ptr(out), _ptr(lse), _stream(stream)))


def da_noalloc_read_status(stream=None) -> tuple[int, int]:
    """Status word and first bad index of the last da_decode_step_noalloc on this device (syncs `stream`)."""
    st, bad = ctypes.c_int32(), ctypes.c_int32()
    _check("da_noalloc_read_status", lib().da_noalloc_read_status(ctypes.byref(st), ctypes.byref(bad),
                                                                   _stream(stream)))
    return st.value, bad.value


def da_balance_words(desc: DaPlanDesc) -> int:
    n = _sz()
    _check("da_balance_words", lib().da_balance_words(ctypes.byref(desc), ctypes.byref(n)))
    return n.value


def da_balance_set(desc: DaPlanDesc, weights, perm, table, stream=None):
    """Check (weights [C], perm [Hkv][C], host int32 arrays) and copy them into the device table."""
    import numpy as np
    w = np.ascontiguousarray(weights, dtype=np.int32)
    p = np.ascontiguousarray(perm, dtype=np.int32)
    _check("da_balance_set", lib().da_balance_set(ctypes.byref(desc), w.ctypes.data, p.ctypes.data, _ptr(table),
                                                  _stream(stream)))


def da_balance_from_times(desc: DaPlanDesc, times, prev_weights=None, prev_perm=None):
    """(weights, perm) from block times [Hkv][C][2] (host int64), measured with the previous
    table in use (None: even split, identity placement)."""
    import numpy as np
    C, H = desc.num_ctas, desc.num_kv_heads
    t = np.ascontiguousarray(times, dtype=np.int64)
    assert t.size == 2 * C * H
    pw = None if prev_weights is None else np.ascontiguousarray(prev_weights, dtype=np.int32)
    pp = None if prev_perm is None else np.ascontiguousarray(prev_perm, dtype=np.int32)
    w = np.zeros(C, np.int32)
    p = np.zeros((H, C), np.int32)
    _check("da_balance_from_times", lib().da_balance_from_times(
        ctypes.byref(desc), t.ctypes.data, None if pw is None else pw.ctypes.data,
        None if pp is None else pp.ctypes.data, w.ctypes.data, p.ctypes.data))
    return w, p


def calibrate_balance(desc: DaPlanDesc, run_step, device, rounds: int = 2, steps: int = 9, stream=None):
    """Measure a balance table for `desc` and install it (sets desc.balance; returns the device
    table, which must outlive the descriptor's use).  run_step(desc) enqueues one step with the
    descriptor it is given.  Each round runs `steps` steps with block times, takes every block's
    median start and end, and refines the table from them."""
    import numpy as np
    import torch
    C, H = desc.num_ctas, desc.num_kv_heads
    table = torch.zeros(da_balance_words(desc), dtype=torch.int32, device=device)
    times = torch.zeros((steps, H, C, 2), dtype=torch.int64, device=device)
    w = p = None
    for _ in range(rounds):
        for k in range(steps):
            desc.block_times = times[k].data_ptr()
            run_step(desc)
        desc.block_times = None
        torch.cuda.synchronize()
        t = times.cpu().numpy()
        med = np.median(t - t[:, :, :, :1].min(axis=(1, 2, 3), keepdims=True), axis=0).astype(np.int64)
        w, p = da_balance_from_times(desc, med, w, p)
        da_balance_set(desc, w, p, table, stream=stream)
        if stream is None:
            torch.cuda.synchronize()
        desc.balance = table.data_ptr()
    return table


# ---- buffers and one whole step --------------------------------------------------------------------

class Buffers:
    """Device buffers for one plan descriptor: workspace, partials, outputs (allocated with torch)."""

    def __init__(self, prob: DaProblem, desc: DaPlanDesc, device):
        import torch
        ws, po, pl = da_workspace_size(prob, desc)
        self.ws = torch.zeros(max(ws // 4, 4), dtype=torch.int32, device=device)
        self.partial_o = torch.empty(max(po // 4, 4), dtype=torch.float32, device=device)
        self.partial_lse = torch.empty(max(pl // 4, 1), dtype=torch.float32, device=device)
        lead = (prob.batch,) if prob.q_len <= 1 else (prob.batch, prob.q_len)
        out_dtype = torch.float32 if desc.out_format == OUT_F32 else torch.bfloat16
        self.out = torch.empty(lead + (prob.num_q_heads, prob.head_dim), dtype=out_dtype, device=device)
        self.lse = torch.empty(lead + (prob.num_q_heads,), dtype=torch.float32, device=device)


def decode_step(prob, desc, q, k_cache, v_cache, block_table, seq_lens, bufs: Buffers, stream=None, k_scale=None,
                v_scale=None, planned: bool = False, separate: bool = False):
    """Plan (dynamic or static, per `desc.kind`) + decode + combine, asynchronously on `stream`.

    One da_decode_step call, or, with separate=True, the three calls one by one.  With
    k_scale/v_scale given, the caches are FP8 E4M3 codes.  planned=True skips the plan
    (da_plan_append has already written it into bufs.ws): decode and combine only."""
    if not planned and not separate:
        da_decode_step(prob, desc, q, k_cache, v_cache, block_table, seq_lens, bufs, k_scale=k_scale, v_scale=v_scale,
                       stream=stream)
        return bufs.out, bufs.lse
    if planned:
        pass
    elif desc.kind == PLAN_DYNAMIC:
        da_plan(prob, desc, seq_lens, bufs.ws, stream=stream)
    else:
        da_static_plan(prob, desc, seq_lens, bufs.ws, stream=stream)
    if k_scale is None:
        da_decode_attention(prob, desc, q, k_cache, v_cache, block_table, seq_lens, bufs.ws, bufs.partial_o,
                            bufs.partial_lse, bufs.out, bufs.lse, stream=stream)
    else:
        da_decode_attention_fp8(prob, desc, q, k_cache, v_cache, k_scale, v_scale, block_table, seq_lens, bufs.ws,
                                bufs.partial_o, bufs.partial_lse, bufs.out, bufs.lse, stream=stream)
    da_combine(prob, desc, bufs.ws, bufs.partial_o, bufs.partial_lse, bufs.out, bufs.lse, stream=stream)
    return bufs.out, bufs.lse


def read_plan(desc: DaPlanDesc, ws) -> dict:
    """Copy a plan out of the workspace into numpy arrays (same keys as the oracle's plan)."""
    import numpy as np
    off = da_workspace_offsets(desc)
    w = ws.detach().cpu().numpy().astype(np.int32)
    hdr = w[off[0]:off[0] + 16]
    S = int(hdr[1])
    segs = w[off[1]:off[1] + 4 * desc.max_segments].reshape(-1, 4)[:S]
    B, C = desc.batch, desc.num_ctas
    return dict(num_units=int(hdr[0]), num_segments=S, num_ctas=int(hdr[2]), tile_tokens=int(hdr[3]),
                status=int(hdr[4]), bad_index=int(hdr[5]), kind=int(hdr[6]), batch=int(hdr[7]),
                max_segments=int(hdr[8]), splits=int(hdr[9]), balance=int(hdr[10]),
                seg_req=segs[:, 0].copy(), seg_cta=segs[:, 1].copy(), seg_tile_begin=segs[:, 2].copy(),
                seg_tile_end=segs[:, 3].copy(), req_tile_prefix=w[off[2]:off[2] + B + 1].copy(),
                req_seg_begin=w[off[3]:off[3] + B + 1].copy(), cta_seg_begin=w[off[4]:off[4] + C + 1].copy())
