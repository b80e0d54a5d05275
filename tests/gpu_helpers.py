"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
compare with the CPU oracle on the same seeded inputs."""

from __future__ import annotations

import numpy as np
import torch

import oracle
from variable_length_paged_b200 import da
from variable_length_paged_b200 import workloads as W

# Tolerances for the decode outputs (bf16 out, fp32 lse) against the fp64 oracle.
OUT_ATOL, OUT_RTOL, LSE_ATOL = 1e-2, 1e-2, 1e-3


def run_step(w: W.Workload | W.DeviceWorkload, kind=da.PLAN_DYNAMIC, tile=64, width=0, dw=None, bufs=None,
             merge_in_decode=False):
    """Plan + decode + combine on cuda:0. Returns (out bf16 [B,Hq,d], lse [B,Hq], desc, bufs, dw)."""
    dw = dw if dw is not None else (w.to("cuda") if isinstance(w, W.Workload) else w)
    prob = da.problem_from(dw.problem)
    desc = da.da_plan_desc_init(prob, kind, tile, width, merge_in_decode=merge_in_decode)
    bufs = bufs if bufs is not None else da.Buffers(prob, desc, "cuda")
    # poison the partials and outputs so that an unwritten value cannot pass
    bufs.partial_o.fill_(float("nan"))
    bufs.partial_lse.fill_(float("nan"))
    bufs.out.fill_(float("nan"))
    bufs.lse.fill_(float("nan"))
    da.decode_step(prob, desc, dw.q, dw.k_cache, dw.v_cache, dw.block_table, dw.seq_lens, bufs)
    torch.cuda.synchronize()
    return bufs.out, bufs.lse, desc, bufs, dw


def check_against_oracle(w: W.Workload, out, lse, pairs=None, seq_lens=None):
    """Compare GPU out/lse with the oracle on all (b, h) pairs, or on the sampled `pairs`."""
    sl = w.seq_lens if seq_lens is None else seq_lens
    ref, ref_lse, st = oracle.attention(w.q, w.k_cache, w.v_cache, w.block_table, sl, scale=w.problem.scale,
                                        pairs=pairs)
    o = out.float().cpu().double().numpy()
    l = lse.cpu().double().numpy()
    if pairs is not None:
        o = o[pairs[0], pairs[1]]
        l = l[pairs[0], pairs[1]]
    assert np.all(np.isfinite(o)), "non-finite output"
    err = np.abs(o - ref)
    bound = OUT_ATOL + OUT_RTOL * np.abs(ref)
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), f"out mismatch at {worst}: gpu {o[worst]} ref {ref[worst]}"
    both_inf = np.isneginf(l) & np.isneginf(ref_lse)
    with np.errstate(invalid="ignore"):
        lerr = np.where(both_inf, 0.0, np.abs(l - ref_lse))
    assert np.all(lerr <= LSE_ATOL), f"lse mismatch: max err {np.nanmax(lerr)}"
    return float(err.max()), float(lerr.max())


def sample_pairs(w: W.Workload, n: int, seed: int = 0, include=()):
    """Random (request, head) pairs plus every head of the requests in `include`."""
    rng = np.random.default_rng(seed)
    B, Hq = w.problem.batch, w.problem.num_q_heads
    pb = list(rng.integers(0, B, n))
    ph = list(rng.integers(0, Hq, n))
    for b in include:
        pb += [b] * Hq
        ph += list(range(Hq))
    return np.array(pb, np.int32), np.array(ph, np.int32)


def assert_plan_equal(gpu: dict, ref: dict):
    for key in ("num_units", "num_segments"):
        assert gpu[key] == ref[key], (key, gpu[key], ref[key])
    for key in ("req_tile_prefix", "req_seg_begin", "cta_seg_begin", "seg_req", "seg_cta", "seg_tile_begin",
                "seg_tile_end"):
        assert np.array_equal(np.asarray(gpu[key]), np.asarray(ref[key])), key
    assert gpu["bad_index"] == ref["bad_index"]


def run_step_fp8(w8: W.Fp8Workload, kind=da.PLAN_DYNAMIC, tile=64, width=0, dw=None):
    """FP8-cache step on cuda:0 (same contract as run_step)."""
    dw = dw if dw is not None else w8.to("cuda")
    prob = da.problem_from(dw.problem)
    desc = da.da_plan_desc_init(prob, kind, tile, width)
    bufs = da.Buffers(prob, desc, "cuda")
    for t in (bufs.partial_o, bufs.partial_lse, bufs.out, bufs.lse):
        t.fill_(float("nan"))
    da.decode_step(prob, desc, dw.q, dw.k_cache, dw.v_cache, dw.block_table, dw.seq_lens, bufs,
                   k_scale=dw.k_scale, v_scale=dw.v_scale)
    torch.cuda.synchronize()
    return bufs.out, bufs.lse, desc, bufs, dw


def check_against_oracle_fp8(w8: W.Fp8Workload, out, lse, pairs=None):
    b = w8.base
    ref, ref_lse, st = oracle.attention_fp8(b.q, w8.k_code, w8.v_code, w8.k_scale.astype(np.float64),
                                            w8.v_scale.astype(np.float64), b.block_table, b.seq_lens,
                                            scale=b.problem.scale, pairs=pairs)
    o = out.float().cpu().double().numpy()
    l = lse.cpu().double().numpy()
    if pairs is not None:
        o, l = o[pairs[0], pairs[1]], l[pairs[0], pairs[1]]
    assert np.all(np.isfinite(o)), "non-finite output"
    err = np.abs(o - ref)
    bound = OUT_ATOL + OUT_RTOL * np.abs(ref)
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), f"out mismatch at {worst}: gpu {o[worst]} ref {ref[worst]}"
    both_inf = np.isneginf(l) & np.isneginf(ref_lse)
    with np.errstate(invalid="ignore"):
        lerr = np.where(both_inf, 0.0, np.abs(l - ref_lse))
    assert np.all(lerr <= LSE_ATOL), f"lse mismatch: max err {np.nanmax(lerr)}"
    return float(err.max()), float(lerr.max())


def check_mq_against_oracle(w: W.Workload, out, lse):
    """Multi-query outputs [B, Q, Hq, d] against the fp64 multi-query oracle."""
    ref, ref_lse, st = oracle.attention_mq(w.q, w.k_cache, w.v_cache, w.block_table, w.seq_lens,
                                           scale=w.problem.scale)
    return _compare(out, lse, ref, ref_lse)


def check_mq_fp8_against_oracle(w8: W.Fp8Workload, out, lse):
    """FP8 multi-query: each (request, query i) is a single-query request over its first
    L - Q + i + 1 tokens (the multi-query definition, pinned in the oracle pins)."""
    b = w8.base
    B, Q = b.q.shape[0], b.q.shape[1]
    lens = np.array([max(int(b.seq_lens[r]) - Q + i + 1, 0) for r in range(B) for i in range(Q)], np.int32)
    bt = np.repeat(b.block_table, Q, axis=0)
    q = b.q.reshape(B * Q, b.q.shape[2], b.q.shape[3])
    ref, ref_lse, st = oracle.attention_fp8(q, w8.k_code, w8.v_code, w8.k_scale.astype(np.float64),
                                            w8.v_scale.astype(np.float64), bt, lens, scale=b.problem.scale)
    return _compare(out, lse, ref.reshape(B, Q, *ref.shape[1:]), ref_lse.reshape(B, Q, -1))


def _compare(out, lse, ref, ref_lse):
    o = out.float().cpu().double().numpy()
    l = lse.cpu().double().numpy()
    assert np.all(np.isfinite(o)), "non-finite output"
    err = np.abs(o - ref)
    bound = OUT_ATOL + OUT_RTOL * np.abs(ref)
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), f"out mismatch at {worst}: gpu {o[worst]} ref {ref[worst]}"
    both_inf = np.isneginf(l) & np.isneginf(ref_lse)
    with np.errstate(invalid="ignore"):
        lerr = np.where(both_inf, 0.0, np.abs(l - ref_lse))
    assert np.all(lerr <= LSE_ATOL), f"lse mismatch: max err {np.nanmax(lerr)}"
    return float(err.max()), float(lerr.max())
