"""Spread long requests' KV caches over several GPUs (context parallelism).

Rank r of W holds a contiguous, page-aligned slice of every request's pages:
pages [floor(r*n/W), floor((r+1)*n/W)) of the request's n = ceil(L/P) pages.
Each rank runs the ordinary decode step (plan, decode, combine) on its slice,
producing (out_r, lse_r) in fp32 (the step runs with fp32 output, so no rank's
result is rounded to bf16 before the merge); softmax over disjoint token sets
merges exactly by log-sum-exp, so after an all-gather of the partial results
every rank merges them with da_merge_partials_f32, which rounds once, at the
end.  The exchange is B * Hq * (d + 1) * 4 bytes per rank and step.  Plain
decode only (q_len = 1): the query is the last token and sees every slice whole.

Source of the method: "Tencent HPC lands in SGLang, challenging default
inference kernels", section "Why Tencent HPC matters for online model serving"
(a longer history means more cached data to read; the work of one request is
split and recombined).
"""

from __future__ import annotations

import numpy as np
import torch

from . import da


def slice_pages(seq_lens, page_size: int, world: int, rank: int):
    """First and one-past-last page of each request held by `rank` (numpy int64 [B] each)."""
    lens = np.asarray(seq_lens, dtype=np.int64)
    n = (np.clip(lens, 0, None) + page_size - 1) // page_size
    return (rank * n) // world, ((rank + 1) * n) // world


def local_view(seq_lens, block_table, page_size: int, world: int, rank: int):
    """This rank's (seq_lens, block_table): the tokens of its pages, the table shifted to them."""
    lens = np.asarray(seq_lens, dtype=np.int64)
    bt = np.asarray(block_table, dtype=np.int32)
    p0, p1 = slice_pages(lens, page_size, world, rank)
    local_lens = np.clip(np.minimum(p1 * page_size, lens) - p0 * page_size, 0, None).astype(np.int32)
    local_bt = np.full_like(bt, -1)
    for b in range(bt.shape[0]):
        local_bt[b, :p1[b] - p0[b]] = bt[b, p0[b]:p1[b]]
    return local_lens, local_bt


def cp_decode_step(prob, desc, q, k_cache, v_cache, local_block_table, local_seq_lens, bufs: da.Buffers,
                   out: torch.Tensor, lse: torch.Tensor, group=None, stream=None):
    """Decode step on this rank's slice, all-gather of the partial results, log-sum-exp merge.

    `desc` must ask for fp32 output (da_plan_desc_init(..., out_f32=True)), and `bufs` be made for it;
    `out` [B, Hq, d] bf16 and `lse` [B, Hq] fp32 receive the merged result on every rank.
    """
    import contextlib

    import torch.distributed as dist

    if prob.q_len > 1:
        raise ValueError("context-parallel decode handles one query per request")
    if desc.out_format != da.OUT_F32 or bufs.out.dtype != torch.float32:
        raise ValueError("context-parallel decode exchanges fp32 results: build desc with out_f32=True")
    # the collectives order themselves after the current stream's work: make `stream` current so that
    # the all-gather follows this rank's decode and the merge follows the all-gather
    on_stream = torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()
    with on_stream:
        da.decode_step(prob, desc, q, k_cache, v_cache, local_block_table, local_seq_lens, bufs, stream=stream)
        world = dist.get_world_size(group)
        parts_out = torch.empty((world,) + tuple(bufs.out.shape), dtype=bufs.out.dtype, device=bufs.out.device)
        parts_lse = torch.empty((world,) + tuple(bufs.lse.shape), dtype=bufs.lse.dtype, device=bufs.lse.device)
        dist.all_gather_into_tensor(parts_out, bufs.out, group=group)
        dist.all_gather_into_tensor(parts_lse, bufs.lse, group=group)
        da.da_merge_partials_f32(parts_out, parts_lse, out, lse, stream=stream)
    return out, lse
