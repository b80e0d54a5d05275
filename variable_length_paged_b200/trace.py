"""Run a DecodeTrace on the device.

The host trace (workloads.DecodeTrace) owns the lengths, the page free list
and the reference copy of the cache; this class keeps a device copy in step:
restarted requests' pages are copied from the host, the block table and
lengths are copied whole, and each step's new K/V rows are written into their
pages by the library's append kernel (da_append_kv).

`advance` does this live, one step at a time.  `record` runs the host trace
ahead and keeps every step's changes on the device; `apply` then replays one
step's changes with device-side copies only, so a timed loop keeps the GPU
busy the way a serving engine does (no host round trip between steps).
"""

from __future__ import annotations

import torch

from . import da
from .workloads import DecodeTrace


class DeviceTrace:
    def __init__(self, trace: DecodeTrace, device="cuda"):
        self.trace = trace
        self.device = torch.device(device)
        self.prob = da.problem_from(trace.problem)
        self.k_cache = trace.k_cache.to(self.device)
        self.v_cache = trace.v_cache.to(self.device)
        self.seq_lens = torch.from_numpy(trace.seq_lens).to(self.device)
        self.block_table = torch.from_numpy(trace.block_table).to(self.device)
        self.q = trace.q.to(self.device)
        self.status = torch.zeros(2, dtype=torch.int32, device=self.device)

    def advance(self, stream=None) -> dict:
        """Advance the host trace one step and bring the device copy along (asynchronous)."""
        upd = self.trace.advance()
        if upd["restarted_pages"]:
            idx = torch.tensor(upd["restarted_pages"], dtype=torch.long)
            didx = idx.to(self.device)
            self.k_cache[didx] = self.trace.k_cache[idx].to(self.device)
            self.v_cache[didx] = self.trace.v_cache[idx].to(self.device)
        self.block_table.copy_(torch.from_numpy(self.trace.block_table))
        self.seq_lens.copy_(torch.from_numpy(self.trace.seq_lens))
        self.q.copy_(upd["q"])
        new_k = upd["new_k"].to(self.device)
        new_v = upd["new_v"].to(self.device)
        da.da_append_kv(self.prob, new_k, new_v, self.block_table, self.seq_lens, self.k_cache, self.v_cache,
                        self.status, stream=stream)
        return upd

    def record(self, steps: int) -> list[dict]:
        """Advance the host trace `steps` times now; each step's changes, kept on the device."""
        ups = []
        for _ in range(steps):
            upd = self.trace.advance()
            d = dict(block_table=torch.from_numpy(self.trace.block_table.copy()).to(self.device),
                     seq_lens=torch.from_numpy(self.trace.seq_lens.copy()).to(self.device),
                     q=upd["q"].to(self.device), new_k=upd["new_k"].to(self.device),
                     new_v=upd["new_v"].to(self.device), kv_bytes=self.trace.kv_bytes())
            if upd["restarted_pages"]:
                idx = torch.tensor(upd["restarted_pages"], dtype=torch.long)
                d["pages"] = idx.to(self.device)
                d["page_k"] = self.trace.k_cache[idx].to(self.device)
                d["page_v"] = self.trace.v_cache[idx].to(self.device)
            ups.append(d)
        return ups

    def apply(self, upd: dict, stream=None, plan=None):
        """Enqueue one recorded step's changes on `stream`: page copies of restarted requests,
        block table, lengths and q (device to device), then the append kernel.

        With plan=(desc, ws) the append is fused with the step's dynamic plan into `ws`
        (da_plan_append), and the decode that follows skips its own planning."""
        s = stream if stream is not None else torch.cuda.current_stream()
        with torch.cuda.stream(s):
            if "pages" in upd:
                self.k_cache.index_copy_(0, upd["pages"], upd["page_k"])
                self.v_cache.index_copy_(0, upd["pages"], upd["page_v"])
            self.block_table.copy_(upd["block_table"])
            self.seq_lens.copy_(upd["seq_lens"])
            self.q.copy_(upd["q"])
        if plan is None:
            da.da_append_kv(self.prob, upd["new_k"], upd["new_v"], self.block_table, self.seq_lens, self.k_cache,
                            self.v_cache, self.status, stream=s)
        else:
            desc, ws = plan
            da.da_plan_append(self.prob, desc, self.seq_lens, ws, upd["new_k"], upd["new_v"], self.block_table,
                              self.k_cache, self.v_cache, self.status, stream=s)
