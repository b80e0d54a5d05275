#!/usr/bin/env python
"""Benchmark: one decode step of dynamic split-KV attention over a paged KV cache.

A step is the whole hot path on one batch: on-device plan -> decode kernel ->
log-sum-exp combine, through the C ABI (libda.so).  The default workload is the
skewed continuous batch (128 requests: 115 with lengths uniform in [256, 2048],
13 with lengths uniform in [16384, 65536]; 1 % of K rows scaled by 8; 64 query /
8 KV heads, head_dim 128, page 64): 2.72 GB of K/V per step, the largest
single-step workload, far larger than the 126 MB L2, so consecutive steps cannot
hit in L2.

Printed (rank 0, one JSON line): KV-read GB/s of the whole step (value), the
step time (mean over the timed region, and median / p10 / p90 of the per-step
times), the decode kernel's own achieved bandwidth against the measured HBM
peak, the same step under the static split-k schedule (default and best split
count), an end-to-end number (one da_decode_step_host call per step from pinned
host buffers: the plan launch reads lengths, block table and q over PCIe, and
out/lse are written in place into host memory), the CPU oracle's rate
on this machine's cores (all of them, and one thread), and the SM clocks seen
during the measurement.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config skewed]

For a bf16 cache (`--balance auto`, the default) a balance table is measured before
the timed steps from a few steps' block times, and kept only if the graph-replayed
step is faster with it; `launch.balance` says what was done.

With N > 1 (torchrun) every rank runs its own, differently seeded batch of the
same shape (weak scaling: requests are independent, so there is no data-path
collective); the step time is the max over ranks and the value is the KV bytes
of all ranks over that time.  `--impl reference` times the CPU oracle instead.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

BALANCE_NOTE = ("measured before the timed steps: 2 rounds of 9 steps with block times, per-block medians "
                "-> da_balance_from_times -> da_balance_set")


def balance_wanted(args) -> bool:
    """Whether the dynamic plan runs with a measured balance table (see --balance)."""
    return args.balance == "measure" or (args.balance == "auto" and args.kv == "bf16")


def measure_balance(da, desc, step, stream, reps: int = 3, n: int = 20) -> dict:
    """Measure a balance table into desc (untimed), then keep it only if the step is faster with
    it: a CUDA graph of the step with the table and one without, `n` replays each, alternated
    `reps` times, best of each.  The table places the plan's CTAs by the SMs the blocks ran on
    while it was measured; the check guards against a launch that lands them elsewhere."""
    import torch
    table = da.calibrate_balance(desc, step, "cuda", stream=stream)
    graphs = {}
    for keep in (True, False):
        desc.balance = table.data_ptr() if keep else None
        step(desc)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step(desc)
        graphs[keep] = g
    best = {True: float("inf"), False: float("inf")}
    for _ in range(reps):
        for keep in (True, False):
            best[keep] = min(best[keep], time_region(stream, graphs[keep].replay, n) / n * 1e3)
    kept = best[True] < best[False]
    desc.balance = table.data_ptr() if kept else None
    del graphs
    return dict(table=table, note={"measured": BALANCE_NOTE, "kept": kept,
                                   "check_us_per_step_with_without": [round(best[True], 2), round(best[False], 2)]})


METRIC = "µs/decode step and KV-read HBM GB/s (% of B200 peak) vs static split-k"
FALLBACK_HBM_GBS = 6650.0
DATASHEET_HBM_GBS = 8000.0
L2_BYTES = 126 * 2**20
# the sources each cache format's decode kernel is built from (the ncu traffic record is keyed to them)
KERNEL_SOURCES = {
    "bf16": ["variable_length_paged_b200/csrc/decode.cu", "variable_length_paged_b200/csrc/da_internal.cuh"],
    "fp8": ["variable_length_paged_b200/csrc/decode_tc.cu", "variable_length_paged_b200/csrc/da_internal.cuh"],
}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_kernel_traffic.txt")


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="skewed", choices=["mixed", "skewed", "low_conc", "uniform", "tiny", "trace"])
    ap.add_argument("--kv", choices=["bf16", "fp8"], default="bf16", help="KV cache format")
    ap.add_argument("--q-len", type=int, default=1, help="queries per request (multi-query decode)")
    ap.add_argument("--tile", type=int, default=64)
    ap.add_argument("--width", type=int, default=0, help="CTAs per KV head (0 = 2 per SM / Hkv)")
    ap.add_argument("--merge-in-decode", action="store_true",
                    help="dynamic plan: merge split requests in the decode kernel instead of a combine launch")
    ap.add_argument("--start-cost", type=int, default=None,
                    help="dynamic plan: units charged to the CTA that starts a request (default: the library's)")
    ap.add_argument("--balance", choices=["auto", "none", "measure"], default="auto",
                    help="dynamic plan: measure a balance table (per-CTA weights and block placement from "
                         "block times, untimed, before the timed steps) or keep the even split; auto = measure "
                         "for a bf16 cache, none for FP8 (the tcgen05 kernel's blocks land on other SMs from "
                         "step to step, so a placement measured once does not hold)")
    ap.add_argument("--no-static", action="store_true", help="skip the static split-k comparison")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    return ap.parse_args()


# ------------------------------------------------------------------------------------------------
# plumbing


def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def reduce_max_sum(values_max, values_sum, world):
    """Max over ranks of `values_max`, sum over ranks of `values_sum` (host floats)."""
    if world == 1:
        return list(values_max), list(values_sum)
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    a = torch.tensor(values_max, dtype=torch.float64, device=dev)
    b = torch.tensor(values_sum, dtype=torch.float64, device=dev)
    dist.all_reduce(a, op=dist.ReduceOp.MAX)
    dist.all_reduce(b, op=dist.ReduceOp.SUM)
    return a.cpu().tolist(), b.cpu().tolist()


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "MEASURED_PEAKS.json hbm_gbs (copy test on this pool; of measured)"
    except Exception:
        return FALLBACK_HBM_GBS, "profiling-recipe fallback 6.65 TB/s (of fallback)"


def kernel_source_hash(kv="bf16"):
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kv]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def decode_kernel_name(problem, fp8, q_len):
    """The decode kernel the library launches for this shape (the one the roofline describes)."""
    if fp8 and q_len <= 1 and problem.num_q_heads // problem.num_kv_heads <= 8:
        return f"decode_tc_kernel<{problem.head_dim},fp8> (tcgen05)"
    return f"decode_kernel<{problem.head_dim},{'fp8' if fp8 else 'bf16'}>"


def recorded_traffic(workload_name, kv="bf16", q_len=1):
    """DRAM bytes per decode launch from the committed ncu record, if it matches this kernel source.

    Returns (bytes or None, where they come from or why there are none)."""
    rel = os.path.relpath(TRAFFIC_FILE, ROOT)
    try:
        with open(TRAFFIC_FILE) as f:
            j = dict(ln.split(": ", 1) for ln in f.read().splitlines() if ln and not ln.startswith("#"))
    except Exception:
        return None, f"no ncu capture recorded ({rel} missing)"
    if os.environ.get("DA_LIB_PATH"):
        return None, "a library built with other definitions (DA_LIB_PATH) is loaded; the record is for the default build"
    if j.get(f"kernel_source_sha.{kv}") != kernel_source_hash(kv):
        return None, f"{kv} decode kernel changed since the ncu capture in {rel}"
    key = f"{workload_name}.{kv}"
    if q_len > 1 or f"{key}.dram_bytes_read_per_launch" not in j:
        return None, f"no ncu capture for {key}" + (f" with {q_len} queries" if q_len > 1 else "") + f" in {rel}"
    return (int(j[f"{key}.dram_bytes_read_per_launch"]) + int(j[f"{key}.dram_bytes_write_per_launch"]),
            f"{rel} ({key}; captured with: {j.get(f'{key}.command', '')})")


class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled every 200 ms while active."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        import torch
        self.proc = None
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        sel = []
        try:
            pr = torch.cuda.get_device_properties(device_index)
            sel = ["-i", f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"]
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
            if vis:
                sel = ["-i", vis.split(",")[device_index]]
        self.cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200", *sel]

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        self.file.flush()
        self.file.seek(0)
        rows = [ln.strip().split(", ") for ln in self.file.read().splitlines() if ln.strip()]
        rows = [r for r in rows if len(r) >= 9]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        smax = [num(r[2]) for r in rows if num(r[2]) is not None]
        power = [num(r[3]) for r in rows if num(r[3]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip().lower() == "active"})
        # median over samples taken while the GPU was clocked up (under load)
        hi = [s for s in sm if smax and s >= 0.5 * max(smax)] or sm
        return {"sm_mhz": statistics.median(hi) if hi else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows), "power_w_max": max(power) if power else None}


# ------------------------------------------------------------------------------------------------
# our arm


def time_region(stream, fn, steps, per_step=False):
    """Device time of `steps` calls of fn() on `stream`, bracketed by CUDA events (ms).

    With per_step, an event is also recorded between consecutive calls, and the list of
    per-call times (ms) is returned as well; their sum is the bracketed time."""
    import torch
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1 if per_step else 2)]
    torch.cuda.synchronize()
    ev[0].record(stream)
    for i in range(steps):
        fn()
        if per_step:
            ev[i + 1].record(stream)
    if not per_step:
        ev[1].record(stream)
    torch.cuda.synchronize()
    total = ev[0].elapsed_time(ev[-1])
    if not per_step:
        return total
    return total, [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]


def step_stats(ms_list):
    """Median, p10 and p90 of per-step times, in µs."""
    import numpy as np
    a = np.asarray(ms_list, dtype=np.float64) * 1e3
    return {"median": round(float(np.median(a)), 2), "p10": round(float(np.percentile(a, 10)), 2),
            "p90": round(float(np.percentile(a, 90)), 2)}


def workload_config(name, w, w8=None, q_len=1):
    """The `config` object of the JSON line: the workload alone, identical for both arms."""
    kv = w8.kv_bytes if w8 is not None else w.kv_bytes
    return {"workload": f"{name}: {w.recipe}" + ("; FP8 E4M3 KV, per-head scales" if w8 is not None else "")
            + (f"; {q_len} queries per request" if q_len > 1 else ""),
            "batch": w.problem.batch, "kv_format": "fp8" if w8 is not None else "bf16", "q_len": q_len,
            "kv_bytes_per_step_per_gpu": int(kv),
            "l2": "inputs larger than L2 (K/V read per step >> 126 MB), no flush" if kv > L2_BYTES else
                  f"inputs fit in L2 ({kv} B of K/V per step): a latency case, not an HBM figure"}


def run_ours(args, world, rank, local):
    import numpy as np
    import torch

    from variable_length_paged_b200 import da
    from variable_length_paged_b200 import workloads as W

    da.lib()  # fail loudly if the CUDA library is missing
    seed_shift = 1000 * rank
    gen = W.CONFIGS[args.config]
    qkw = {"q_len": args.q_len} if args.q_len > 1 else {}
    w = gen(seed=gen.__defaults__[0] + seed_shift, **qkw) if rank else gen(**qkw)
    w8 = W.quantize_fp8(w) if args.kv == "fp8" else None
    dw = w8.to("cuda") if w8 is not None else w.to("cuda")
    prob = da.problem_from(dw.problem)
    desc = da.da_plan_desc_init(prob, da.PLAN_DYNAMIC, args.tile, args.width, merge_in_decode=args.merge_in_decode,
                                start_cost=args.start_cost)
    bufs = da.Buffers(prob, desc, "cuda")
    kv_bytes = w8.kv_bytes if w8 is not None else w.kv_bytes
    stream = torch.cuda.Stream()
    steps, warm = max(1, args.steps), max(3, args.warmup)

    def step(d=desc, b=bufs):
        da.decode_step(prob, d, dw.q, dw.k_cache, dw.v_cache, dw.block_table, dw.seq_lens, b, stream=stream,
                       k_scale=dw.k_scale, v_scale=dw.v_scale)

    def decode_only(d=desc, b=bufs):
        if w8 is None:
            da.da_decode_attention(prob, d, dw.q, dw.k_cache, dw.v_cache, dw.block_table, dw.seq_lens, b.ws,
                                   b.partial_o, b.partial_lse, b.out, b.lse, stream=stream)
        else:
            da.da_decode_attention_fp8(prob, d, dw.q, dw.k_cache, dw.v_cache, dw.k_scale, dw.v_scale,
                                       dw.block_table, dw.seq_lens, b.ws, b.partial_o, b.partial_lse, b.out, b.lse,
                                       stream=stream)

    result = {}
    clocks = ClockSampler(local)
    with clocks:
        with torch.cuda.stream(stream):
            for _ in range(warm):
                step()
            balance = {"note": "none"}
            if balance_wanted(args):  # untimed: block times of a few steps -> the table in desc
                balance = measure_balance(da, desc, lambda d: step(d, bufs), stream)
                for _ in range(warm):
                    step()
            torch.cuda.synchronize()
            status = da.da_read_status(bufs.ws, stream=stream)
            # headline: the step captured in a CUDA graph (plan, decode, combine), replayed K times
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                step()
            for _ in range(warm):
                graph.replay()
            barrier(world)
            ms_graph = time_region(stream, graph.replay, steps)  # the headline: K replays, events around them
            barrier(world)
            # per-step times from a second pass with an event between replays (an event per step
            # is a stream operation of its own, so the headline is not taken from this pass)
            _, per_step_ms = time_region(stream, graph.replay, steps, per_step=True)
            barrier(world)
            ms_eager = time_region(stream, step, steps)
            # decode kernel alone, per launch, inside a run of eager steps
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
            torch.cuda.synchronize()
            for a, b in ev:
                da.da_plan(prob, desc, dw.seq_lens, bufs.ws, stream=stream)
                a.record(stream)
                decode_only()
                b.record(stream)
                da.da_combine(prob, desc, bufs.ws, bufs.partial_o, bufs.partial_lse, bufs.out, bufs.lse,
                              stream=stream)
            torch.cuda.synchronize()
            dec_ms = [a.elapsed_time(b) for a, b in ev]
            # static split-k comparator: default split count, then a sweep
            static = {}
            if not args.no_static:
                sdef = da.da_plan_desc_init(prob, da.PLAN_STATIC, args.tile, 0)
                for S in [sdef.splits] + [s for s in (1, 2, 4, 8, 16, 32, 64) if s != sdef.splits]:
                    sd = da.da_plan_desc_init(prob, da.PLAN_STATIC, args.tile, S)
                    sb = da.Buffers(prob, sd, "cuda")
                    for _ in range(warm):
                        step(sd, sb)
                    g2 = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g2, stream=stream):
                        step(sd, sb)
                    ks = max(3, steps // 4)
                    static[S] = time_region(stream, g2.replay, ks) / ks
                    del g2, sb
                static_default = static[sdef.splits]
                best_S = min(static, key=static.get)
            # end to end: host inputs -> device, step, outputs -> host, every step
            q_h = w.q.pin_memory()
            sl_h = torch.from_numpy(w.seq_lens).pin_memory()
            bt_h = torch.from_numpy(w.block_table).pin_memory()
            out_h = torch.empty(bufs.out.shape, dtype=bufs.out.dtype).pin_memory()
            lse_h = torch.empty(bufs.lse.shape, dtype=bufs.lse.dtype).pin_memory()

            def e2e_step():  # one C call: the plan launch reads lengths, block table and q from the pinned
                # host buffers; decode and combine write out / lse in place in pinned host memory
                da.da_decode_step_host(prob, desc, q_h, bt_h, sl_h, dw.k_cache, dw.v_cache, dw.q, dw.block_table,
                                       dw.seq_lens, bufs, out_h, lse_h, k_scale=dw.k_scale, v_scale=dw.v_scale,
                                       stream=stream)

            for _ in range(warm):
                e2e_step()
            barrier(world)
            ms_e2e = time_region(stream, e2e_step, steps)
    h2d = q_h.numel() * q_h.element_size() + sl_h.numel() * 4 + bt_h.numel() * 4
    d2h = out_h.numel() * out_h.element_size() + lse_h.numel() * 4

    dec_avg_ms = statistics.mean(dec_ms)
    st = step_stats(per_step_ms)
    maxes, sums = reduce_max_sum([ms_graph, ms_eager, ms_e2e, dec_avg_ms, st["median"], st["p10"], st["p90"]],
                                 [float(kv_bytes)], world)
    ms_graph, ms_eager, ms_e2e, dec_avg_ms = maxes[:4]
    st = {"median": round(maxes[4], 2), "p10": round(maxes[5], 2), "p90": round(maxes[6], 2)}
    total_bytes = sums[0]
    step_s = ms_graph / 1e3 / steps
    value = total_bytes / step_s / 1e9
    peak, peak_src = measured_peak()
    dec_gbs = kv_bytes / (dec_avg_ms / 1e3) / 1e9
    traffic, traffic_note = recorded_traffic(args.config, args.kv, args.q_len)
    result.update(
        metric=METRIC, value=round(value, 2), unit="GB/s", n_gpus=world, steps=steps, warmup=warm,
        ms_per_step=round(ms_graph / steps, 5), us_per_step=round(ms_graph / steps * 1e3, 2),
        us_per_step_median_p10_p90=[st["median"], st["p10"], st["p90"]],
        higher_is_better=True, scaling="weak", vs_baseline=None, dtype="bf16", data="synthetic",
        config=workload_config(args.config, w, w8, args.q_len),
        launch={"tile_tokens": desc.tile_tokens, "ctas_per_kv_head": desc.num_ctas,
                "merge_in_decode": bool(desc.merge_in_decode), "start_cost": int(desc.start_cost), "graph": True,
                "balance": balance["note"],
                "timing": "one CUDA graph per step (plan, decode, combine), K replays between CUDA events on "
                          "the launching stream; median/p10/p90 from a second pass of K replays with an event "
                          "between replays"},
        frac_of_peak=round(value / world / peak, 4), frac_of_datasheet_8tbs=round(value / world / DATASHEET_HBM_GBS, 4),
        eager_us_per_step=round(ms_eager / steps * 1e3, 2),
        roofline={"bound": "hbm", "achieved": round(dec_gbs, 2), "peak": peak, "unit": "GB/s",
                  "frac": round(dec_gbs / peak, 4), "traffic": traffic,
                  "kernel": decode_kernel_name(w.problem, bool(w8), args.q_len),
                  "algorithmic_bytes_per_launch": kv_bytes,
                  "launch_us": round(dec_avg_ms * 1e3, 2), "peak_source": peak_src, "traffic_source": traffic_note},
        e2e={"value": round(total_bytes / (ms_e2e / 1e3 / steps) / 1e9, 2), "unit": "GB/s",
             "us_per_step": round(ms_e2e / steps * 1e3, 2), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
             "transfer": "da_decode_step_host with pinned host buffers: the plan launch reads seq_lens, block "
                         "table and q over PCIe; decode and combine write out/lse in place over PCIe"},
        # plan, decode (+ combine unless merged in decode), for each timed step of the headline graph
        gpu_launches=(3 - desc.merge_in_decode) * steps,
        device_status=status[0],
    )
    if static:
        result["static_split_k"] = {"default_splits": sdef.splits,
                                    "default_us_per_step": round(static_default * 1e3, 2),
                                    "best_splits": best_S, "best_us_per_step": round(static[best_S] * 1e3, 2),
                                    "sweep_us": {str(k): round(v * 1e3, 2) for k, v in sorted(static.items())}}
        result["speedup_vs_static_default"] = round(static_default / (ms_graph / steps), 3)
        result["speedup_vs_static_best"] = round(static[best_S] / (ms_graph / steps), 3)
    result["clocks"] = clocks.summary()
    if rank == 0 and world == 1 and not args.no_cpu:
        result["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds, w8)
    return result


def warm_apply_path(da, prob, stream):
    """Run every kernel on a step's change path once on scratch data, so that the first timed step
    does not pay for loading them (CUDA loads kernels lazily, on first launch)."""
    import torch
    with torch.cuda.stream(stream):
        p1 = da.problem(1, prob.num_q_heads, prob.num_kv_heads, prob.head_dim, prob.page_size, 1, 2, prob.scale)
        d1 = da.da_plan_desc_init(p1, da.PLAN_DYNAMIC, 64, 0)
        ws = da.Buffers(p1, d1, "cuda").ws
        kc = torch.zeros(2, prob.num_kv_heads, prob.page_size, prob.head_dim, dtype=torch.bfloat16, device="cuda")
        vc = torch.zeros_like(kc)
        nk = torch.zeros(1, prob.num_kv_heads, prob.head_dim, dtype=torch.bfloat16, device="cuda")
        sl = torch.ones(1, dtype=torch.int32, device="cuda")
        bt = torch.zeros(1, 1, dtype=torch.int32, device="cuda")
        st = torch.zeros(2, dtype=torch.int32, device="cuda")
        kc.index_copy_(0, torch.ones(1, dtype=torch.long, device="cuda"), vc[:1])
        da.da_append_kv(p1, nk, nk, bt, sl, kc, vc, st, stream=stream)
        da.da_plan_append(p1, d1, sl, ws, nk, nk, bt, kc, vc, st, stream=stream)
    torch.cuda.synchronize()


def run_trace(args, world, rank, local):
    """The 256-step decode trace: per step, that step's recorded changes applied on the device (untimed),
    then the timed step."""
    import numpy as np
    import torch

    from variable_length_paged_b200 import da
    from variable_length_paged_b200 import workloads as W
    from variable_length_paged_b200.trace import DeviceTrace

    da.lib()
    tr = W.DecodeTrace(seed=4 + 1000 * rank)
    dt = DeviceTrace(tr)
    prob = dt.prob
    stream = torch.cuda.Stream()
    desc = da.da_plan_desc_init(prob, da.PLAN_DYNAMIC, args.tile, args.width, merge_in_decode=args.merge_in_decode,
                                start_cost=args.start_cost)
    sdesc = da.da_plan_desc_init(prob, da.PLAN_STATIC, args.tile, 0)
    bufs, sbufs = da.Buffers(prob, desc, "cuda"), da.Buffers(prob, sdesc, "cuda")
    steps, warm = min(max(1, args.steps), tr.steps), max(3, args.warmup)

    def step(d, b, planned=False):
        da.decode_step(prob, d, dt.q, dt.k_cache, dt.v_cache, dt.block_table, dt.seq_lens, b, stream=stream,
                       planned=planned)

    balance = {"note": "none"}
    if balance_wanted(args):  # untimed, on the trace's first lengths
        with torch.cuda.stream(stream):
            balance = measure_balance(da, desc, lambda d: step(d, bufs), stream)
        torch.cuda.synchronize()

    graphs = {}
    with torch.cuda.stream(stream):
        for key, d, b, planned in (("dynamic", desc, bufs, False), ("static", sdesc, sbufs, False),
                                   ("after_plan_append", desc, bufs, True)):
            for _ in range(warm):
                step(d, b, planned)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                step(d, b, planned)
            graphs[key] = g
        torch.cuda.synchronize()
    # the host trace runs ahead; its per-step changes wait on the device, so the timed loop below
    # is device work only: apply step t's changes (untimed), then the two timed step variants
    warm_apply_path(da, prob, stream)
    kv0 = tr.kv_bytes()
    ups = dt.record(steps - 1)
    kv = [kv0] + [u["kv_bytes"] for u in ups]
    ev = {k: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
          for k in ("dynamic", "static", "append_separate", "append_fused")}
    clocks = ClockSampler(local)
    with clocks, torch.cuda.stream(stream):  # replay() launches on the current stream
        torch.cuda.synchronize()
        barrier(world)
        for t in range(steps):
            if t > 0:
                # the step's changes plus the step, twice: append kernel then the planned step, and the
                # fused plan + append launch then the step without its plan (both leave the same state,
                # every change is written at an absolute place)
                for key, plan in (("append_separate", None), ("append_fused", (desc, bufs.ws))):
                    e0, e1 = ev[key][t]
                    e0.record(stream)
                    dt.apply(ups[t - 1], stream=stream, plan=plan)
                    graphs["dynamic" if plan is None else "after_plan_append"].replay()
                    e1.record(stream)
            for key in ("dynamic", "static"):
                e0, e1 = ev[key][t]
                e0.record(stream)
                graphs[key].replay()
                e1.record(stream)
        torch.cuda.synchronize()
        status = da.da_read_status(bufs.ws, stream=stream)
    times = {k: [a.elapsed_time(b) for a, b in (v[1:] if k.startswith("append") else v)] for k, v in ev.items()}
    tot_ms = {k: sum(v) for k, v in times.items()}
    maxes, sums = reduce_max_sum([tot_ms["dynamic"], tot_ms["static"]], [float(sum(kv))], world)
    dyn_ms, st_ms = maxes
    value = sums[0] / (dyn_ms / 1e3) / 1e9
    peak, peak_src = measured_peak()
    d = np.array(times["dynamic"])
    return dict(
        metric=METRIC, value=round(value, 2), unit="GB/s", n_gpus=world, steps=steps, warmup=warm,
        ms_per_step=round(dyn_ms / steps, 5), us_per_step=round(dyn_ms / steps * 1e3, 2),
        us_per_step_median=round(float(np.median(d)) * 1e3, 2),
        us_per_step_p10_p90=[round(float(np.percentile(d, 10)) * 1e3, 2), round(float(np.percentile(d, 90)) * 1e3, 2)],
        higher_is_better=True, scaling="weak", vs_baseline=None, dtype="bf16", data="synthetic",
        config={"workload": f"trace: {tr.recipe}", "batch": prob.batch, "steps_timed": steps,
                "kv_bytes_first_last_step": [kv[0], kv[-1]], "tile_tokens": desc.tile_tokens,
                "ctas_per_kv_head": desc.num_ctas, "merge_in_decode": bool(desc.merge_in_decode),
                "start_cost": int(desc.start_cost), "graph": True, "balance": balance["note"], 
                "untimed": "device copies of each step's changes (restarted pages, block table, lengths, q) "
                           "and the KV append kernel, enqueued between the timed steps",
                "l2": f"inputs larger than L2 ({min(kv) / 1e9:.1f}-{max(kv) / 1e9:.1f} GB K/V per step), no flush"},
        frac_of_peak=round(value / world / peak, 4), peak=peak, peak_source=peak_src,
        static_split_k={"default_splits": sdesc.splits, "us_per_step": round(st_ms / steps * 1e3, 2)},
        speedup_vs_static_default=round(st_ms / dyn_ms, 3),
        with_append={"note": "steps 1.. with their changes applied inside the timed region: device copies of "
                             "block table, lengths, q and restarted pages, then the KV append",
                     "separate_us_per_step": round(float(np.mean(times["append_separate"])) * 1e3, 2),
                     "fused_plan_append_us_per_step": round(float(np.mean(times["append_fused"])) * 1e3, 2),
                     "separate_us_median": round(float(np.median(times["append_separate"])) * 1e3, 2),
                     "fused_plan_append_us_median": round(float(np.median(times["append_fused"])) * 1e3, 2)},
        # per step: dynamic (plan, decode, combine unless merged) + static (3); steps 1..: append + dynamic step,
        # plan_append + decode (+ combine)
        gpu_launches=(6 - desc.merge_in_decode) * steps + (7 - 2 * desc.merge_in_decode) * (steps - 1),
        device_status=status[0],
        append_status=dt.status.tolist(), clocks=clocks.summary())


def _oracle_run(w, w8, pairs=None, threads=0):
    """One oracle call over the (request, head) pairs (all of them when None)."""
    import numpy as np

    import oracle
    if w8 is None and w.q.dim() == 4:  # multi-query: whole batch only
        oracle.attention_mq(w.q, w.k_cache, w.v_cache, w.block_table, w.seq_lens, scale=w.problem.scale,
                            threads=threads)
    elif w8 is None:
        oracle.attention(w.q, w.k_cache, w.v_cache, w.block_table, w.seq_lens, scale=w.problem.scale, pairs=pairs,
                         threads=threads)
    else:
        oracle.attention_fp8(w.q, w8.k_code, w8.v_code, w8.k_scale.astype(np.float64), w8.v_scale.astype(np.float64),
                             w.block_table, w.seq_lens, scale=w.problem.scale, pairs=pairs, threads=threads)


def request_sample(w, w8, seconds, threads):
    """A seeded sample of whole requests (all heads) that the oracle runs in about `seconds` with
    `threads` threads (at least one request), from a calibration run on the shortest request.
    Returns (pairs, requests, tokens)."""
    import numpy as np
    B, Hq = w.problem.batch, w.problem.num_q_heads
    live = [b for b in range(B) if w.seq_lens[b] > 0] or [0]
    short = min(live, key=lambda b: w.seq_lens[b])
    t0 = time.perf_counter()
    _oracle_run(w, w8, (np.full(Hq, short, np.int32), np.arange(Hq, dtype=np.int32)), threads)
    rate = max(int(w.seq_lens[short]), 1) / max(time.perf_counter() - t0, 1e-6)  # tokens/s, all heads
    budget = rate * seconds
    picks, acc = [], 0
    for b in np.random.default_rng(0).permutation(B):
        if picks and acc + w.seq_lens[b] > budget:
            continue
        picks.append(int(b))
        acc += int(w.seq_lens[b])
    pairs = (np.repeat(np.array(picks, np.int32), Hq), np.tile(np.arange(Hq, dtype=np.int32), len(picks)))
    return pairs, picks, acc


def cpu_baseline(w, seconds, w8=None):
    """The CPU oracle (fp64) on this host: all cores over whole batches, repeated for about `seconds`;
    then one thread over a seeded sample of requests sized to about `seconds`."""
    import oracle
    oracle.build()
    kv = w8.kv_bytes if w8 is not None else w.kv_bytes
    per_token = kv / max(int(w.seq_lens.sum()), 1)  # K/V bytes per cached token (all KV heads)
    t0 = time.perf_counter()
    passes = 0
    while True:
        _oracle_run(w, w8)
        passes += 1
        if time.perf_counter() - t0 >= seconds or passes >= 50:
            break
    dt = time.perf_counter() - t0
    res = {"value": round(passes * kv / dt / 1e9, 4), "unit": "GB/s", "cores": oracle.num_threads(),
           "kind": "oracle", "sample": f"{passes} pass(es) of the fp64 oracle over the full batch "
                                       f"({w.problem.batch} requests x {w.problem.num_q_heads} heads), {dt:.1f} s"}
    if w.q.dim() == 4 and w8 is None:
        t0 = time.perf_counter()
        _oracle_run(w, w8, threads=1)
        dt1, tok, desc = time.perf_counter() - t0, int(w.seq_lens.sum()), "the full batch"
    else:
        pairs, picks, tok = request_sample(w, w8, seconds, 1)
        t0 = time.perf_counter()
        _oracle_run(w, w8, pairs, threads=1)
        dt1 = time.perf_counter() - t0
        desc = f"{len(picks)} of {w.problem.batch} requests (all {w.problem.num_q_heads} heads, {tok} tokens)"
    res["one_thread"] = {"value": round(tok * per_token / dt1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                         "sample": f"{desc}, {dt1:.1f} s"}
    return res


# ------------------------------------------------------------------------------------------------
# reference arm: the CPU oracle, timed on bounded samples of the same workload


def run_reference(args, rank):
    import oracle
    from variable_length_paged_b200 import workloads as W

    oracle.build()
    w = W.DecodeTrace().workload() if args.config == "trace" else W.CONFIGS[args.config]()
    w8 = W.quantize_fp8(w) if args.kv == "fp8" else None
    steps, warm = max(1, args.steps), max(3, args.warmup)
    # about one second of oracle work per step, and at most ~150 s in total
    pairs, picks, tok = request_sample(w, w8, min(1.0, 150.0 / (steps + warm)), 0)
    per_token = (w8.kv_bytes if w8 is not None else w.kv_bytes) / max(int(w.seq_lens.sum()), 1)
    sample_bytes = int(round(tok * per_token))
    for _ in range(warm):
        _oracle_run(w, w8, pairs)
    t0 = time.perf_counter()
    for _ in range(steps):
        _oracle_run(w, w8, pairs)
    dt = time.perf_counter() - t0
    value = steps * sample_bytes / dt / 1e9
    B, Hq = w.problem.batch, w.problem.num_q_heads
    cpu = {"value": round(value, 4), "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
           "sample": f"{len(picks)} of {B} requests (all {Hq} heads, {tok} tokens, {sample_bytes} K/V bytes) "
                     f"per step"}
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": 1,
            "steps": steps, "warmup": warm, "ms_per_step": round(dt / steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(args.config if args.config != "trace" else "trace", w, w8),
            "cpu_baseline": cpu,
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse_args()
    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return 0
        print(json.dumps(run_reference(args, 0)), flush=True)
        return 0
    world, rank, local = dist_setup(args)
    try:
        res = run_trace(args, world, rank, local) if args.config == "trace" else run_ours(args, world, rank, local)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
