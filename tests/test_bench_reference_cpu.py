"""bench.py's reference arm (the fp64 oracle on the host cores) and its output contract, on CPU.

The arm is the one part of bench.py that runs without a GPU, so its JSON line is checked here:
the keys the driver reads, a positive rate, a CPU baseline that says what it timed, and an
end-to-end object with no bus traffic.  A rank other than 0 prints nothing and exits 0.
"""

import json
import os
import subprocess
import sys

from conftest import ROOT


def run_bench(*args, env_extra=None, timeout=300):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                          timeout=timeout, cwd=ROOT, env=env)


def test_reference_arm_line(oracle_lib):
    res = run_bench("--impl", "reference", "--config", "tiny", "--steps", "2", "--warmup", "3")
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["data"] == "synthetic" and d["vs_baseline"] is None
    assert d["config"]["workload"].startswith("tiny")
    # the reference arm's config is the GPU arm's (both come from one function of the workload)
    sys.argv = ["bench.py"]
    sys.path.insert(0, ROOT)
    import bench
    from variable_length_paged_b200 import workloads as W
    assert d["config"] == bench.workload_config("tiny", W.tiny())
    cpu = d["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["cores"] >= 1 and cpu["value"] == d["value"] and cpu["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_are_silent():
    res = run_bench("--impl", "reference", "--config", "tiny", "--steps", "1", "--warmup", "3",
                    env_extra={"RANK": "1", "WORLD_SIZE": "2"})
    assert res.returncode == 0 and res.stdout.strip() == ""
