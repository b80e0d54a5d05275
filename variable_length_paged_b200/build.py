"""Build libda.so (the CUDA library) in-tree with nvcc for sm_100a.

    python -m variable_length_paged_b200.build [--force] [--define NAME=VALUE ...] [--out PATH]

The library is written next to this file; it is git-ignored but travels with
the source tree, so a machine without nvcc can still load it.  `--define`
passes a preprocessor definition to every source (e.g. DA_BF16_FFMA=1, the
FP32-FMA consumer of the bf16 decode kernel kept for comparison); such a build
goes to `--out` and is loaded by setting DA_LIB_PATH to that file.
"""

from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libda.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17", "-shared",
         "-Xcompiler", "-fPIC,-fvisibility=hidden", "-Xptxas", "-v", "--expt-relaxed-constexpr"]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")))


def _inputs() -> list[str]:
    return sources() + sorted(glob.glob(os.path.join(HERE, "csrc", "*.cuh"))) + [os.path.join(ROOT, "include", "da.h")]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False, defines: tuple[str, ...] = (), out: str | None = None) -> str:
    dst = os.path.abspath(out) if out else LIB
    if defines and dst == LIB:
        raise ValueError("a build with --define goes to --out, not over the library the package loads")
    if not force and not defines and up_to_date():
        return LIB
    tmp = dst + f".tmp{os.getpid()}"
    cmd = [NVCC, *FLAGS, *(f"-D{d}" for d in defines), "-I", os.path.join(ROOT, "include"), *sources(), "-o", tmp]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stderr}")
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(tmp, dst)
    return dst


def _main(argv: list[str]) -> None:
    defines, out, i = [], None, 0
    while i < len(argv):
        if argv[i] == "--define" and i + 1 < len(argv):
            defines.append(argv[i + 1])
            i += 2
        elif argv[i] == "--out" and i + 1 < len(argv):
            out = argv[i + 1]
            i += 2
        else:
            i += 1
    print(build(force="--force" in argv, verbose=True, defines=tuple(defines), out=out))


if __name__ == "__main__":
    _main(sys.argv[1:])
