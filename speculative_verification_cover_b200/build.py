"""Build libdd.so in place with nvcc for sm_100a (B200), and beside it
libdd_checked.so, the same source with the device index checks compiled in
(DD_CHECK_BOUNDS; include/dd.h, dd_bounds_checked).

    python -m speculative_verification_cover_b200.build [--force] [-v]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
OUT = os.path.join(HERE, "libdd.so")
OUT_CHECKED = os.path.join(HERE, "libdd_checked.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def _nvcc():
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC)
                  if f.endswith((".cu", ".cuh", ".h"))) + [
        os.path.join(os.path.dirname(HERE), "include", "dd.h")]


def up_to_date(out: str = OUT) -> bool:
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile whichever of the two libraries is missing or older than a source
    (both at once), and return the path of libdd.so."""
    jobs = []
    for out, extra in ((OUT, []), (OUT_CHECKED, ["-DDD_CHECK_BOUNDS"])):
        if not force and up_to_date(out):
            continue
        tmp = out + ".tmp"
        cmd = [_nvcc(), *NVCC_FLAGS, *extra, "-o", tmp, os.path.join(CSRC, "libdd.cu")]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd), flush=True)
        jobs.append((subprocess.Popen(cmd), tmp, out, cmd))
    failed = None
    for proc, tmp, out, cmd in jobs:
        if proc.wait() != 0:
            failed = failed or subprocess.CalledProcessError(proc.returncode, cmd)
        else:
            os.replace(tmp, out)
    if failed:
        raise failed
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
