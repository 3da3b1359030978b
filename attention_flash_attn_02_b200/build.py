"""Builds libattn_sm100.so in-tree with nvcc for sm_100a.

Usage: ``python -m attention_flash_attn_02_b200.build [--verbose]`` (or call
``build()``).  Rebuilds only when a source is newer than the library.
"""
from __future__ import annotations

import glob
import os
import re
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB_NAME = "libattn_sm100.so"
LIB_PATH = os.path.join(PKG, LIB_NAME)

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build " + LIB_NAME)


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    files = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
    files += glob.glob(os.path.join(ROOT, "include", "*.h"))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB_PATH):
        return False
    t = os.path.getmtime(LIB_PATH)
    return all(os.path.getmtime(f) <= t for f in _inputs())


# The prefill kernel redistributes registers between its warpgroups with
# setmaxnreg; the split assumes this launch register count (see
# csrc/prefill_sm100.cu).  A different count could make the increase wait
# forever, so the build refuses to produce such a library.
PREFILL_LAUNCH_REGS = 128


# Kernels whose inner loops must not touch local memory: a spill there costs
# more than any tuning gains, so the build refuses it.
NO_SPILL_KERNELS = ("prefill_kernel", "decode_split_kernel", "bwd_kernel")


def check_register_counts(ptxas_log: str) -> None:
    """Checks ptxas -v output: the prefill kernels launch with
    PREFILL_LAUNCH_REGS registers and the hot kernels do not spill."""
    entry = None
    seen = 0
    for line in ptxas_log.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            entry = m.group(1)
            continue
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m and entry and any(k in entry for k in NO_SPILL_KERNELS):
            if int(m.group(1)) or int(m.group(2)):
                raise RuntimeError(f"{entry}: spills ({line.strip()})")
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and entry and "prefill_kernel" in entry:
            seen += 1
            n = int(m.group(1))
            if n != PREFILL_LAUNCH_REGS:
                raise RuntimeError(f"{entry}: launches with {n} registers, the setmaxnreg split needs "
                                   f"{PREFILL_LAUNCH_REGS}")
            entry = None
    if seen == 0:
        raise RuntimeError("ptxas reported no prefill kernel register counts")


def build(verbose: bool = False, force: bool = False, defines=(), out: str = None) -> str:
    """Compiles the library.  ``defines`` (e.g. ``["ATTN_EMU_PAIRS_PER8=3"]``)
    and ``out`` build a variant at another path; the default build needs
    neither."""
    out = out or LIB_PATH
    if not force and not defines and out == LIB_PATH and up_to_date():
        return LIB_PATH
    cmd = [_nvcc(), *NVCC_FLAGS, "-I", os.path.join(ROOT, "include")]
    cmd += [f"-D{d}" for d in defines]
    cmd += ["-Xptxas", "-v"]
    tmp = out + ".tmp"
    cmd += ["-o", tmp, *sources()]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    if verbose:
        sys.stdout.write(res.stdout + res.stderr)
    try:
        check_register_counts(res.stdout + res.stderr)
    except RuntimeError:
        os.unlink(tmp)
        raise
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    import argparse
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-D", dest="defines", action="append", default=[])
    ap.add_argument("--out", default=None)
    a = ap.parse_args()
    print(build(verbose=a.verbose, force=a.force, defines=a.defines, out=a.out))
