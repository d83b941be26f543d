"""Build libll_swa.so in-tree for sm_100a with nvcc (no GPU needed)."""
from __future__ import annotations

import os
import re
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libll_swa.so")
SOURCES = ["ll_api.cu"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps():
    out = [os.path.join(ROOT, "include", "ll_api.h")]
    for f in os.listdir(CSRC):
        if f.endswith((".cu", ".cuh", ".h")):
            out.append(os.path.join(CSRC, f))
    return out


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in _deps())


# Kernels that re-split registers between warpgroups (setmaxnreg) must be
# launched with exactly this many registers per thread, or the increase would
# wait for registers that do not exist.
LAUNCH_REGS = {"sink_window_attention_kernel": 168}


def check_register_split(ptxas_log: str) -> None:
    current = None
    for line in ptxas_log.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            current = m.group(1)
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and current:
            for name, regs in LAUNCH_REGS.items():
                if name in current and int(m.group(1)) != regs:
                    raise RuntimeError(f"{current}: ptxas allocated {m.group(1)} registers, the warpgroup "
                                       f"register split needs exactly {regs}")


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    if not force and up_to_date():
        return LIB
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr", "-Xptxas", "-v",
           "-I", os.path.join(ROOT, "include"),
           "-o", LIB + ".tmp"] + list(extra) + [os.path.join(CSRC, s) for s in SOURCES]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building libll_swa.so")
    if verbose:
        sys.stderr.write(r.stderr)
    try:
        check_register_split(r.stderr)
    except RuntimeError:
        os.remove(LIB + ".tmp")
        raise
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
