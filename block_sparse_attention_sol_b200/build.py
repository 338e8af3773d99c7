"""Builds libsol.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python block_sparse_attention_sol_b200/build.py [--verbose]

One translation unit (csrc/sol_api.cu includes every kernel header), static
CUDA runtime, no torch dependency: the library only needs the driver at run time.
"""
from __future__ import annotations

import os
import re
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libsol.so")
SOURCES = [os.path.join(HERE, "csrc", "sol_api.cu")]
NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xptxas", "-warn-spills",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return "nvcc"


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    mtime = os.path.getmtime(LIB)
    deps = [os.path.join(ROOT, "include", "sol.h"), __file__]
    for d in os.listdir(os.path.join(HERE, "csrc")):
        deps.append(os.path.join(HERE, "csrc", d))
    return any(os.path.getmtime(p) > mtime for p in deps)


# Kernels whose spilling would silently cost performance: the build refuses them.
NO_SPILL_KERNELS = ("sparse_attn_fwd_kernel", "sparse_attn_fp8_kernel", "qk_prologue_pool_staged_kernel")
# Register ceilings that launches need: a CTA's warps are spread over the SM's four
# sub-partitions of 16 K registers each, so 10 warps (3 on some sub-partitions) get
# at most 168 per thread; a kernel built above that fails to launch.
MAX_REGS = {"sparse_attn_fwd_kernel": 168, "sparse_attn_fp8_kernel": 168}


def _check_ptxas_report(report: str) -> None:
    lines = report.splitlines()
    for name, cap in MAX_REGS.items():
        for i, line in enumerate(lines):
            if "Compiling entry function" in line and name in line:
                for follow in lines[i + 1:i + 4]:
                    m = re.search(r"Used (\d+) registers", follow)
                    if m and int(m.group(1)) > cap:
                        raise RuntimeError(f"{name} uses {m.group(1)} registers, more than the {cap} a launch allows")
    for name in NO_SPILL_KERNELS:
        found = False
        for i, line in enumerate(lines):
            if "Compiling entry function" in line and name in line:
                found = True
                for follow in lines[i + 1:i + 4]:
                    m = re.search(r"(\d+) bytes spill stores", follow)
                    if m and int(m.group(1)) != 0:
                        raise RuntimeError(f"{name} spills registers: {follow.strip()}")
        if not found:
            raise RuntimeError(f"no ptxas report for {name}")


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    cmd = [nvcc(), *NVCC_FLAGS, "-Xptxas", "-v", "-o", LIB + ".tmp", *SOURCES]
    proc = subprocess.run(cmd, capture_output=True, text=True)
    if proc.returncode != 0:
        sys.stderr.write(proc.stdout + proc.stderr)
        raise RuntimeError("nvcc failed building libsol.so")
    if verbose:
        sys.stderr.write(proc.stderr)
    _check_ptxas_report(proc.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
