"""Build libbsmt.so in-tree for sm_100a with nvcc.

Usage: python block_sparse_masked_tile_b200/build.py [--verbose-ptxas]

Run it as a script (or load it by path): importing it through the package
would first try to load the library it builds.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libbsmt.so")
SOURCES = ["bsmt.cu"]
HEADERS = sorted(f for f in os.listdir(CSRC) if f.endswith(".cuh"))


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "bsmt.h"), __file__]
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    if not force and not needs_build():
        return LIB
    cmd = [
        nvcc(), "-shared", "-Xcompiler", "-fPIC", "-std=c++17", "-O3", "-lineinfo",
        "-gencode", "arch=compute_100a,code=sm_100a",
        "--expt-relaxed-constexpr",
        "-I", INCLUDE, "-I", CSRC,
        "-o", LIB + ".tmp",
    ] + [os.path.join(CSRC, f) for f in SOURCES] + ["-lcudart"]
    cmd[1:1] = ["-Xptxas", "-v"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if ptxas_verbose or res.returncode != 0:
        sys.stderr.write(res.stderr)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed")
    check_attention_registers(res.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


# The attention kernels (forward and backward) are sized for 168 registers per
# thread (384 threads, one CTA per SM, split further by setmaxnreg); a
# different count means the launch or the layout changed.
LAUNCH_REGS = 168


def check_attention_registers(ptxas_log: str) -> None:
    current = None
    seen = 0
    for line in ptxas_log.splitlines():
        if "Compiling entry function" in line:
            current = line
        elif "Used" in line and "registers" in line and current and (
                "attn_fwd_kernel" in current or "attn_bwd_kernel" in current):
            regs = int(line.split("Used")[1].split("registers")[0])
            seen += 1
            if regs != LAUNCH_REGS:
                raise RuntimeError(f"attention kernel compiled to {regs} registers, expected {LAUNCH_REGS}")
    if seen == 0:
        raise RuntimeError("ptxas report has no attention kernel entries")


if __name__ == "__main__":
    build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv)
    print(LIB)
