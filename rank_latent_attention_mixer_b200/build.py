"""Builds the CUDA library libflarepp.so in-tree for sm_100a with nvcc.

    python -m rank_latent_attention_mixer_b200.build [--verbose-ptxas]
"""
from __future__ import annotations

import glob
import os
import re
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libflarepp.so")
ROOT = os.path.dirname(PKG)

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    "-I", os.path.join(ROOT, "include"),
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = glob.glob(os.path.join(CSRC, "*")) + glob.glob(os.path.join(ROOT, "include", "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


# The tcgen05 kernel splits its launch registers between warpgroups with
# setmaxnreg (softmax warpgroups grow, the producer warpgroup shrinks).  The
# split is sized for exactly 65536 / threads registers per thread at launch
# (rounded down to a multiple of 8); a smaller launch allocation would leave
# the growing warpgroups waiting, so the build refuses any other count.  The
# kernel's template arguments are <D, NW, KT, NST, QS, MODE, CS>, threads =
# (NW*CS+1)*128.


# The backward kernel bwd_kernel<E, D, NW, DUAL> splits its registers the same
# way when NW = 2 (384 threads: 168 at launch); with NW = 1 it does not split.


def expected_launch_regs(kernel_name: str):
    if "bwd_kernel" in kernel_name:
        m = re.search(r"bwd_kernelI\d+\w+?Li(\d+)ELi(\d+)ELb[01]E", kernel_name)
        if not m:
            raise RuntimeError(f"cannot read the warpgroup count from {kernel_name}")
        nw = int(m.group(2))
        return (65536 // ((nw + 1) * 128)) // 8 * 8 if nw == 2 else None
    # attn_kernel<E, D, NW, KT, NST, QS, MODE, CS>: NW row tiles x CS column
    # shares softmax warpgroups and one producer warpgroup
    m = re.search(r"attn_kernelI\d+\w+?((?:Li\d+E){7})", kernel_name)
    if not m:
        raise RuntimeError(f"cannot read the warpgroup count from {kernel_name}")
    args = [int(x) for x in re.findall(r"Li(\d+)E", m.group(1))]
    nw, cs = args[1], args[6]
    return (65536 // ((nw * cs + 1) * 128)) // 8 * 8


def check_registers(ptxas_log: str) -> None:
    current = None
    found = 0
    for line in ptxas_log.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            current = m.group(1)
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and current and ("attn_kernel" in current or "bwd_kernel" in current):
            found += 1
            regs = int(m.group(1))
            want = expected_launch_regs(current)
            if want is not None and regs != want:
                raise RuntimeError(f"{current}: ptxas allocated {regs} registers per thread, the register split "
                                   f"needs exactly {want}; refusing to build")
    if found == 0:
        raise RuntimeError("no attn_kernel register report found in the ptxas log")


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and not _stale():
        return LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc, *NVCC_FLAGS, "-Xptxas", "-v", "-o", tmp, *sources()]
    res = subprocess.run(cmd, capture_output=True, text=True)
    log = res.stdout + res.stderr
    if res.returncode != 0:
        errors = "\n".join(line for line in log.splitlines() if "error" in line) or log[-4000:]
        raise RuntimeError(f"nvcc failed (exit {res.returncode}):\n{errors}")
    if verbose_ptxas:
        print(log)
    try:
        check_registers(log)
    except Exception:
        os.remove(tmp)
        raise
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv))
