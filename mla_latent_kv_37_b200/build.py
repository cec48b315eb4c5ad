"""Builds libmla_b200.so (all kernels and the C ABI) in-tree for sm_100a with nvcc."""
from __future__ import annotations

import os
import re
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libmla_b200.so")
SOURCES = [os.path.join(HERE, "csrc", "mla_api.cu")]
DEPS = [os.path.join(HERE, "csrc", f) for f in sorted(os.listdir(os.path.join(HERE, "csrc")))] + [
    os.path.join(ROOT, "include", "mla.h")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(out: str = LIB, extra=()) -> list[str]:
    return [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
            "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"),
            *extra, "-o", out, *SOURCES]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in DEPS)


# When the decode split kernel re-divides its registers between warpgroups (setmaxnreg), the
# division assumes it is compiled to exactly kLaunchRegs registers per thread.
SPLIT_KERNEL = "_ZN3mla4attn12split_kernel"


def split_kernel_regs() -> int:
    with open(os.path.join(HERE, "csrc", "attn_sm100.cuh")) as f:
        m = re.search(r"constexpr int kLaunchRegs = (\d+);", f.read())
    return int(m.group(1)) if m else 0


def check_split_kernel_regs(ptxas_log: str) -> None:
    want = split_kernel_regs()
    if want == 0:
        return
    lines = ptxas_log.splitlines()
    for i, ln in enumerate(lines):
        if "Function properties for" in ln and SPLIT_KERNEL in ln:
            for nxt in lines[i + 1:i + 4]:
                m = re.search(r"Used (\d+) registers", nxt)
                if m:
                    if int(m.group(1)) != want:
                        raise RuntimeError(f"split_kernel compiled to {m.group(1)} registers per "
                                           f"thread, expected {want}")
                    return
    raise RuntimeError("ptxas did not report the register count of split_kernel")


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    tmp = LIB + ".tmp"
    cmd = command(tmp, extra=("-Xptxas", "-v"))
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    res = subprocess.run(cmd, check=True, capture_output=True, text=True)
    check_split_kernel_regs(res.stdout + res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    print(LIB)
