"""Build libsala.so in-tree with nvcc for sm_100a (no GPU needed to compile)."""
from __future__ import annotations

import json
import os
import re
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libsala.so")
SOURCES = ["api.cu"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
    "--expt-relaxed-constexpr",
    # the decoder block's GEMMs
    "-lcublasLt", "-Xlinker", "-rpath,/usr/local/cuda/lib64",
]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(ROOT, "include", "sala.h")]
    return any(os.path.getmtime(p) > t for p in deps if os.path.isfile(p))


# Kernels whose in-kernel register reallocation (setmaxnreg) is sized for a
# fixed launch allocation: the build fails unless ptxas gave each exactly
# this many registers per thread, so a library that built cannot hang on a
# register split larger than its launch allocation.
REGISTER_SPLIT_KERNELS = {"linear_segout_kernel": 128}
REPORT = os.path.join(PKG, "libsala.ptxas.json")


def parse_ptxas(text: str) -> dict:
    """{mangled kernel name: registers per thread} from `ptxas -v` output."""
    regs, cur = {}, None
    for line in text.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            cur = m.group(1)
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and cur:
            regs[cur] = int(m.group(1))
            cur = None
    return regs


def check_register_splits(regs: dict) -> None:
    for short, want in REGISTER_SPLIT_KERNELS.items():
        got = {k: v for k, v in regs.items() if short in k}
        if not got:
            raise RuntimeError(f"ptxas report has no entry for {short}")
        bad = {k: v for k, v in got.items() if v != want}
        if bad:
            raise RuntimeError(f"{short}: built with {sorted(set(bad.values()))} registers per "
                               f"thread; its register split needs exactly {want}")


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    if not force and not needs_build():
        return LIB
    cmd = [nvcc_path(), *NVCC_FLAGS, "-Xptxas", "-v", *extra, "-I", os.path.join(ROOT, "include"),
           "-o", LIB + ".tmp", *[os.path.join(CSRC, s) for s in SOURCES]]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise subprocess.CalledProcessError(r.returncode, cmd)
    cur = ""
    for line in (r.stdout + r.stderr).splitlines():
        m = re.search(r"Function properties for (\S+)", line)
        if m:
            cur = m.group(1)
        if re.search(r"[1-9]\d* bytes spill", line) or "warning" in line.lower():
            sys.stderr.write(f"{cur}: {line.strip()}\n")
    regs = parse_ptxas(r.stdout + r.stderr)
    check_register_splits(regs)
    with open(REPORT, "w") as f:
        json.dump({"registers_per_thread": regs}, f, indent=1, sort_keys=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    print(LIB)
