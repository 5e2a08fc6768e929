"""Builds the CUDA shared library ``libattn_b200.so`` in-tree with nvcc for sm_100a.

The library is the whole compute path (prefill, tile map, split-KV decode, merge) behind the
C ABI declared in ``include/attn.h``; nothing else is compiled.  No GPU is needed to build.

    python -m io_aware_softmax_b200.build [--force] [--verbose]
"""
from __future__ import annotations

import argparse
import os
import re
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
LIB_NAME = "libattn_b200.so"
LIB_PATH = os.path.join(PKG_DIR, LIB_NAME)
SOURCES = ["attn_api.cu", "attn_prefill.cu", "attn_decode.cu", "attn_blockmap.cu",
           "attn_decode_noalloc.cu", "attn_backward.cu", "attn_fp8.cu"]
HEADERS = ["attn_internal.h", "mask.cuh", "sm100_ptx.cuh", "tmem_ldst.cuh"]
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]

# The prefill kernel splits its launch registers between warpgroups with setmaxnreg
# (two softmax warpgroups, one warpgroup of MMA/TMA warps, 384 threads).  The split must fit
# in what the CTA is launched with, or the increase would wait forever: check the count
# ptxas chose against the split constants read from the kernel source.
PREFILL_KERNEL = "attn_fwd_sm100_kernel"
PREFILL_THREADS = 384


def _prefill_split_regs() -> int:
    src = open(os.path.join(CSRC, "attn_prefill.cu"), encoding="utf-8").read()
    soft = int(re.search(r"kRegsSoftmax\s*=\s*(\d+)", src).group(1))
    other = int(re.search(r"kRegsOther\s*=\s*(\d+)", src).group(1))
    return 2 * 128 * soft + 128 * other


PREFILL_SPLIT_REGS = _prefill_split_regs()


def check_register_budget(ptxas_log: str) -> dict:
    """Launch register counts of the prefill kernels from ``-Xptxas -v`` output; raises if
    the setmaxnreg split would not fit."""
    counts = {}
    current = None
    for line in ptxas_log.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            current = m.group(1)
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and current is not None:
            counts[current] = int(m.group(1))
            current = None
    found = {k: v for k, v in counts.items() if PREFILL_KERNEL in k}
    if not found:
        raise RuntimeError("ptxas output lists no prefill kernel; cannot check registers")
    for name, regs in found.items():
        if regs * PREFILL_THREADS < PREFILL_SPLIT_REGS:
            raise RuntimeError(f"{name}: launched with {regs} registers/thread, the warpgroup "
                               f"split needs {PREFILL_SPLIT_REGS / PREFILL_THREADS:.1f}")
    return found


def nvcc_path() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libattn_b200")
    return cand


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    files.append(os.path.join(ROOT, "include", "attn.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB_PATH):
        return False
    t = os.path.getmtime(LIB_PATH)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB_PATH
    cmd = [nvcc_path(), *ARCH_FLAGS, "-O3", "-lineinfo", "-std=c++17", "-shared",
           "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
           "-I", os.path.join(ROOT, "include"), "-Xptxas", "-v", "-o", LIB_PATH + ".tmp"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    log = res.stdout + res.stderr
    if "setmaxnreg' ignored" in log:
        os.remove(LIB_PATH + ".tmp")
        raise RuntimeError("ptxas ignored setmaxnreg; the warpgroup register split is lost")
    try:
        check_register_budget(log)
    except RuntimeError:
        os.remove(LIB_PATH + ".tmp")
        raise
    if verbose:
        sys.stderr.write(log)
    with open(os.path.join(PKG_DIR, "ptxas_info.txt"), "w") as f:
        f.write(log)
    os.replace(LIB_PATH + ".tmp", LIB_PATH)
    return LIB_PATH


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args(argv)
    print(build(force=a.force, verbose=a.verbose))


if __name__ == "__main__":
    main()
