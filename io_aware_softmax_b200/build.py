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
HEADERS = ["attn_internal.h", "mask.cuh", "sm100_ptx.cuh", "tmem_ldst.cuh", "tanh_poly.cuh"]
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]

# Kernels that split their launch registers between warpgroups with setmaxnreg (two
# element-wise / softmax warpgroups and one warpgroup of MMA/TMA warps, 384 threads).  A split
# must fit in what the CTA is launched with, or the increase would wait forever: the build
# checks the count ptxas chose against the split constants read from each kernel's source.
# (kernel name fragment, source, constant of the two big warpgroups, constant of the third)
SPLIT_KERNELS = [
    ("attn_fwd_sm100_kernel", "attn_prefill.cu", "kRegsSoftmax", "kRegsOther"),
    ("attn_fwd_sm100_kernel", "attn_prefill.cu", "kRegsSoftmaxCap", "kRegsOtherCap"),
    ("attn_bwd_dq_kernel", "attn_backward.cu", "kBwdRegsElem", "kBwdRegsOther"),
    ("attn_bwd_dkdv_kernel", "attn_backward.cu", "kBwdRegsElem", "kBwdRegsOther"),
]
SPLIT_THREADS = 384
PREFILL_KERNEL = SPLIT_KERNELS[0][0]
PREFILL_THREADS = SPLIT_THREADS


def split_regs(source: str, big: str, other: str) -> int:
    src = open(os.path.join(CSRC, source), encoding="utf-8").read()
    n_big = int(re.search(big + r"\s*=\s*(\d+);", src).group(1))
    n_other = int(re.search(other + r"\s*=\s*(\d+);", src).group(1))
    return 2 * 128 * n_big + 128 * n_other


PREFILL_SPLIT_REGS = split_regs(*SPLIT_KERNELS[0][1:])


def check_register_budget(ptxas_log: str) -> dict:
    """Launch register counts of the kernels that split registers, from ``-Xptxas -v``
    output; raises if a split would not fit or a kernel is missing."""
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
    found = {}
    for frag, source, big, other in SPLIT_KERNELS:
        need = split_regs(source, big, other)
        hits = {k: v for k, v in counts.items() if frag in k}
        if not hits:
            raise RuntimeError(f"ptxas output lists no {frag}; cannot check registers")
        for name, regs in hits.items():
            if regs * SPLIT_THREADS < need:
                raise RuntimeError(f"{name}: launched with {regs} registers/thread, the "
                                   f"warpgroup split needs {need / SPLIT_THREADS:.1f}")
        found.update(hits)
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
