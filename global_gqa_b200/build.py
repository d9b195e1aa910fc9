"""Builds libg3attn.so (the C-ABI library) in-tree with nvcc for sm_100a.

Usage: python -m global_gqa_b200.build  [--force] [--verbose]
"""
from __future__ import annotations

import argparse
import hashlib
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
SOURCES = ["api.cu", "prologue.cu", "prefill.cu", "decode.cu", "decode_static.cu", "projector.cu", "backward.cu", "backward256.cu"]
HEADERS = ["g3_internal.h", "sm100_ptx.cuh", "tmem_wide.cuh", "func_attr.cuh", "backward_common.cuh", os.path.join("..", "..", "include", "g3attn.h")]
LIB = os.path.join(HERE, "libg3attn.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC,-O2",
         "-Xptxas", "-v"]


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found")
    return cand


def _digest() -> str:
    h = hashlib.sha256()
    for f in SOURCES + HEADERS:
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    h.update(" ".join(ARCH + FLAGS).encode())
    return h.hexdigest()


# Test-only variant (never the product library): waits give up after 20 ms
# instead of 2 s, and g3attn_test_withhold_s_commit() lets a test make the MMA
# thread of one CTA skip one "S ready" arrival, so that the softmax warps'
# bounded wait runs out (tests/test_gpu_timeout.py).
FAULT_LIB = os.path.join(ROOT, "_build", "fault_inject", "libg3attn_fault_inject.so")
FAULT_FLAGS = ["-DG3_FAULT_INJECT", "-DG3_WAIT_TIMEOUT_NS=20000000ull"]


def _compile_all(objdir: str, extra: list) -> list:
    """Compiles every source into objdir in parallel; returns the ptxas logs."""
    from concurrent.futures import ThreadPoolExecutor
    os.makedirs(objdir, exist_ok=True)

    def one(src):
        obj = os.path.join(objdir, src.replace(".cu", ".o"))
        cmd = [nvcc(), *ARCH, *FLAGS, *extra, "-I", os.path.join(ROOT, "include"), "-c",
               os.path.join(CSRC, src), "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        return src, obj, r

    with ThreadPoolExecutor(max_workers=min(len(SOURCES), os.cpu_count() or 1)) as ex:
        done = list(ex.map(one, SOURCES))
    for src, _, r in done:
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError(f"nvcc failed on {src}")
    return [obj for _, obj, _ in done], [r.stdout + r.stderr for _, _, r in done]


def build_fault_inject(force: bool = False) -> str:
    """The test-only library with short waits and the withheld-arrival hook."""
    stamp = FAULT_LIB + ".sha256"
    dig = _digest() + " ".join(FAULT_FLAGS)
    if not force and os.path.exists(FAULT_LIB) and os.path.exists(stamp):
        with open(stamp) as f:
            if f.read().strip() == dig:
                return FAULT_LIB
    objs, _ = _compile_all(os.path.dirname(FAULT_LIB), FAULT_FLAGS)
    tmp = FAULT_LIB + ".tmp"
    r = subprocess.run([nvcc(), *ARCH, "-shared", "-o", tmp, *objs], capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("link failed")
    os.replace(tmp, FAULT_LIB)
    with open(stamp, "w") as f:
        f.write(dig)
    return FAULT_LIB


def build(force: bool = False, verbose: bool = False) -> str:
    stamp = LIB + ".sha256"
    dig = _digest()
    if not force and os.path.exists(LIB) and os.path.exists(stamp):
        with open(stamp) as f:
            if f.read().strip() == dig:
                return LIB
    objdir = os.path.join(ROOT, "_build")
    objs, logs = _compile_all(objdir, [])
    tmp = LIB + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("link failed")
    os.replace(tmp, LIB)
    with open(os.path.join(objdir, "ptxas.log"), "w") as f:
        f.write("\n".join(logs))
    with open(stamp, "w") as f:
        f.write(dig)
    if verbose:
        print("\n".join(logs))
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--fault-inject", action="store_true", help="also build the test-only library")
    a = ap.parse_args()
    print(build(a.force, a.verbose))
    if a.fault_inject:
        print(build_fault_inject(a.force))
