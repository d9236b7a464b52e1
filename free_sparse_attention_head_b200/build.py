"""Builds libsvoo.so (the C-ABI CUDA library) in-tree for sm_100a with nvcc.

It also links libsvoo_stall.so, a test-only variant whose pipelined kernels
(attention, clustering assignment) are compiled with SVOO_TEST_STALL: one
pipeline wait on a barrier that nothing completes and a pipeline wait budget
of about 10 ms, so a test can drive the device timeout path and read the
error word. No product code loads it.

    python -m free_sparse_attention_head_b200.build [--force]
"""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libsvoo.so")
STALL_LIB = os.path.join(HERE, "libsvoo_stall.so")
SOURCES = ["api.cu", "cluster.cu", "mask.cu", "permute.cu", "attn.cu", "psa.cu"]
STALL_SOURCES = ["cluster.cu", "attn.cu"]  # the kernels with pipeline waits
HEADERS = ["common.cuh", "internal.h"]
INCLUDE = os.path.join(os.path.dirname(HERE), "include")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC",
    "-diag-suppress", "177",
]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _newest_input() -> float:
    paths = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    paths.append(os.path.join(INCLUDE, "svoo.h"))
    return max(os.path.getmtime(p) for p in paths)


def _link(out: str, objs) -> None:
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call([_nvcc(), "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-o", tmp, *objs])
    os.replace(tmp, out)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every .cu to an object and link libsvoo.so (and the test-only
    libsvoo_stall.so); skipped when both are up to date."""
    newest = _newest_input()
    if (not force and all(os.path.exists(p) and os.path.getmtime(p) >= newest
                          for p in (LIB, STALL_LIB))):
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    jobs = []  # (source, object, extra flags)
    for src in SOURCES:
        jobs.append((src, os.path.join(BUILD, src.replace(".cu", ".o")), []))
    for src in STALL_SOURCES:
        jobs.append((src, os.path.join(BUILD, src.replace(".cu", "_stall.o")), ["-DSVOO_TEST_STALL"]))

    def compile_one(job):
        src, obj, extra = job
        cmd = [_nvcc(), *NVCC_FLAGS, *extra, "-I", INCLUDE, "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.check_call(cmd)

    with ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 1)) as ex:
        list(ex.map(compile_one, jobs))
    _link(LIB, [os.path.join(BUILD, src.replace(".cu", ".o")) for src in SOURCES])
    _link(STALL_LIB, [os.path.join(BUILD, src.replace(".cu", "_stall.o") if src in STALL_SOURCES
                                   else src.replace(".cu", ".o")) for src in SOURCES])
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    print(LIB)
