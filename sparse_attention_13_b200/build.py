"""Builds the in-tree shared libraries with nvcc for sm_100a.

libdsa.so       -- the C ABI of include/dsa.h (kernels + host logic)
libdsa_synth.so -- the seeded synthetic-input generator (test/bench inputs)
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-shared",
                "-cudart", "static", "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]

LIBS = {
    "libdsa.so": ["dsa_api.cu", "indexer_topk.cu", "decode_indexer.cu", "sparse_attn.cu", "noalloc.cu",
                  "selection_quality.cu", "csa.cu", "lowprec.cu"],
    "libdsa_synth.so": ["synth.cu"],
}
DEPS = ["dsa_ptx.cuh", "dsa_internal.h"]


def _stale(out: str, srcs: list[str]) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    deps = srcs + [os.path.join(CSRC, d) for d in DEPS] + [os.path.join(ROOT, "include", "dsa.h")]
    return any(os.path.getmtime(s) > t for s in deps)


def build(force: bool = False, verbose: bool = False) -> None:
    for lib, names in LIBS.items():
        out = os.path.join(HERE, lib)
        srcs = [os.path.join(CSRC, n) for n in names]
        if not force and not _stale(out, srcs):
            continue
        cmd = [NVCC] + FLAGS + (["-Xptxas", "-v"] if verbose else []) + ["-o", out] + srcs
        print("[build]", " ".join(cmd), flush=True)
        subprocess.check_call(cmd)


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
