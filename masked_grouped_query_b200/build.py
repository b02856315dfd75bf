"""Build ``libgqa_attn.so`` in-tree with nvcc for sm_100a.

Run ``python -m masked_grouped_query_b200.build`` (or ``__graft_entry__.build()``).
The library is a single translation unit, ``csrc/gqa_attn.cu``, with the C ABI
of ``include/gqa_attn.h``; it links the CUDA runtime statically and reaches
the driver's tensor-map encoder through ``cudaGetDriverEntryPoint``.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBRARY = os.path.join(PKG, "libgqa_attn.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def sources() -> list[str]:
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC)
                  if f.endswith((".cu", ".cuh")))


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the library unless it is newer than every source and header."""
    deps = sources() + [os.path.join(INCLUDE, "gqa_attn.h")]
    if (not force and os.path.exists(LIBRARY)
            and os.path.getmtime(LIBRARY) >= max(os.path.getmtime(d) for d in deps)):
        return LIBRARY
    cmd = [nvcc(), *NVCC_FLAGS, f"-I{INCLUDE}", os.path.join(CSRC, "gqa_attn.cu"),
           "-o", LIBRARY + ".tmp"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stderr)
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(LIBRARY + ".tmp", LIBRARY)
    return LIBRARY


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
