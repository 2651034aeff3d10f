"""Build libdsa.so (the C-ABI library of include/dsa.h) in-tree for sm_100a.

Usage: python -m sparse_attention_05_b200.build   (or __graft_entry__.build())
"""

from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libdsa.so")
SOURCES = ["dsa_api.cu"]
HEADERS = ["ptx.cuh", "rows.cuh", "topk.cuh", "indexer.cuh", "sparse_mla.cuh", "indexer_kl.cuh",
           "mha_prefill.cuh"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    home = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    cand = os.path.join(home, "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


# the header that holds each kernel (for per-kernel digests)
KERNEL_HEADER = {"indexer": "indexer.cuh", "topk": "topk.cuh", "sparse_mla": "sparse_mla.cuh",
                 "indexer_kl": "indexer_kl.cuh", "mask": "mha_prefill.cuh",
                 "up_proj": "mha_prefill.cuh", "masked_mha": "mha_prefill.cuh"}


def source_digest(kernel=None) -> str:
    """Digest of the CUDA sources and the ABI header (identifies a library build);
    with ``kernel``, of that kernel's header and the shared PTX and row helpers only."""
    import hashlib
    h = hashlib.sha256()
    files = (["ptx.cuh", "rows.cuh", KERNEL_HEADER[kernel]] if kernel else SOURCES + HEADERS)
    for f in files:
        h.update(open(os.path.join(CSRC, f), "rb").read())
    if not kernel:
        h.update(open(os.path.join(ROOT, "include", "dsa.h"), "rb").read())
    return h.hexdigest()[:16]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "dsa.h"))
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    cmd = [_nvcc(), *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"),
           *[os.path.join(CSRC, s) for s in SOURCES], "-o", LIB + ".tmp"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
