"""The CUDA sources compile for sm_100a (no GPU needed) and no kernel spills
registers to local memory: a spill in one of the hot loops would cost more than any
tuning of it gains. The library is built into a temporary directory with the
package's own flags, so the in-tree libdsa.so is left alone."""

import os
import re
import subprocess
import tempfile

import pytest

from sparse_attention_05_b200 import build as B

KERNELS = ["indexer_kernel", "topk_kernel", "cand_select_kernel", "sparse_mla_kernel",
           "mla_combine_kernel", "indexer_kl_kernel", "mla_up_proj_kernel",
           "selection_mask_kernel", "masked_mha_kernel"]


@pytest.fixture(scope="module")
def ptxas_report():
    with tempfile.TemporaryDirectory() as d:
        cmd = [B._nvcc(), "-Xptxas=-v", *B.NVCC_FLAGS, "-I", os.path.join(B.ROOT, "include"),
               *[os.path.join(B.CSRC, s) for s in B.SOURCES], "-o", os.path.join(d, "lib.so")]
        r = subprocess.run(cmd, capture_output=True, text=True)
        assert r.returncode == 0, r.stderr[-2000:]
        return r.stdout + r.stderr


def _entries(report):
    """(mangled entry name, the report lines that follow it) per compiled kernel."""
    out, cur = [], None
    for line in report.splitlines():
        m = re.search(r"Compiling entry function '([^']+)' for 'sm_100a'", line)
        if m:
            cur = [m.group(1), []]
            out.append(cur)
        elif cur is not None:
            cur[1].append(line)
    return out


def test_every_kernel_compiles_for_sm100a(ptxas_report):
    names = [n for n, _ in _entries(ptxas_report)]
    for k in KERNELS:
        assert any(k in n for n in names), f"{k} missing from the build"


def test_no_kernel_spills(ptxas_report):
    for name, lines in _entries(ptxas_report):
        text = " ".join(lines[:4])
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", text)
        assert m, f"no spill report for {name}"
        assert m.group(1) == "0" and m.group(2) == "0", f"{name} spills: {m.group(0)}"
