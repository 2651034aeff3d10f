"""CPU checks of the C ABI (no GPU needed): the library builds and loads, exports
every entry point include/dsa.h declares, the Python binding mirrors the header
and its struct layouts, and the host-side argument checks return the documented
status codes without launching anything."""

import ctypes
import os
import re
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"DSA_API\s+[\w\s\*]+?\b(dsa_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from sparse_attention_05_b200.build import build
    build()
    from sparse_attention_05_b200 import dsa
    return dsa.lib()


def test_header_declares_the_four_path_calls():
    names = _declared()
    for n in ("dsa_indexer_scores", "dsa_topk", "dsa_sparse_mla_fwd", "dsa_forward"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    from sparse_attention_05_b200 import dsa
    out = subprocess.run(["nm", "-D", "--defined-only", dsa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(dsa_\w+)", out))
    missing = set(_declared()) - exported
    assert not missing, f"not exported: {missing}"


def test_binding_mirrors_header():
    from sparse_attention_05_b200 import dsa
    assert sorted(dsa.SIGNATURES) == _declared()


def test_struct_layouts_match_c():
    from sparse_attention_05_b200 import dsa
    src = r"""
    #include <stdio.h>
    #include <stddef.h>
    #include "dsa.h"
    int main(void) {
      printf("%zu %zu %zu %zu %zu %zu\n", sizeof(dsa_kv_desc_t),
             offsetof(dsa_kv_desc_t, block_table), offsetof(dsa_kv_desc_t, seqlens),
             sizeof(dsa_q_desc_t), offsetof(dsa_q_desc_t, row_count),
             offsetof(dsa_q_desc_t, q_start));
      return 0;
    }
    """
    with tempfile.TemporaryDirectory() as d:
        c, exe = os.path.join(d, "l.c"), os.path.join(d, "l")
        open(c, "w").write(src)
        subprocess.run(["gcc", "-I", os.path.dirname(HEADER), c, "-o", exe], check=True)
        got = [int(x) for x in subprocess.run([exe], capture_output=True, text=True).stdout.split()]
    want = [ctypes.sizeof(dsa.KvDescC), dsa.KvDescC.block_table.offset, dsa.KvDescC.seqlens.offset,
            ctypes.sizeof(dsa.QDescC), dsa.QDescC.row_count.offset, dsa.QDescC.q_start.offset]
    assert got == want


def test_status_strings_and_timeout_setting(lib):
    from sparse_attention_05_b200 import dsa
    assert dsa.dsa_status_string(0) == "DSA_OK"
    assert "TIMEOUT" in dsa.dsa_status_string(4)
    old = dsa.dsa_set_wait_timeout_ns(123)
    assert dsa.dsa_set_wait_timeout_ns(old) == 123


def _kv(batch=2, max_ctx=512, layout=0, page=64, pages=0, max_pages=0, bt=None):
    from sparse_attention_05_b200 import dsa
    d = dsa.KvDescC()
    d.layout, d.batch, d.max_ctx = layout, batch, max_ctx
    d.page_size, d.num_pages, d.max_pages = page, pages, max_pages
    d.block_table = bt
    d.seqlens = None
    return d


def test_host_argument_checks_without_gpu(lib):
    from sparse_attention_05_b200 import dsa
    L = lib
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: the checks fail first
    kv, q = _kv(), dsa.QDescC(2, 1, 0, 0)
    by = ctypes.byref
    # null output
    assert L.dsa_topk(fake, 512, by(kv), by(q), 2048, None, None) == 1
    # k out of range
    assert L.dsa_topk(fake, 512, by(kv), by(q), 4096, fake, None) == 2
    assert L.dsa_topk(fake, 512, by(kv), by(q), 0, fake, None) == 2
    # T != batch * q_per_seq
    bad_q = dsa.QDescC(3, 1, 0, 0)
    assert L.dsa_topk(fake, 512, by(kv), by(bad_q), 2048, fake, None) == 1
    # row window outside the sequence
    assert L.dsa_topk(fake, 512, by(kv), by(dsa.QDescC(2, 1, 1, 0)), 2048, fake, None) == 1
    # ragged batch: more query rows than batch * q_per_seq, or a negative count
    assert L.dsa_topk(fake, 512, by(kv), by(dsa.QDescC(5, 2, 0, 0, 0x3000)), 2048, fake,
                      None) == 1
    assert L.dsa_topk(fake, 512, by(kv), by(dsa.QDescC(-1, 2, 0, 0, 0x3000)), 2048, fake,
                      None) == 1
    # top-k score rows must be 16-byte aligned
    assert L.dsa_topk(fake, 514, by(kv), by(q), 2048, fake, None) == 1
    # ld below max_ctx rounded to 128
    assert L.dsa_indexer_scores(fake, fake, fake, fake, by(kv), by(q), fake, 500, None) == 1
    # misaligned pointer
    assert L.dsa_indexer_scores(ctypes.c_void_p(0x1001), fake, fake, fake, by(kv), by(q), fake,
                                512, None) == 1
    # paged: page size not a multiple of 64, missing block table
    pk = _kv(layout=1, page=48, pages=4, max_pages=16, bt=0x2000)
    assert L.dsa_sparse_mla_fwd(fake, fake, by(pk), by(q), fake, 2048, 0.04, fake, fake, None) == 2
    pk = _kv(layout=1, page=64, pages=4, max_pages=16, bt=None)
    assert L.dsa_sparse_mla_fwd(fake, fake, by(pk), by(q), fake, 2048, 0.04, fake, fake, None) == 1
    # scale must be positive and finite
    assert L.dsa_sparse_mla_fwd(fake, fake, by(kv), by(q), fake, 2048, -1.0, fake, fake, None) == 1
    # workspace too small / misaligned
    ws_need = L.dsa_workspace_size(by(kv), by(q), 2048)
    assert ws_need >= 2 * 2048 * 4
    assert L.dsa_forward(fake, fake, fake, fake, fake, fake, by(kv), by(q), 2048, 0.04,
                         ctypes.c_void_p(0x1000), 16, None, fake, fake, None) == 6
    assert L.dsa_forward(fake, fake, fake, fake, fake, fake, by(kv), by(q), 2048, 0.04,
                         ctypes.c_void_p(0x1010), ws_need, None, fake, fake, None) == 6


def test_workspace_size_plan(lib):
    from sparse_attention_05_b200 import dsa
    by = ctypes.byref
    def split(rows):  # the split top-k's candidates (8192 keys + positions), counts, thresholds
        return rows * 8192 * 8 + 2 * ((rows * 4 + 255) // 256 * 256)
    # decode, 64 x 32768: indices + all score rows in one chunk (the forward's top-k
    # is one CTA per row); dsa_topk_ws's split scratch on its own
    kv, q = _kv(batch=64, max_ctx=32768), dsa.QDescC(64, 1, 0, 0)
    n = lib.dsa_workspace_size(by(kv), by(q), 2048)
    assert n == 64 * 2048 * 4 + 64 * 32768 * 4
    assert lib.dsa_topk_workspace_size(by(kv), by(q), 2048) == split(64)
    # prefill 131072: indices + one 2 GiB chunk of score rows
    kv, q = _kv(batch=1, max_ctx=131072), dsa.QDescC(131072, 131072, 0, 0)
    n = lib.dsa_workspace_size(by(kv), by(q), 2048)
    assert n == 131072 * 2048 * 4 + 4096 * 131072 * 4
    # dsa_topk_ws's scratch for one 4096-row window of it
    q = dsa.QDescC(131072, 131072, 0, 4096)
    assert lib.dsa_topk_workspace_size(by(kv), by(q), 2048) == split(4096)
    # rows no longer than 4k keys, or longer than the selection bitmaps: no split
    kv, q = _kv(batch=4, max_ctx=8192), dsa.QDescC(4, 1, 0, 0)
    assert lib.dsa_topk_workspace_size(by(kv), by(q), 2048) == 0
    kv, q = _kv(batch=1, max_ctx=131073), dsa.QDescC(1, 1, 0, 0)
    assert lib.dsa_topk_workspace_size(by(kv), by(q), 2048) == 0
    # invalid geometry -> 0
    assert lib.dsa_workspace_size(by(kv), by(dsa.QDescC(5, 131072, 0, 0)), 2048) == 0


@pytest.mark.parametrize("batch,q_per_seq,max_ctx,k", [
    (4, 1, 4096, 2048),      # one partial wave: every row split (7 segments)
    (40, 2, 512, 2048),      # 80 rows: a 6-row tail after one wave of 74
    (1, 1500, 1500, 2048),   # prefill: 20-row tail, 3 segments
    (3, 1, 300, 100),        # too few key blocks to split
    (37, 2, 256, 2048),      # exactly one full wave: no split
])
def test_workspace_size_includes_the_split_rows(lib, batch, q_per_seq, max_ctx, k):
    """Without a GPU the library plans for 148 SMs; the benchmark's mirror of the
    split rule must give the same scratch the library reserves."""
    from bench import MLA_PART_BYTES, mla_split_plan
    from sparse_attention_05_b200 import dsa
    by = ctypes.byref
    kv, q = _kv(batch=batch, max_ctx=max_ctx), dsa.QDescC(batch * q_per_seq, q_per_seq, 0, 0)
    n = lib.dsa_workspace_size(by(kv), by(q), k)
    rows = batch * q_per_seq
    idx = -(-rows * k * 4 // 256) * 256
    ld = -(-max_ctx // 128) * 128
    score = -(-min(q_per_seq, max(1, (2 << 30) // (ld * 4 * batch))) * batch * ld * 4 // 256) * 256
    n_split, nseg = mla_split_plan(rows, k, 1 << 62, sms=148)
    part = -(-n_split * nseg * MLA_PART_BYTES // 256) * 256
    assert n == idx + max(score, part)
    assert lib.dsa_sparse_mla_workspace_size() == 74 * MLA_PART_BYTES


def test_every_binding_call_that_forwards_q_start_accepts_it():
    """Each wrapper that builds a query descriptor takes the ragged offsets."""
    import inspect
    from sparse_attention_05_b200 import dsa
    for name in sorted(dsa.SIGNATURES):
        fn = getattr(dsa, name, None)
        if fn is None:
            continue
        src = inspect.getsource(fn)
        if "_qdesc(" in src:
            assert "q_start" in inspect.signature(fn).parameters, name
