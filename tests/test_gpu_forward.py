"""End-to-end GPU parity of dsa_forward (indexer -> top-k -> sparse MLA)
against the oracle: index sets equal up to near-ties at the k-th score, and the
attention output equal to the oracle's attention over the selected set. Also
the chunked path (small workspace), caller-provided index output, host errors
and the bounded-wait timeout self test."""

import numpy as np
import pytest
import torch

from oracle import indexer_scores, sparse_mla, topk_rows
from sparse_attention_05_b200 import synth
from tests.helpers import check_attention, check_index_sets, oracle_args

pytestmark = pytest.mark.gpu


def _dsa():
    from sparse_attention_05_b200 import dsa
    return dsa


def _gpu_forward(p, workspace_bytes=None, k=2048):
    dsa = _dsa()
    g = p.to("cuda")
    kv = dsa.KvLayout.of(g)
    ws = None
    if workspace_bytes is not None:
        ws = torch.empty(workspace_bytes, dtype=torch.uint8, device="cuda")
    idx = torch.empty(p.num_q, k, dtype=torch.int32, device="cuda")
    out, lse, _ = dsa.dsa_forward(g.q_idx, g.w, g.k_idx, g.k_scale, g.q, g.kv, kv, p.q_per_seq,
                                  k, p.scale, workspace=ws, idx_out=idx)
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == 0
    return idx.cpu().numpy(), out.float().cpu().numpy(), lse.cpu().numpy()


def _check_forward(p, rows=None, workspace_bytes=None, k=2048):
    idx_g, o_g, l_g = _gpu_forward(p, workspace_bytes, k)
    a = oracle_args(p)
    rows = np.arange(p.num_q) if rows is None else np.asarray(rows)
    ld = (p.max_ctx + 127) // 128 * 128
    sc = indexer_scores(a["q_idx"], a["w"], a["k_idx"], a["k_scale"], a["q_seq"], a["q_pos"],
                        ld=ld, rows=rows, block_table=a["block_table"], page_size=p.page_size)
    idx_r = topk_rows(sc, a["q_pos"], k, rows=rows)
    nd = check_index_sets(idx_g[rows], idx_r, sc, a["q_pos"][rows], k)
    o_r, l_r = sparse_mla(a["q"], a["kv"], a["q_seq"], a["q_pos"], idx_g[rows], p.scale, 512,
                          rows=rows, block_table=a["block_table"], page_size=p.page_size)
    check_attention(o_g[rows], l_g[rows], o_r, l_r)
    return nd


def test_decode_contiguous():
    p = synth.decode(batch=4, ctx=5000, q_per_seq=1, seed=50)
    _check_forward(p)


def test_paged_two_queries_per_sequence():
    p = synth.paged_decode(batch=3, q_per_seq=2, min_ctx=1000, max_ctx=6000, seed=51)
    _check_forward(p)


def test_prefill_rows_below_and_above_k():
    p = synth.prefill(L=3000, seed=52)
    rows = synth.sample_rows(3000, 12, seed=3, must=(0, 1, 2047, 2048, 2999)).numpy()
    _check_forward(p, rows)


def test_chunked_small_workspace_matches():
    dsa = _dsa()
    p = synth.prefill(L=1500, seed=53)
    need = dsa.dsa_workspace_size(dsa.KvLayout.of(p.to("cuda")), 1500, 1500, 2048)
    ld = (1500 + 127) // 128 * 128
    small = 1500 * 2048 * 4 + 5 * ld * 4 + 256  # indices + about 5 score rows -> chunks of 4
    assert small < need
    full = _gpu_forward(p)
    chunked = _gpu_forward(p, workspace_bytes=small)
    np.testing.assert_array_equal(chunked[0], full[0])   # the selection, bit for bit
    # The attention of the rows of a partly filled last wave is split into key
    # segments when the workspace holds their partial outputs (the full one does,
    # the small one does not): those rows agree up to rounding, the others exactly.
    wave = torch.cuda.get_device_properties(0).multi_processor_count // 2
    n_whole = 1500 - 1500 % wave
    np.testing.assert_array_equal(chunked[1][:n_whole], full[1][:n_whole])
    np.testing.assert_array_equal(chunked[2][:n_whole], full[2][:n_whole])
    assert np.abs(chunked[2] - full[2]).max() <= 5e-5
    assert np.all(np.abs(chunked[1] - full[1]) <= 2.0 ** -7 * np.abs(chunked[1]) + 2e-3)
    rows = np.array([0, 5, 777, 1499])
    _check_forward(p, rows, workspace_bytes=small)


def test_full_size_decode_sampled_rows():
    p = synth.decode(batch=64, ctx=32768, q_per_seq=1, seed=1)
    rows = synth.sample_rows(64, 4, seed=4, must=(0, 63)).numpy()
    _check_forward(p, rows)


def test_workspace_errors():
    dsa = _dsa()
    p = synth.decode(batch=2, ctx=512, q_per_seq=1, seed=54).to("cuda")
    kv = dsa.KvLayout.of(p)
    tiny = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(dsa.DSAError) as e:
        dsa.dsa_forward(p.q_idx, p.w, p.k_idx, p.k_scale, p.q, p.kv, kv, 1, 2048, p.scale,
                        workspace=tiny)
    assert e.value.status == 6
    with pytest.raises(dsa.DSAError) as e:
        dsa.dsa_forward(p.q_idx, p.w, p.k_idx, p.k_scale, p.q, p.kv, kv, 1, 4096, p.scale)
    assert e.value.status == 2


def test_wait_timeout_selftest_reports_timeout():
    dsa = _dsa()
    old = dsa.dsa_set_wait_timeout_ns(50_000_000)  # 50 ms
    try:
        assert dsa.dsa_selftest_wait_timeout() == 4
        assert dsa.dsa_get_device_error() == 0
    finally:
        dsa.dsa_set_wait_timeout_ns(old)
