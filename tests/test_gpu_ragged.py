"""Ragged batches (dsa_q_desc_t.q_start): several sequences with different numbers
of query rows in one call, on a paged cache ("dynamic KV cache", DSA principle
section of the nsmao.com report). Sequence b's query rows are its last q_len[b]
tokens: a whole prompt (q_len = seqlen), a chunk of prefill appended to tokens
already cached (q_len < seqlen), or a decode step (q_len = 1 or 2).

Each test runs the library's public calls through the C ABI and checks against
the oracle, whose row geometry (q_seq, q_pos per row) comes from the same q_start:
index sets up to near-ties at the k-th score, outputs and LSE within the parity
tolerances. Also: a ragged batch whose rows are all equal reproduces the uniform
call bit for bit, row windows and small workspaces give the same selection, the
KL term and the MHA mode follow the same geometry, and an out-of-range q_start
is reported as DSA_ERR_BOUNDS without any access outside the given buffers."""

import numpy as np
import pytest
import torch

from oracle import indexer_scores, masked_mha, sparse_indexer_kl, sparse_mla, topk_rows
from sparse_attention_05_b200 import synth
from tests.helpers import check_attention, check_index_sets, oracle_args

pytestmark = pytest.mark.gpu


def _dsa():
    from sparse_attention_05_b200 import dsa
    return dsa


def _forward(p, k, workspace_bytes=None):
    dsa = _dsa()
    g = p.to("cuda")
    kv = dsa.KvLayout.of(g)
    ws = None if workspace_bytes is None else torch.empty(workspace_bytes, dtype=torch.uint8,
                                                          device="cuda")
    idx = torch.full((p.num_q, k), -7, dtype=torch.int32, device="cuda")
    out, lse, _ = dsa.dsa_forward(g.q_idx, g.w, g.k_idx, g.k_scale, g.q, g.kv, kv, p.q_per_seq,
                                  k, p.scale, workspace=ws, idx_out=idx, q_start=g.q_start)
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == 0
    return idx.cpu().numpy(), out.float().cpu().numpy(), lse.cpu().numpy()


def _oracle_check(p, k, idx_g, o_g, l_g, rows):
    a = oracle_args(p)
    ld = (p.max_ctx + 127) // 128 * 128
    sc = indexer_scores(a["q_idx"], a["w"], a["k_idx"], a["k_scale"], a["q_seq"], a["q_pos"],
                        ld=ld, rows=rows, block_table=a["block_table"], page_size=p.page_size)
    check_index_sets(idx_g[rows], topk_rows(sc, a["q_pos"], k, rows=rows), sc,
                     a["q_pos"][rows], k)
    o_r, l_r = sparse_mla(a["q"], a["kv"], a["q_seq"], a["q_pos"], idx_g[rows], p.scale, 512,
                          rows=rows, block_table=a["block_table"], page_size=p.page_size)
    check_attention(o_g[rows], l_g[rows], o_r, l_r)


def _edge_rows(p, n, seed):
    """Every sequence's first and last query row plus seeded ones."""
    qs = p.q_start.cpu().numpy()
    must = [int(x) for b in range(p.batch) if qs[b + 1] > qs[b] for x in (qs[b], qs[b + 1] - 1)]
    return synth.sample_rows(p.num_q, n, seed=seed, must=must).numpy()


def test_three_prompts_of_different_lengths():
    """Three whole prompts (700, 2600, 2100 tokens) in one prefill call, k = 512."""
    p = synth.ragged([700, 2600, 2100], [700, 2600, 2100], seed=120)
    idx, o, l = _forward(p, 512)
    _oracle_check(p, 512, idx, o, l, _edge_rows(p, 40, 121))


def test_chunked_prefill_and_decode_mixed():
    """A chunk after cached tokens, a whole prompt, a short chunk, two decode steps;
    k = 2048 (the longest rows see more than k keys)."""
    p = synth.ragged([5000, 1500, 2300, 900, 4100], [512, 1500, 64, 1, 2], seed=122)
    idx, o, l = _forward(p, 2048)
    _oracle_check(p, 2048, idx, o, l, _edge_rows(p, 30, 123))


def test_empty_sequence_and_a_longer_row_bound():
    """A sequence with no query rows, and q_per_seq above the largest q_len (window
    rows no sequence has): nothing outside the real rows is written."""
    dsa = _dsa()
    p = synth.ragged([1200, 800, 3000], [300, 0, 2], seed=124)
    g = p.to("cuda")
    kv = dsa.KvLayout.of(g)
    k = 256
    idx = torch.full((p.num_q, k), -7, dtype=torch.int32, device="cuda")
    out = torch.full((p.num_q, 128, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((p.num_q, 128), float("nan"), dtype=torch.float32, device="cuda")
    dsa.dsa_forward(g.q_idx, g.w, g.k_idx, g.k_scale, g.q, g.kv, kv, 400, k, p.scale,
                    idx_out=idx, out=out, lse=lse, q_start=g.q_start)
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == 0
    o, l = out.float().cpu().numpy(), lse.cpu().numpy()
    assert np.isfinite(o).all() and np.isfinite(l).all()  # every real row was written
    _oracle_check(p, k, idx.cpu().numpy(), o, l, _edge_rows(p, 20, 125))


def test_equal_rows_match_the_uniform_call_bit_for_bit():
    """A ragged description of a uniform batch gives the uniform call's results."""
    dsa = _dsa()
    u = synth.paged_decode(batch=4, q_per_seq=2, min_ctx=2500, max_ctx=7000, seed=126)
    g = u.to("cuda")
    kv = dsa.KvLayout.of(g)
    q_start = torch.arange(0, 2 * 4 + 1, 2, dtype=torch.int32, device="cuda")
    res = []
    for qs in (None, q_start):
        idx = torch.empty(u.num_q, 2048, dtype=torch.int32, device="cuda")
        out, lse, _ = dsa.dsa_forward(g.q_idx, g.w, g.k_idx, g.k_scale, g.q, g.kv, kv, 2, 2048,
                                      u.scale, idx_out=idx, q_start=qs)
        res.append((idx, out, lse))
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == 0
    for a, b in zip(res[0], res[1]):
        assert torch.equal(a, b)


def test_small_workspace_chunks_give_the_same_selection():
    """Score rows in chunks of window rows over a ragged batch: same indices."""
    dsa = _dsa()
    p = synth.ragged([1800, 600, 1300], [1800, 600, 900], seed=127)
    full = _forward(p, 512)
    ld = (p.max_ctx + 127) // 128 * 128
    small = p.num_q * 512 * 4 + 256 + 5 * 3 * ld * 4  # indices + about 5 rows per sequence
    g = p.to("cuda")
    assert small < dsa.dsa_workspace_size(dsa.KvLayout.of(g), p.num_q, p.q_per_seq, 512,
                                          q_start=g.q_start)
    chunked = _forward(p, 512, workspace_bytes=small)
    np.testing.assert_array_equal(chunked[0], full[0])


def test_indexer_kl_follows_the_ragged_rows():
    """The KL term of every real row against the oracle's (absent rows get 0)."""
    dsa = _dsa()
    p = synth.ragged([900, 2200, 400], [300, 700, 1], seed=128)
    k = 256
    idx, o, l = _forward(p, k)
    a = oracle_args(p)
    ld = (p.max_ctx + 127) // 128 * 128
    rows = np.arange(p.num_q)
    sc = indexer_scores(a["q_idx"], a["w"], a["k_idx"], a["k_scale"], a["q_seq"], a["q_pos"],
                        ld=ld, rows=rows, block_table=a["block_table"], page_size=p.page_size)
    ref = sparse_indexer_kl(a["q"], a["kv"], a["q_seq"], a["q_pos"], idx, sc, p.scale,
                            block_table=a["block_table"], page_size=p.page_size)
    # score rows in the window layout: window row i of sequence b at b * q_per_seq + i
    qs = p.q_start.numpy()
    win = np.zeros((p.batch * p.q_per_seq, ld), np.float32)
    for b in range(p.batch):
        n = qs[b + 1] - qs[b]
        win[b * p.q_per_seq: b * p.q_per_seq + n] = sc[qs[b]:qs[b + 1]]
    g = p.to("cuda")
    kl = dsa.dsa_indexer_kl(g.q, g.kv, dsa.KvLayout.of(g), p.q_per_seq,
                            torch.from_numpy(idx).cuda(), p.scale, torch.from_numpy(l).cuda(),
                            torch.from_numpy(win).cuda(), q_start=g.q_start)
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == 0
    got = kl.cpu().numpy().astype(np.float64)
    for b in range(p.batch):
        n = qs[b + 1] - qs[b]
        w = got[b * p.q_per_seq: (b + 1) * p.q_per_seq]
        err = np.abs(w[:n] - ref[qs[b]:qs[b + 1]])
        assert np.all(err <= 5e-4 + 1e-3 * np.abs(ref[qs[b]:qs[b + 1]]))
        assert not w[n:].any()


def test_mha_prefill_follows_the_ragged_rows():
    """The MHA-mode short prefill (masked MHA) over a ragged batch, k = 256."""
    dsa = _dsa()
    from tests.helpers import mha_lse_tolerance
    p = synth.ragged([600, 1000, 300], [600, 400, 300], seed=129)
    m = synth.mha_inputs(p, 130)
    g, gm = p.to("cuda"), m.to("cuda")
    k = 256
    idx = torch.empty(p.num_q, k, dtype=torch.int32, device="cuda")
    out, lse, _ = dsa.dsa_mha_prefill(g.q_idx, g.w, g.k_idx, g.k_scale, gm.q_mha, g.kv, gm.w_uk,
                                      gm.w_uv, dsa.KvLayout.of(g), p.q_per_seq, k, p.scale,
                                      idx_out=idx, q_start=g.q_start)
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == 0
    rows = _edge_rows(p, 16, 131)
    a = oracle_args(p)
    ld = (p.max_ctx + 127) // 128 * 128
    sc = indexer_scores(a["q_idx"], a["w"], a["k_idx"], a["k_scale"], a["q_seq"], a["q_pos"],
                        ld=ld, rows=rows, block_table=a["block_table"], page_size=p.page_size)
    idx_g = idx.cpu().numpy()[rows]
    check_index_sets(idx_g, topk_rows(sc, a["q_pos"], k, rows=rows), sc, a["q_pos"][rows], k)
    q_mha, w_uk, w_uv = (x.float().numpy() for x in (m.q_mha, m.w_uk, m.w_uv))
    o_r, l_r = masked_mha(q_mha, a["kv"], a["q_seq"], a["q_pos"], idx_g, p.scale, w_uk, w_uv,
                          rows=rows, block_table=a["block_table"], page_size=p.page_size)
    pos = a["q_pos"]
    sets = [np.unique([s for s in idx_g[r] if 0 <= s <= pos[t]]) for r, t in enumerate(rows)]
    tol = mha_lse_tolerance(q_mha, a["kv"], a["q_seq"], pos, sets, w_uk, p.scale, rows,
                            block_table=a["block_table"], page_size=p.page_size)
    check_attention(out.float().cpu().numpy()[rows], lse.cpu().numpy()[rows], o_r, l_r,
                    lse_tol=tol)


def test_out_of_range_q_start_is_reported():
    """A q_len above q_per_seq, offsets past num_q, a decreasing offset: each is
    reported as DSA_ERR_BOUNDS; a valid sequence of the same call is still computed
    and no access leaves the given buffers (q_start has batch + 1 entries)."""
    dsa = _dsa()
    p = synth.ragged([900, 1500], [200, 100], seed=132)  # 300 query rows
    g = p.to("cuda")
    kv = dsa.KvLayout.of(g)
    # q_per_seq = 150: the host accepts num_q = 300 <= 2 x 150
    cases = (([0, 200, 305], None),   # q_len 200 > 150; end past num_q
             ([0, 100, 50], 0),       # second sequence decreasing; the first is valid
             ([0, 160, 300], 1))      # first q_len 160 > 150; the second (140 rows) valid
    for bad, valid_seq in cases:
        qs = torch.tensor(bad, dtype=torch.int32, device="cuda")
        idx = torch.full((p.num_q, 256), -7, dtype=torch.int32, device="cuda")
        dsa.dsa_forward(g.q_idx, g.w, g.k_idx, g.k_scale, g.q, g.kv, kv, 150, 256, p.scale,
                        idx_out=idx, q_start=qs)
        torch.cuda.synchronize()
        assert dsa.dsa_get_device_error() == 5  # DSA_ERR_BOUNDS
        if valid_seq is not None:
            got = idx.cpu().numpy()[bad[valid_seq]:bad[valid_seq + 1]]
            assert (got != -7).all()
