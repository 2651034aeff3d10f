"""GPU parity of dsa_sparse_mla_fwd (tcgen05, 2-CTA clusters) against the
oracle's fp64 sparse MLA, fed the same index sets: the oracle's own top-k
selection, random sets, unsorted / padded / out-of-range / duplicate entries,
k not a multiple of the 64-key block, paged caches, dense rows (k >= t + 1),
empty selections, large logits (lazy-rescale path) and sampled rows at the
full decode size."""

import numpy as np
import pytest
import torch

from oracle import dense_causal_mqa, indexer_scores, sparse_mla, topk_rows
from sparse_attention_05_b200 import synth
from tests.helpers import check_attention, oracle_args

pytestmark = pytest.mark.gpu


def _dsa():
    from sparse_attention_05_b200 import dsa
    return dsa


def _gpu_mla(p, idx_np, ws=False):
    """ws=True: through dsa_sparse_mla_fwd_ws with a full scratch, so the rows of a
    partly filled last wave run as key segments merged by the combine kernel."""
    dsa = _dsa()
    g = p.to("cuda")
    idx = torch.from_numpy(np.ascontiguousarray(idx_np, dtype=np.int32)).cuda()
    if ws:
        out, lse = dsa.dsa_sparse_mla_fwd_ws(g.q, g.kv, dsa.KvLayout.of(g), p.q_per_seq, idx,
                                             p.scale)
    else:
        out, lse = dsa.dsa_sparse_mla_fwd(g.q, g.kv, dsa.KvLayout.of(g), p.q_per_seq, idx,
                                          p.scale)
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == 0
    return out.float().cpu().numpy(), lse.cpu().numpy()


def _check(p, idx_np, rows=None, ws=False):
    o_g, l_g = _gpu_mla(p, idx_np, ws)
    a = oracle_args(p)
    rows = np.arange(p.num_q) if rows is None else np.asarray(rows)
    o_r, l_r = sparse_mla(a["q"], a["kv"], a["q_seq"], a["q_pos"], idx_np[rows], p.scale, 512,
                          rows=rows, block_table=a["block_table"], page_size=p.page_size)
    return check_attention(o_g[rows], l_g[rows], o_r, l_r)


def _random_idx(p, k, seed, sort=True):
    rng = np.random.default_rng(seed)
    pos = p.q_pos().numpy()
    out = np.full((p.num_q, k), -1, np.int32)
    for t in range(p.num_q):
        n = min(k, int(pos[t]) + 1)
        sel = rng.choice(int(pos[t]) + 1, n, replace=False)
        out[t, :n] = np.sort(sel) if sort else sel
    return out


def test_oracle_topk_selection_decode():
    p = synth.decode(batch=4, ctx=4096, q_per_seq=1, seed=40)
    a = oracle_args(p)
    sc = indexer_scores(a["q_idx"], a["w"], a["k_idx"], a["k_scale"], a["q_seq"], a["q_pos"],
                        ld=4096)
    idx = topk_rows(sc, a["q_pos"], 2048)
    _check(p, idx)


@pytest.mark.parametrize("k", [2048, 100, 64, 1])
def test_random_sets_various_k(k):
    p = synth.decode(batch=3, ctx=3000, q_per_seq=2, seed=41)
    _check(p, _random_idx(p, k, seed=k))


def test_unsorted_padded_out_of_range_and_duplicates():
    p = synth.decode(batch=2, ctx=2000, q_per_seq=2, seed=42)
    idx = _random_idx(p, 256, seed=3, sort=False)
    pos = p.q_pos().numpy()
    idx[:, 10] = -1
    idx[:, 20] = -7
    idx[0, 30] = pos[0] + 1          # beyond the query position: skipped
    idx[0, 31] = pos[0] + 5          # beyond pos, still inside the cache: skipped
    idx[2, 40] = idx[2, 41]          # duplicate: counted twice on both sides
    _check(p, idx)


@pytest.mark.parametrize("page_size", [64, 256])
def test_paged(page_size):
    p = synth.paged_decode(batch=3, q_per_seq=2, min_ctx=500, max_ctx=5000, page_size=page_size,
                           seed=43)
    _check(p, _random_idx(p, 2048, seed=5))


def test_dense_rows_equal_dense_causal_mqa():
    """k >= pos + 1 selects every visible key: the result is dense causal MQA."""
    p = synth.prefill(L=700, seed=44)
    idx = np.full((700, 768), -1, np.int32)
    for t in range(700):
        idx[t, :t + 1] = np.arange(t + 1)
    o_g, l_g = _gpu_mla(p, idx)
    a = oracle_args(p)
    rows = np.array([0, 1, 63, 64, 65, 300, 699])
    o_r, l_r = dense_causal_mqa(a["q"], a["kv"], a["q_seq"], a["q_pos"], p.scale, 512, rows=rows)
    check_attention(o_g[rows], l_g[rows], o_r, l_r)


@pytest.mark.parametrize("ws", [False, True])
def test_short_rows_with_scattered_and_trailing_entries(ws):
    """Rows with fewer than k visible keys stop after the block of their last entry
    inside [0, pos]: entries scattered among -1 pads, a valid entry in the very last
    slot, out-of-range entries after the last valid one, and a row whose only valid
    entry comes first."""
    p = synth.prefill(L=1500, seed=49)
    rows = np.array([0, 1, 47, 48, 100, 700, 1499])
    rng = np.random.default_rng(9)
    idx = np.full((1500, 2048), -1, np.int32)
    for t in range(1500):
        n = t + 1
        slots = np.sort(rng.choice(2048, n, replace=False))
        idx[t, slots] = rng.permutation(n)          # every visible key once, scattered
    idx[700, 2047] = 3                               # a valid entry in the last slot
    idx[100, 1900:] = 5000                           # beyond pos after the last valid entry
    idx[1] = -1
    idx[1, 0] = 1                                    # only the first slot is valid
    _check(p, idx, rows=rows, ws=ws)


def test_empty_selection_gives_zero_and_neg_inf():
    p = synth.decode(batch=2, ctx=300, q_per_seq=1, seed=45)
    idx = np.full((2, 128), -1, np.int32)
    idx[1, :5] = [3, 1, 4, 1, 5]
    o_g, l_g = _gpu_mla(p, idx)
    assert np.all(o_g[0] == 0) and np.all(np.isneginf(l_g[0]))
    _check(p, idx)


def test_large_logits_exercise_rescale():
    p = synth.decode(batch=2, ctx=4096, q_per_seq=1, seed=46)
    p.q = (p.q.float() * 6.0).to(torch.bfloat16)
    # ascending magnitudes make the running max grow block after block
    p.kv = (p.kv.float() * torch.linspace(0.2, 3.0, 4096)[None, :, None]).to(torch.bfloat16)
    _check(p, _random_idx(p, 2048, seed=6))


def test_full_size_decode_sampled_rows():
    p = synth.decode(batch=64, ctx=32768, q_per_seq=1, seed=1)
    idx = _random_idx(p, 2048, seed=7)
    rows = synth.sample_rows(p.num_q, 4, seed=2, must=(0, 63)).numpy()
    _check(p, idx, rows)


# ---- rows split into key segments (dsa_sparse_mla_fwd_ws) -----------------------------
# A call runs (SMs / 2) rows per wave; the rows of a last wave at most half full are
# split into 2..8 segments of at least 6 key blocks. The cases below have few rows
# (a single partial wave: every row is split) or a tail after full waves.

def test_split_oracle_selection_decode():
    p = synth.decode(batch=4, ctx=4096, q_per_seq=1, seed=140)
    a = oracle_args(p)
    sc = indexer_scores(a["q_idx"], a["w"], a["k_idx"], a["k_scale"], a["q_seq"], a["q_pos"],
                        ld=4096)
    _check(p, topk_rows(sc, a["q_pos"], 2048), ws=True)


@pytest.mark.parametrize("k", [2048, 1200, 576, 300])
def test_split_random_sets_various_k(k):
    p = synth.decode(batch=3, ctx=3000, q_per_seq=2, seed=141)
    _check(p, _random_idx(p, k, seed=k), ws=True)


def test_split_unsorted_padded_out_of_range_and_duplicates():
    p = synth.decode(batch=2, ctx=2000, q_per_seq=2, seed=142)
    idx = _random_idx(p, 1200, seed=3, sort=False)
    pos = p.q_pos().numpy()
    idx[:, 10] = -1
    idx[:, 700] = -7
    idx[0, 30] = pos[0] + 1
    idx[1, 900] = pos[1] + 5
    idx[2, 40] = idx[2, 1100]        # a duplicate across two segments
    _check(p, idx, ws=True)


@pytest.mark.parametrize("page_size", [64, 256])
def test_split_paged(page_size):
    p = synth.paged_decode(batch=3, q_per_seq=2, min_ctx=500, max_ctx=5000, page_size=page_size,
                           seed=143)
    _check(p, _random_idx(p, 2048, seed=5), ws=True)


def test_split_empty_segments_and_empty_rows():
    """Segments holding no valid entry merge as weight 0; a row with none at all
    stays o = 0, lse = -inf."""
    p = synth.decode(batch=3, ctx=3000, q_per_seq=1, seed=144)
    idx = np.full((3, 2048), -1, np.int32)
    idx[1, :5] = [3, 1, 4, 1, 5]                    # first segment only
    idx[2, 2040:] = np.arange(8) * 300               # last segment only
    o_g, l_g = _gpu_mla(p, idx, ws=True)
    assert np.all(o_g[0] == 0) and np.all(np.isneginf(l_g[0]))
    _check(p, idx, ws=True)


def test_split_large_logits():
    p = synth.decode(batch=2, ctx=4096, q_per_seq=1, seed=146)
    p.q = (p.q.float() * 6.0).to(torch.bfloat16)
    p.kv = (p.kv.float() * torch.linspace(0.2, 3.0, 4096)[None, :, None]).to(torch.bfloat16)
    _check(p, _random_idx(p, 2048, seed=6), ws=True)


def test_split_tail_after_full_waves():
    """More rows than one wave: the whole rows and the split tail rows both match
    the oracle, and the split result differs from the unsplit one only by rounding
    (which also shows that the split ran)."""
    wave = torch.cuda.get_device_properties(0).multi_processor_count // 2
    batch = (wave + 7) // 2
    nq = 2 * batch                                    # a tail of 6 or 7 rows
    p = synth.paged_decode(batch=batch, q_per_seq=2, min_ctx=2100, max_ctx=12000,
                           page_size=64, seed=147)
    idx = _random_idx(p, 2048, seed=8)
    rows = np.array([0, 1, wave - 1, wave, wave + 2, nq - 1])
    o_s, l_s = _gpu_mla(p, idx, ws=True)
    o_w, l_w = _gpu_mla(p, idx, ws=False)
    a = oracle_args(p)
    o_r, l_r = sparse_mla(a["q"], a["kv"], a["q_seq"], a["q_pos"], idx[rows], p.scale, 512,
                          rows=rows, block_table=a["block_table"], page_size=p.page_size)
    check_attention(o_s[rows], l_s[rows], o_r, l_r)
    assert np.array_equal(o_s[:wave], o_w[:wave]) and np.array_equal(l_s[:wave], l_w[:wave])
    assert np.abs(l_s - l_w).max() <= 5e-5
    assert np.all(np.abs(o_s - o_w) <= 2.0 ** -7 * np.abs(o_w) + 2e-3)
    assert not np.array_equal(l_s[wave:], l_w[wave:])


def test_split_through_forward_equals_oracle():
    """dsa_forward's workspace serves as the split scratch once the selection is done."""
    dsa = _dsa()
    p = synth.decode(batch=4, ctx=5000, q_per_seq=2, seed=148)
    g = p.to("cuda")
    kv = dsa.KvLayout.of(g)
    idx = torch.empty(p.num_q, 2048, dtype=torch.int32, device="cuda")
    o, l, _ = dsa.dsa_forward(g.q_idx, g.w, g.k_idx, g.k_scale, g.q, g.kv, kv, p.q_per_seq,
                              2048, p.scale, idx_out=idx)
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == 0
    idx_np = idx.cpu().numpy()
    a = oracle_args(p)
    o_r, l_r = sparse_mla(a["q"], a["kv"], a["q_seq"], a["q_pos"], idx_np, p.scale, 512,
                          rows=np.arange(p.num_q))
    check_attention(o.float().cpu().numpy(), l.cpu().numpy(), o_r, l_r)
