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


def _gpu_mla(p, idx_np):
    dsa = _dsa()
    g = p.to("cuda")
    idx = torch.from_numpy(np.ascontiguousarray(idx_np, dtype=np.int32)).cuda()
    out, lse = dsa.dsa_sparse_mla_fwd(g.q, g.kv, dsa.KvLayout.of(g), p.q_per_seq, idx, p.scale)
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == 0
    return out.float().cpu().numpy(), lse.cpu().numpy()


def _check(p, idx_np, rows=None):
    o_g, l_g = _gpu_mla(p, idx_np)
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
