"""Full-size parity of dsa_forward on the benchmark workloads, on sampled rows.

Each workload is generated on the GPU with the benchmark's own seeds and run
through dsa_forward at full size (the same launches, chunking plan and grid
shapes the benchmark times). The oracle then checks sampled query rows one at
a time: for a row of sequence b at position pos, the sequence's indexer keys,
key scales and latent rows 0..pos are gathered (through the block table when
the cache is paged, with plain torch indexing) into a single contiguous
sequence, on which the oracle computes the scores, the top-k set and the
attention over the GPU's selected set.

Checks per sampled row: the index set (equal up to near-ties at the k-th
score), the bf16 output and fp32 LSE against the oracle's attention over that
set; rows t < k must also equal dense causal MQA; the planted hot key
positions of the 128K prefill must be selected by almost every later row.
"""

import numpy as np
import pytest
import torch

from oracle import dense_causal_mqa, indexer_scores, sparse_mla, topk_rows
from sparse_attention_05_b200 import synth
from tests.helpers import check_attention, check_index_sets, np32

pytestmark = pytest.mark.gpu

K = 2048


def _dsa():
    from sparse_attention_05_b200 import dsa
    return dsa


def _run_forward(g):
    """dsa_forward over every query row of a GPU-resident problem."""
    dsa = _dsa()
    kv = dsa.KvLayout.of(g)
    idx = torch.empty(g.num_q, K, dtype=torch.int32, device="cuda")
    out, lse, _ = dsa.dsa_forward(g.q_idx, g.w, g.k_idx, g.k_scale, g.q, g.kv, kv, g.q_per_seq,
                                  K, g.scale, idx_out=idx)
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == 0
    return idx, out, lse


def _sequence_rows(g, b, n):
    """Physical cache rows of logical tokens 0..n-1 of sequence b (torch, on GPU)."""
    s = torch.arange(n, device="cuda")
    if not g.paged:
        return b * g.max_ctx + s
    pages = g.block_table[b].long()[s // g.page_size]
    return pages * g.page_size + s % g.page_size


def _row_oracle(g, t, gpu_idx_row):
    """Oracle scores, top-k set and attention (over the GPU's set) for row t,
    computed on the row's sequence gathered into one contiguous sequence."""
    b = int(g.q_seq()[t])
    pos = int(g.q_pos()[t])
    n = pos + 1
    rows = _sequence_rows(g, b, n)
    k_idx = g.k_idx.reshape(-1, g.k_idx.shape[-1])[rows].cpu().numpy()[None]
    k_scale = np32(g.k_scale.reshape(-1)[rows])[None]
    kv = np32(g.kv.reshape(-1, g.kv.shape[-1])[rows])[None]
    q_idx = np32(g.q_idx[t:t + 1])
    w = np32(g.w[t:t + 1])
    q = np32(g.q[t:t + 1])
    q_seq, q_pos = np.zeros(1, np.int64), np.array([pos], np.int64)
    ld = (n + 127) // 128 * 128
    sc = indexer_scores(q_idx, w, k_idx, k_scale, q_seq, q_pos, ld=ld)
    ref_idx = topk_rows(sc, q_pos, K)
    o, lse = sparse_mla(q, kv, q_seq, q_pos, gpu_idx_row[None], g.scale, 512)
    dense = dense_causal_mqa(q, kv, q_seq, q_pos, g.scale, 512) if n <= K else None
    return sc, ref_idx, (o, lse), dense, pos


def _check_rows(g, rows, idx, out, lse):
    ndiff = 0
    for t in rows:
        gi = idx[t].cpu().numpy()
        sc, ref_idx, (o_r, l_r), dense, pos = _row_oracle(g, int(t), gi)
        ndiff += check_index_sets(gi[None], ref_idx, sc, np.array([pos]), K)
        o_g = out[t:t + 1].float().cpu().numpy()
        l_g = lse[t:t + 1].cpu().numpy()
        check_attention(o_g, l_g, o_r, l_r)
        if dense is not None:  # every visible key selected: DSA equals dense causal MQA
            check_attention(o_g, l_g, dense[0], dense[1])
    return ndiff


def _free():
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def test_full_size_paged_decode_sampled_rows():
    """128 sequences x 2 queries, ctx U{4096..131072}, page 64, permuted block table."""
    g = synth.paged_decode(batch=128, q_per_seq=2, min_ctx=4096, max_ctx=131072, page_size=64,
                           seed=4, device="cuda")
    idx, out, lse = _run_forward(g)
    seqlens = g.seqlens.cpu()
    longest, shortest = int(torch.argmax(seqlens)), int(torch.argmin(seqlens))
    must = (2 * longest, 2 * longest + 1, 2 * shortest + 1, 0, g.num_q - 1)
    rows = synth.sample_rows(g.num_q, 3, seed=41, must=must).tolist()
    _check_rows(g, rows, idx, out, lse)
    del g, idx, out, lse
    _free()


def test_full_size_prefill_8k_sampled_rows():
    """L = 8192; rows below k are dense (checked against dense causal MQA)."""
    g = synth.prefill(L=8192, seed=2, device="cuda")
    idx, out, lse = _run_forward(g)
    rows = synth.sample_rows(g.num_q, 4, seed=42, must=(0, 1, 2047, 2048, 8191)).tolist()
    _check_rows(g, rows, idx, out, lse)
    del g, idx, out, lse
    _free()


def test_full_size_prefill_128k_sampled_rows():
    """L = 131072 with 64 planted hot key positions (indexer keys x4)."""
    g = synth.prefill(L=131072, seed=3, n_hot=64, device="cuda")
    idx, out, lse = _run_forward(g)
    rows = synth.sample_rows(g.num_q, 3, seed=43, must=(0, 2047, 2048, 131071)).tolist()
    _check_rows(g, rows, idx, out, lse)
    # planted structure: a hot position p is selected by almost every row t >= p
    hot = g.hot.cpu().numpy()
    probe = synth.sample_rows(g.num_q, 64, seed=44, must=(131071,)).tolist()
    hits = total = 0
    for t in probe:
        sel = set(idx[t].cpu().numpy().tolist())
        vis = [int(p) for p in hot if p <= t]
        hits += sum(p in sel for p in vis)
        total += len(vis)
    assert total > 0 and hits >= 0.9 * total, f"hot positions selected {hits}/{total}"
    del g, idx, out, lse
    _free()
