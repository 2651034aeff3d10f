"""Full-size parity of dsa_forward on the benchmark workloads, on the sampled rows
each workload is specified with.

Each workload is generated on the GPU with the benchmark's own seeds and run
through dsa_forward at full size (the same launches, chunking plan and grid
shapes the benchmark times). The oracle then checks the rows:

  * 128K causal prefill: 512 seeded rows (seed 3, uniform over [0, L), always
    including rows 0, 2047, 2048 and L - 1);
  * varlen paged decode: all 256 rows (128 sequences x 2 query tokens);
  * 32K batched decode: all 64 rows;
  * 8K causal prefill: 256 seeded rows plus the edges of the dense band.

For each sequence the sampled rows belong to, its indexer keys and key scales
0..(last sampled position) are gathered once (through the block table when the
cache is paged, with plain torch indexing) into a contiguous sequence, on which
the oracle computes every sampled row's scores and top-k set. The attention is
checked per row over the GPU's selected set, whose latent rows are gathered the
same way. Per row: the index set (equal up to near-ties at the k-th score), the
bf16 output and the fp32 LSE against the oracle's attention over that set; rows
with at most k visible keys must also equal dense causal MQA; the planted hot
key positions of the 128K prefill must be selected by almost every later row.
"""

import numpy as np
import pytest
import torch

from oracle import indexer_scores, sparse_mla_token, topk_rows
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


def _cache_rows(g, b, positions):
    """Physical cache rows of logical tokens ``positions`` of sequence b (torch)."""
    s = torch.as_tensor(positions, device=g.k_idx.device, dtype=torch.int64)
    if not g.paged:
        return b * g.max_ctx + s
    pages = g.block_table[b].long()[s // g.page_size]
    return pages * g.page_size + s % g.page_size


def _latent_rows(g, b, positions):
    kv = g.kv.reshape(-1, g.kv.shape[-1])
    return np32(kv[_cache_rows(g, b, positions)])


def _check_rows(g, rows, idx, out, lse):
    """Oracle check of query rows ``rows``; returns the number of near-tie index
    differences seen."""
    q_seq, q_pos = g.q_seq().numpy(), g.q_pos().numpy()
    rows = [int(t) for t in rows]
    ndiff = 0
    by_seq = {}
    for t in rows:
        by_seq.setdefault(int(q_seq[t]), []).append(t)
    for b, mine in sorted(by_seq.items()):
        n = int(max(q_pos[t] for t in mine)) + 1
        r = _cache_rows(g, b, torch.arange(n))
        k_idx = g.k_idx.reshape(-1, g.k_idx.shape[-1])[r].cpu().numpy()[None]
        k_scale = np32(g.k_scale.reshape(-1)[r])[None]
        tr = torch.as_tensor(mine)
        pos = q_pos[mine].astype(np.int64)
        sc = indexer_scores(np32(g.q_idx[tr]), np32(g.w[tr]), k_idx, k_scale,
                            np.zeros(len(mine), np.int64), pos, ld=(n + 127) // 128 * 128)
        ref_idx = topk_rows(sc, pos, K)
        gpu_idx = idx[tr].cpu().numpy()
        o_gpu = out[tr].float().cpu().numpy()
        l_gpu = lse[tr].cpu().numpy()
        q_rows = np32(g.q[tr])
        for j, t in enumerate(mine):
            gi = gpu_idx[j]
            ndiff += check_index_sets(gi[None], ref_idx[j:j + 1], sc[j:j + 1], pos[j:j + 1], K)
            sel = [int(s) for s in gi if 0 <= int(s) <= pos[j]]
            o_r, l_r = sparse_mla_token(q_rows[j], _latent_rows(g, b, sel), g.scale, 512)
            check_attention(o_gpu[j:j + 1], l_gpu[j:j + 1], o_r[None], l_r[None])
            if pos[j] + 1 <= K:  # every visible key selected: DSA equals dense causal MQA
                o_d, l_d = sparse_mla_token(q_rows[j], _latent_rows(g, b, range(pos[j] + 1)),
                                            g.scale, 512)
                check_attention(o_gpu[j:j + 1], l_gpu[j:j + 1], o_d[None], l_d[None])
    return ndiff


def _free():
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def test_full_size_paged_decode_all_256_rows():
    """128 sequences x 2 queries, ctx U{4096..131072}, page 64, permuted block table:
    every one of the 256 query rows against the oracle."""
    g = synth.paged_decode(batch=128, q_per_seq=2, min_ctx=4096, max_ctx=131072, page_size=64,
                           seed=4, device="cuda")
    idx, out, lse = _run_forward(g)
    _check_rows(g, range(g.num_q), idx, out, lse)
    del g, idx, out, lse
    _free()


def test_full_size_decode_32k_all_64_rows():
    """64 sequences x 1 query at position 32767 on a contiguous cache: all 64 rows."""
    g = synth.decode(batch=64, ctx=32768, q_per_seq=1, seed=1, latent_std=0.5, device="cuda")
    idx, out, lse = _run_forward(g)
    _check_rows(g, range(g.num_q), idx, out, lse)
    del g, idx, out, lse
    _free()


def test_full_size_prefill_8k_256_sampled_rows():
    """L = 8192; rows below k are dense (checked against dense causal MQA)."""
    g = synth.prefill(L=8192, seed=2, device="cuda")
    idx, out, lse = _run_forward(g)
    rows = synth.sample_rows(g.num_q, 256, seed=42, must=(0, 1, 2046, 2047, 2048, 8191)).tolist()
    _check_rows(g, rows, idx, out, lse)
    del g, idx, out, lse
    _free()


def test_full_size_prefill_128k_512_sampled_rows():
    """L = 131072 with 64 planted hot key positions (indexer keys x4): 512 seeded rows
    (seed 3) including 0, 2047, 2048 and L - 1."""
    L = 131072
    g = synth.prefill(L=L, seed=3, n_hot=64, device="cuda")
    idx, out, lse = _run_forward(g)
    rows = synth.sample_rows(L, 512, seed=3, must=(0, 2047, 2048, L - 1)).tolist()
    assert len(rows) == 512 and {0, 2047, 2048, L - 1} <= set(rows)
    _check_rows(g, rows, idx, out, lse)
    # planted structure: a hot position p is selected by almost every row t >= p
    hot = g.hot.cpu().numpy()
    sel_rows = idx[torch.as_tensor(rows)].cpu().numpy()
    hits = total = 0
    for t, sel in zip(rows, sel_rows):
        sel = set(sel.tolist())
        vis = [int(p) for p in hot if p <= t]
        hits += sum(p in sel for p in vis)
        total += len(vis)
    assert total > 0 and hits >= 0.9 * total, f"hot positions selected {hits}/{total}"
    del g, idx, out, lse
    _free()
