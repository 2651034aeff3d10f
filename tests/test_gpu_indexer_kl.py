"""GPU parity of dsa_indexer_kl (the indexer's KL loss term, [TR] §2.1) against
the oracle: the oracle computes the scores, the selected sets (top-k, or every
visible key for the dense warm-up form) and the per-head LSE in fp64; the GPU
kernel receives exactly those inputs, so the comparison isolates its own
arithmetic (fp32 dot products from the tensor core, exp2, the head mean, the
sums and the log-sum-exp of I).

Tolerance: the only rounding the kernel adds to the oracle's definition is fp32
(LSE passed as fp32: ~5e-6 relative in p; fp32 sums over <= 2048 keys), so the
KL term may move by about 1e-4 absolute: the bound below is 5e-4 + 1e-3 |KL|."""

import numpy as np
import pytest
import torch

from oracle import dense_indexer_kl, indexer_scores, sparse_indexer_kl, sparse_mla, topk_rows
from sparse_attention_05_b200 import synth
from tests.helpers import oracle_args

pytestmark = pytest.mark.gpu

KL_ATOL, KL_RTOL = 5e-4, 1e-3


def _dsa():
    from sparse_attention_05_b200 import dsa
    return dsa


def _check(p, k=2048, rows=None, dense=False):
    dsa = _dsa()
    a = oracle_args(p)
    T = p.num_q
    rows = np.arange(T) if rows is None else np.asarray(rows)
    ld = (p.max_ctx + 127) // 128 * 128
    sc = indexer_scores(a["q_idx"], a["w"], a["k_idx"], a["k_scale"], a["q_seq"], a["q_pos"],
                        ld=ld, rows=rows, block_table=a["block_table"], page_size=p.page_size)
    if dense:
        kk = int(a["q_pos"][rows].max()) + 1
        idx_r = np.full((len(rows), kk), -1, np.int32)
        for r, t in enumerate(rows):
            idx_r[r, : int(a["q_pos"][t]) + 1] = np.arange(int(a["q_pos"][t]) + 1)
        ref = dense_indexer_kl(a["q"], a["kv"], a["q_seq"], a["q_pos"], sc, p.scale, rows=rows,
                               block_table=a["block_table"], page_size=p.page_size)
    else:
        kk = k
        idx_r = topk_rows(sc, a["q_pos"], k, rows=rows)
        ref = sparse_indexer_kl(a["q"], a["kv"], a["q_seq"], a["q_pos"], idx_r, sc, p.scale,
                                rows=rows, block_table=a["block_table"], page_size=p.page_size)
    _, lse_r = sparse_mla(a["q"], a["kv"], a["q_seq"], a["q_pos"], idx_r, p.scale, 512, rows=rows,
                          block_table=a["block_table"], page_size=p.page_size)
    # GPU inputs: every row of the window gets the oracle's set, LSE and score row
    # (unchecked rows keep an empty set, whose term is 0)
    idx = np.full((T, kk), -1, np.int32)
    lse = np.zeros((T, 128), np.float32)
    scores = np.zeros((T, ld), np.float32)
    idx[rows] = idx_r
    lse[rows] = lse_r.astype(np.float32)
    scores[rows] = sc
    g = p.to("cuda")
    kl = dsa.dsa_indexer_kl(g.q, g.kv, dsa.KvLayout.of(g), p.q_per_seq,
                            torch.from_numpy(idx).cuda(), p.scale, torch.from_numpy(lse).cuda(),
                            torch.from_numpy(scores).cuda())
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == 0
    got = kl.cpu().numpy().astype(np.float64)
    err = np.abs(got[rows] - ref)
    assert np.all(err <= KL_ATOL + KL_RTOL * np.abs(ref)), \
        f"KL max abs err {err.max():.3e} (ref {ref[np.argmax(err)]:.4f})"
    others = np.setdiff1d(np.arange(T), rows)
    assert np.all(got[others] == 0.0)
    assert np.all(ref >= 0.0)
    return got[rows], ref


def test_decode_contiguous_sparse():
    p = synth.decode(batch=4, ctx=3000, q_per_seq=1, seed=60)
    got, ref = _check(p)
    assert np.all(ref > 1e-3)  # a non-trivial target on random inputs


def test_paged_two_queries_sparse():
    p = synth.paged_decode(batch=3, q_per_seq=2, min_ctx=2500, max_ctx=5000, page_size=64,
                           seed=61)
    _check(p)


@pytest.mark.parametrize("k", [1, 100, 128, 300])
def test_small_k_partial_tiles(k):
    p = synth.decode(batch=2, ctx=1500, q_per_seq=1, seed=62 + k)
    got, ref = _check(p, k=k)
    if k == 1:
        assert np.all(np.abs(got) <= KL_ATOL)  # one key: p = q = 1


def test_prefill_rows_dense_warmup_form():
    p = synth.prefill(L=1200, seed=63)
    _check(p, rows=[0, 1, 5, 300, 777, 1199], dense=True)


def test_full_size_decode_sampled_rows():
    """Batch 64 x 32768 contiguous decode (the decode benchmark's inputs)."""
    p = synth.decode(batch=64, ctx=32768, q_per_seq=1, seed=1)
    rows = synth.sample_rows(p.num_q, 4, seed=64, must=(0, p.num_q - 1)).numpy()
    _check(p, rows=rows)


def test_host_argument_checks():
    dsa = _dsa()
    p = synth.decode(batch=2, ctx=256, q_per_seq=1, seed=65).to("cuda")
    kv = dsa.KvLayout.of(p)
    idx = torch.zeros(2, 16, dtype=torch.int32, device="cuda")
    lse = torch.zeros(2, 128, device="cuda")
    short = torch.zeros(2, 100, device="cuda")  # ld below max_ctx
    with pytest.raises(dsa.DSAError) as e:
        dsa.dsa_indexer_kl(p.q, p.kv, kv, 1, idx, p.scale, lse, short)
    assert e.value.status == 1
