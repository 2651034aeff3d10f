"""GPU parity of dsa_indexer_scores (FP8 tcgen05 kernel) against the oracle's
FP8-emulated fp64 scores: contiguous and paged caches, 1..4 query rows per
sequence, causal prefill rows, ragged key tiles, sampled rows at full size and
device-side bounds errors."""

import numpy as np
import pytest
import torch

from oracle import indexer_scores
from sparse_attention_05_b200 import synth
from tests.helpers import SCORE_RTOL, check_scores, oracle_args

pytestmark = pytest.mark.gpu


def _dsa():
    from sparse_attention_05_b200 import dsa
    return dsa


def _gpu_scores(p):
    dsa = _dsa()
    g = p.to("cuda")
    s = dsa.dsa_indexer_scores(g.q_idx, g.w, g.k_idx, g.k_scale, dsa.KvLayout.of(g), p.q_per_seq)
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == 0
    return s.cpu().numpy()


def _check(p, rows=None):
    got = _gpu_scores(p)
    a = oracle_args(p)
    rows = np.arange(p.num_q) if rows is None else np.asarray(rows)
    ref = indexer_scores(a["q_idx"], a["w"], a["k_idx"], a["k_scale"], a["q_seq"], a["q_pos"],
                         ld=got.shape[1], rows=rows, block_table=a["block_table"],
                         page_size=p.page_size)
    pos = a["q_pos"][rows]
    worst = check_scores(got[rows], ref, pos)
    # identical FP8 query codes on both sides leave only fp32-vs-fp64 rounding
    assert worst < 1e-4, f"worst rel err {worst:.2e}: FP8 emulation differs"
    for r, t in enumerate(rows):  # masked tail of the last 128-key tile is -inf
        end = (int(pos[r]) // 128 + 1) * 128
        assert np.all(np.isneginf(got[t, pos[r] + 1:end]))
    return worst


@pytest.mark.parametrize("q_per_seq,batch,ctx", [(1, 4, 1000), (2, 3, 2500), (3, 2, 700),
                                                 (4, 2, 129), (1, 1, 1)])
def test_decode_contiguous(q_per_seq, batch, ctx):
    p = synth.decode(batch=batch, ctx=ctx, q_per_seq=q_per_seq, seed=20 + q_per_seq)
    _check(p)


def test_contiguous_shorter_seqlens():
    p = synth.decode(batch=5, ctx=3000, q_per_seq=2, seed=31)
    p.seqlens = torch.tensor([3000, 2, 1500, 129, 128], dtype=torch.int32)
    _check(p)


@pytest.mark.parametrize("L", [1101, 2048])
def test_causal_prefill_rows(L):
    p = synth.prefill(L=L, seed=32)
    _check(p)


@pytest.mark.parametrize("page_size", [64, 128])
def test_paged(page_size):
    p = synth.paged_decode(batch=4, q_per_seq=2, min_ctx=100, max_ctx=3000, page_size=page_size,
                           seed=33)
    _check(p)


def test_full_size_decode_sampled_rows():
    """Batch 64 x 32768 contiguous decode: every row checked on sampled rows."""
    p = synth.decode(batch=64, ctx=32768, q_per_seq=1, seed=1)
    rows = synth.sample_rows(p.num_q, 6, seed=1, must=(0, 63)).numpy()
    _check(p, rows)


def test_bounds_errors_are_reported():
    dsa = _dsa()
    p = synth.paged_decode(batch=2, q_per_seq=1, min_ctx=200, max_ctx=400, seed=34)
    g = p.to("cuda")
    g.block_table[1, 0] = p.k_idx.shape[0] + 5  # page beyond the cache
    dsa.dsa_indexer_scores(g.q_idx, g.w, g.k_idx, g.k_scale, dsa.KvLayout.of(g), 1)
    assert dsa.dsa_get_device_error() == 5
    assert dsa.dsa_get_device_error() == 0  # cleared by the read
    g.block_table[1, 0] = 0
    g.seqlens[0] = 401  # longer than max_ctx
    dsa.dsa_indexer_scores(g.q_idx, g.w, g.k_idx, g.k_scale, dsa.KvLayout.of(g), 1)
    assert dsa.dsa_get_device_error() == 5


def test_host_argument_checks():
    dsa = _dsa()
    p = synth.decode(batch=2, ctx=256, q_per_seq=1, seed=35).to("cuda")
    kv = dsa.KvLayout.of(p)
    bad = torch.empty(2, 200, device="cuda")  # ld below max_ctx rounded to 128
    with pytest.raises(dsa.DSAError) as e:
        dsa.dsa_indexer_scores(p.q_idx, p.w, p.k_idx, p.k_scale, kv, 1, scores=bad)
    assert e.value.status == 1
    with pytest.raises(dsa.DSAError):
        dsa.dsa_indexer_scores(p.q_idx, p.w, p.k_idx, p.k_scale, kv, 3)  # T != B * q_per_seq
