"""Fused indexer -> top-k (the selection without stored score rows) on the GPU: the
selected indices must equal those of the unfused path (dsa_indexer_scores +
dsa_topk, itself pinned to the oracle) bit for bit — on decode, paged and prefill
rows, on keys with planted hot positions, and with candidate capacities small
enough that rows take the full-row path — and the fused forward's output must equal
the unfused forward's. One case is also checked against the oracle directly."""

import numpy as np
import pytest
import torch

from oracle import indexer_scores, topk_rows
from sparse_attention_05_b200 import synth
from tests.helpers import check_index_sets, oracle_args

pytestmark = pytest.mark.gpu


def _dsa():
    from sparse_attention_05_b200 import dsa
    return dsa


def _both(p, k=2048, cand_cap=0):
    dsa = _dsa()
    g = p.to("cuda")
    kv = dsa.KvLayout.of(g)
    scores = dsa.dsa_indexer_scores(g.q_idx, g.w, g.k_idx, g.k_scale, kv, p.q_per_seq)
    ref = dsa.dsa_topk(scores, kv, p.q_per_seq, k)
    got = dsa.dsa_select_fused(g.q_idx, g.w, g.k_idx, g.k_scale, kv, p.q_per_seq, k,
                               cand_cap=cand_cap)
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == 0
    return got.cpu().numpy(), ref.cpu().numpy()


def test_decode_rows_equal_the_unfused_selection():
    got, ref = _both(synth.decode(batch=8, ctx=20000, q_per_seq=1, seed=120))
    assert np.array_equal(got, ref)


def test_paged_varlen_two_rows_equal_the_unfused_selection():
    got, ref = _both(synth.paged_decode(batch=6, q_per_seq=2, min_ctx=1500, max_ctx=30000,
                                        page_size=64, seed=121))
    assert np.array_equal(got, ref)


def test_prefill_rows_below_and_above_k():
    got, ref = _both(synth.prefill(L=5000, seed=122))
    assert np.array_equal(got, ref)


def test_hot_positions():
    """Planted high-scoring keys (the 128K prefill's structure, at 6K)."""
    got, ref = _both(synth.prefill(L=6000, seed=123, n_hot=64))
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("cap", [2048, 2600])
def test_small_candidate_capacity_takes_the_full_row_path(cap):
    """With at most k (or k + 552) candidates per row nearly every long row overflows
    its list and is selected from its full score row: still identical."""
    got, ref = _both(synth.decode(batch=4, ctx=12000, q_per_seq=2, seed=124), cand_cap=cap)
    assert np.array_equal(got, ref)


def test_small_k():
    got, ref = _both(synth.decode(batch=4, ctx=9000, q_per_seq=1, seed=125), k=100)
    assert np.array_equal(got, ref)


def test_against_the_oracle():
    p = synth.decode(batch=3, ctx=7000, q_per_seq=2, seed=126)
    got, _ = _both(p)
    a = oracle_args(p)
    sc = indexer_scores(a["q_idx"], a["w"], a["k_idx"], a["k_scale"], a["q_seq"], a["q_pos"],
                        ld=7040)
    check_index_sets(got, topk_rows(sc, a["q_pos"], 2048), sc, a["q_pos"], 2048)


def test_paged_long_rows_against_the_oracle():
    """Paged varlen decode with rows past 4k keys (the sampled threshold and the
    filtering pass decide them): the fused selection against the oracle's top-k of
    the oracle's scores."""
    p = synth.paged_decode(batch=3, q_per_seq=2, min_ctx=9000, max_ctx=20000, page_size=64,
                           seed=129)
    got, _ = _both(p)
    a = oracle_args(p)
    sc = indexer_scores(a["q_idx"], a["w"], a["k_idx"], a["k_scale"], a["q_seq"], a["q_pos"],
                        ld=(p.max_ctx + 127) // 128 * 128,
                        block_table=a["block_table"], page_size=p.page_size)
    check_index_sets(got, topk_rows(sc, a["q_pos"], 2048), sc, a["q_pos"], 2048)


def test_fused_forward_equals_forward():
    dsa = _dsa()
    p = synth.paged_decode(batch=4, q_per_seq=2, min_ctx=3000, max_ctx=16000, page_size=64,
                           seed=127).to("cuda")
    kv = dsa.KvLayout.of(p)
    o0, l0, _ = dsa.dsa_forward(p.q_idx, p.w, p.k_idx, p.k_scale, p.q, p.kv, kv, p.q_per_seq,
                                2048, p.scale)
    o1, l1, _ = dsa.dsa_forward_fused(p.q_idx, p.w, p.k_idx, p.k_scale, p.q, p.kv, kv,
                                      p.q_per_seq, 2048, p.scale)
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == 0
    assert torch.equal(o0, o1) and torch.equal(l0, l1)


def test_host_argument_checks():
    dsa = _dsa()
    p = synth.decode(batch=2, ctx=300, q_per_seq=1, seed=128).to("cuda")
    kv = dsa.KvLayout.of(p)
    with pytest.raises(dsa.DSAError) as e:
        dsa.dsa_select_fused(p.q_idx, p.w, p.k_idx, p.k_scale, kv, 1, 64, cand_cap=9000)
    assert e.value.status == 1
    big = dsa.KvLayout(batch=2, max_ctx=140000, seqlens=p.seqlens)
    with pytest.raises(dsa.DSAError) as e:
        dsa.dsa_select_fused(p.q_idx, p.w, p.k_idx, p.k_scale, big, 1, 64,
                             workspace=torch.empty(1 << 20, dtype=torch.uint8, device="cuda"))
    assert e.value.status == 2
