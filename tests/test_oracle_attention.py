"""Pins for the oracle's sparse MLA (MQA mode): a hand-worked example, dense
causal MQA against PyTorch's scaled_dot_product_attention (fp64, CPU), closed
forms (identical keys, one-hot queries, a constant value column) and
invariances (index permutation, -1 / out-of-range entries)."""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import dense_causal_mqa, sparse_mla, sparse_mla_token, dsa_forward
from sparse_attention_05_b200 import synth
from tests.helpers import oracle_args

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_golden_hand_example():
    g = json.load(open(os.path.join(GOLDEN, "attention_hand.json")))
    o, lse = sparse_mla_token(np.array(g["q"]), np.array(g["kv"]), g["scale"], g["d_v"])
    np.testing.assert_allclose(o, np.array(g["expected_o"]), rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, np.array(g["expected_lse"]), rtol=0, atol=1e-15)


def _sdpa_dense(q, kv, scale, d_v):
    """Causal MQA through torch SDPA (fp64): keys = kv, values = kv[:, :d_v]."""
    L, H, D = q.shape
    qt = torch.from_numpy(q).double().permute(1, 0, 2)                 # [H, L, D]
    k = torch.from_numpy(kv).double()[None].expand(H, L, D)
    v = torch.from_numpy(kv[:, :d_v]).double()[None].expand(H, L, d_v)
    o = torch.nn.functional.scaled_dot_product_attention(qt, k, v, is_causal=True, scale=scale)
    return o.permute(1, 0, 2).numpy()


@pytest.mark.parametrize("dims,L", [(synth.TINY, 256), (synth.Dims(heads=4, topk=64), 96)])
def test_dense_matches_torch_sdpa(dims, L):
    p = synth.tiny(L=L, dims=dims) if dims is synth.TINY else \
        synth.prefill(L=L, seed=12, dims=dims)
    a = oracle_args(p)
    o, lse = dense_causal_mqa(a["q"], a["kv"], a["q_seq"], a["q_pos"], p.scale, dims.d_v)
    want = _sdpa_dense(a["q"], a["kv"][0], p.scale, dims.d_v)
    np.testing.assert_allclose(o, want, rtol=1e-10, atol=1e-12)


def test_dsa_with_k_at_least_t_equals_dense():
    """k >= pos + 1 selects every visible key, so DSA reduces to dense causal MQA."""
    p = synth.tiny(L=64)
    a = oracle_args(p)
    res = dsa_forward(a["q_idx"], a["w"], a["k_idx"], None, a["q"], a["kv"], a["q_seq"],
                      a["q_pos"], k=64, scale=p.scale, d_v=64, ld=64, fp8=False)
    o, lse = dense_causal_mqa(a["q"], a["kv"], a["q_seq"], a["q_pos"], p.scale, 64)
    np.testing.assert_array_equal(res["o"], o)
    np.testing.assert_array_equal(res["lse"], lse)
    want = _sdpa_dense(a["q"], a["kv"][0], p.scale, 64)
    np.testing.assert_allclose(res["o"], want, rtol=1e-10, atol=1e-12)


def test_rows_below_k_are_dense_in_tiny_config():
    p = synth.tiny(L=256)
    a = oracle_args(p)
    res = dsa_forward(a["q_idx"], a["w"], a["k_idx"], None, a["q"], a["kv"], a["q_seq"],
                      a["q_pos"], k=32, scale=p.scale, d_v=64, ld=256, fp8=False)
    o, _ = dense_causal_mqa(a["q"], a["kv"], a["q_seq"], a["q_pos"], p.scale, 64, rows=range(32))
    np.testing.assert_array_equal(res["o"][:32], o)
    # beyond k the selection is a strict subset, so outputs differ from dense
    o2, _ = dense_causal_mqa(a["q"], a["kv"], a["q_seq"], a["q_pos"], p.scale, 64, rows=[200])
    assert np.abs(res["o"][200] - o2[0]).max() > 1e-3


def test_weights_sum_to_one_via_constant_value_column():
    rng = np.random.default_rng(4)
    kv = rng.standard_normal((50, 24))
    kv[:, 0] = 1.0  # value dim 0 is constant, so o[:, 0] = sum of softmax weights
    q = rng.standard_normal((6, 24))
    o, _ = sparse_mla_token(q, kv, 0.3, 8)
    np.testing.assert_allclose(o[:, 0], 1.0, rtol=0, atol=1e-12)


def test_identical_keys_closed_form():
    rng = np.random.default_rng(5)
    c = rng.standard_normal(24)
    q = rng.standard_normal((3, 24))
    n = 37
    o, lse = sparse_mla_token(q, np.tile(c, (n, 1)), 0.5, 10)
    np.testing.assert_allclose(o, np.tile(c[:10], (3, 1)), atol=1e-12)
    np.testing.assert_allclose(lse, 0.5 * (q @ c) + math.log(n), atol=1e-12)


def test_single_key_one_hot_query():
    rng = np.random.default_rng(6)
    c = rng.standard_normal((1, 16))
    q = np.zeros((16, 16))
    q[np.arange(16), np.arange(16)] = 2.0  # head h reads dim h
    o, lse = sparse_mla_token(q, c, 0.25, 12)
    np.testing.assert_array_equal(o, np.tile(c[0, :12], (16, 1)))
    np.testing.assert_allclose(lse, 0.5 * c[0], atol=1e-15)


def test_permutation_and_padding_invariance():
    p = synth.decode(batch=2, ctx=200, q_per_seq=2, seed=13, dims=synth.Dims(heads=4, topk=64))
    a = oracle_args(p)
    rng = np.random.default_rng(0)
    idx = np.stack([np.sort(rng.choice(int(a["q_pos"][t]) + 1, 64, replace=False))
                    for t in range(p.num_q)]).astype(np.int32)
    o1, l1 = sparse_mla(a["q"], a["kv"], a["q_seq"], a["q_pos"], idx, p.scale, 512)
    perm = np.stack([rng.permutation(r) for r in idx])
    o2, l2 = sparse_mla(a["q"], a["kv"], a["q_seq"], a["q_pos"], perm, p.scale, 512)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l2, l1, rtol=1e-13, atol=1e-13)
    # -1 and entries beyond the query position are ignored
    extra = np.concatenate([idx, np.full((p.num_q, 3), -1, np.int32),
                            (a["q_pos"][:, None] + 1 + np.arange(2)[None]).astype(np.int32)], 1)
    o3, l3 = sparse_mla(a["q"], a["kv"], a["q_seq"], a["q_pos"], extra, p.scale, 512)
    np.testing.assert_array_equal(o3, o1)
    np.testing.assert_array_equal(l3, l1)


def test_disjoint_parts_merge_to_the_whole_selection():
    """Attention over a set equals the merge of attention over disjoint parts of it:
    LSE = ln sum_s e^{LSE_s}, o = sum_s e^{LSE_s - LSE} o_s (an empty part has
    LSE = -inf and weight 0). The split rows of the GPU path rely on this identity."""
    p = synth.decode(batch=2, ctx=300, q_per_seq=1, seed=15, dims=synth.Dims(heads=4, topk=96))
    a = oracle_args(p)
    rng = np.random.default_rng(2)
    idx = np.stack([rng.choice(int(a["q_pos"][t]) + 1, 96, replace=False)
                    for t in range(p.num_q)]).astype(np.int32)
    o, l = sparse_mla(a["q"], a["kv"], a["q_seq"], a["q_pos"], idx, p.scale, 512)
    parts = [idx[:, :40], idx[:, 40:41], np.full((p.num_q, 5), -1, np.int32), idx[:, 41:]]
    res = [sparse_mla(a["q"], a["kv"], a["q_seq"], a["q_pos"], x, p.scale, 512) for x in parts]
    ls = np.stack([r[1] for r in res])                       # [parts, T, H]
    lse = np.logaddexp.reduce(ls, axis=0)
    wts = np.exp(ls - lse[None])                             # empty part: exp(-inf) = 0
    om = sum(w[..., None] * r[0] for w, r in zip(wts, res))
    np.testing.assert_allclose(lse, l, rtol=1e-13, atol=1e-12)
    np.testing.assert_allclose(om, o, rtol=1e-11, atol=1e-12)
    assert np.all(np.isneginf(ls[2]))


def test_empty_selection():
    o, lse = sparse_mla_token(np.ones((2, 8)), [], 1.0, 4)
    assert np.all(o == 0) and np.all(np.isneginf(lse))


def test_paged_equals_contiguous():
    p = synth.paged_decode(batch=2, q_per_seq=2, min_ctx=70, max_ctx=200, seed=14,
                           dims=synth.Dims(heads=4))
    a = oracle_args(p)
    rng = np.random.default_rng(1)
    idx = np.stack([rng.choice(int(a["q_pos"][t]) + 1, 32, replace=False)
                    for t in range(p.num_q)]).astype(np.int32)
    o_p, l_p = sparse_mla(a["q"], a["kv"], a["q_seq"], a["q_pos"], idx, p.scale, 512,
                          block_table=a["block_table"], page_size=64)
    bt = a["block_table"]
    kvc = np.zeros((p.batch, p.max_ctx, 576), np.float32)
    for b in range(p.batch):
        for s in range(int(p.seqlens[b])):
            kvc[b, s] = a["kv"][bt[b, s // 64], s % 64]
    o_c, l_c = sparse_mla(a["q"], kvc, a["q_seq"], a["q_pos"], idx, p.scale, 512)
    np.testing.assert_array_equal(o_p, o_c)
    np.testing.assert_array_equal(l_p, l_c)
