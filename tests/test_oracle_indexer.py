"""Pins for the oracle's lightning-indexer scores: a hand-worked example, a
brute-force re-implementation on tiny inputs (library FP8 casts), closed forms
(single head = ReLU of a matmul, exact key-scale homogeneity, lossless query
quantization) and invariants (non-negativity for w >= 0, causal mask, paged ==
contiguous)."""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import e4m3_decode, indexer_scores, quantize_indexer_query
from sparse_attention_05_b200 import synth
from tests.helpers import oracle_args

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _scores(p, rows=None):
    a = oracle_args(p)
    return indexer_scores(a["q_idx"], a["w"], a["k_idx"], a["k_scale"], a["q_seq"], a["q_pos"],
                          ld=p.max_ctx, rows=rows, fp8=p.fp8, block_table=a["block_table"],
                          page_size=p.page_size)


def test_golden_hand_example():
    g = json.load(open(os.path.join(GOLDEN, "indexer_hand.json")))
    q = np.array(g["q_idx"], np.float32)
    w = np.array(g["w"], np.float32)
    keys = np.array(g["keys"], np.float32)[None]
    got = indexer_scores(q, w, keys, None, [0], [g["pos"]], ld=keys.shape[1], fp8=False)
    want = np.array([float(v) for v in g["expected"]], np.float32)
    np.testing.assert_array_equal(got[0], want)


def test_single_head_unit_weight_is_relu_of_matmul():
    rng = np.random.default_rng(3)
    L, d = 40, 16
    q = rng.standard_normal((L, 1, d)).astype(np.float32)
    k = rng.standard_normal((1, L, d)).astype(np.float32)
    got = indexer_scores(q, np.ones((L, 1), np.float32), k, None, np.zeros(L, int), np.arange(L),
                         ld=L, fp8=False)
    full = np.maximum(np.matmul(q[:, 0, :].astype(np.float64), k[0].T.astype(np.float64)), 0)
    want = np.where(np.tril(np.ones((L, L), bool)), full, -np.inf).astype(np.float32)
    np.testing.assert_array_equal(got, want)


def _bruteforce_fp8(q_bf16, w, codes, kscale, pos):
    """Pure-Python loops; FP8 via PyTorch's e4m3 cast, not the oracle's codec."""
    H, d = q_bf16.shape
    out = []
    qhat, sq = [], []
    for j in range(H):
        amax = max(abs(float(v)) for v in q_bf16[j])
        s = np.float32(max(amax, 2.0 ** -120)) / np.float32(448.0)
        quot = torch.tensor([np.float32(v) / s for v in q_bf16[j]], dtype=torch.float32)
        qhat.append(quot.to(torch.float8_e4m3fn).double().tolist())
        sq.append(float(s))
    kdec = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).double().numpy()
    for s_ in range(pos + 1):
        tot = 0.0
        for j in range(H):
            dot = sum(qhat[j][i] * kdec[s_][i] for i in range(d))
            tot += float(w[j]) * sq[j] * max(0.0, dot)
        out.append(np.float32(float(kscale[s_]) * tot))
    return np.array(out, np.float32)


def test_bruteforce_fp8_tiny():
    dims = synth.Dims(h_idx=3, d_idx=8, heads=2, d_qk=16, d_v=8, topk=4)
    p = synth.decode(batch=2, ctx=24, q_per_seq=3, seed=11, dims=dims)
    got = _scores(p)
    a = oracle_args(p)
    for t in range(p.num_q):
        b, pos = int(a["q_seq"][t]), int(a["q_pos"][t])
        want = _bruteforce_fp8(a["q_idx"][t], a["w"][t], a["k_idx"][b], a["k_scale"][b], pos)
        np.testing.assert_allclose(got[t, :pos + 1], want, rtol=1e-6, atol=0)
        assert np.all(np.isneginf(got[t, pos + 1:]))


def test_nonnegative_for_nonnegative_weights_and_causal_mask():
    p = synth.decode(batch=3, ctx=300, q_per_seq=2, seed=5, dims=synth.Dims(topk=64))
    s = _scores(p)
    pos = p.q_pos().numpy()
    for t in range(p.num_q):
        assert np.all(s[t, :pos[t] + 1] >= 0)
        assert np.all(np.isneginf(s[t, pos[t] + 1:]))
    assert (s[np.isfinite(s)] > 0).mean() > 0.9


def test_key_scale_homogeneity_is_exact():
    p = synth.decode(batch=2, ctx=200, q_per_seq=1, seed=6)
    s1 = _scores(p)
    p.k_scale = p.k_scale * 4.0
    s4 = _scores(p)
    fin = np.isfinite(s1)
    np.testing.assert_array_equal(s4[fin], 4.0 * s1[fin])


def test_query_quantization_lossless_on_representable_rows():
    rng = np.random.default_rng(7)
    fin = e4m3_decode(np.arange(0, 127, dtype=np.uint8))  # non-negative finite codes
    v = rng.choice(fin, size=(5, 4, 32)) * np.where(rng.random((5, 4, 32)) < 0.5, -1, 1)
    v[..., 0] = 448.0  # amax of every row is exactly 448
    s = np.exp2(rng.integers(-8, 8, size=(5, 4))).astype(np.float32)
    q = (v * s[..., None]).astype(np.float32)
    codes, s_q = quantize_indexer_query(q)
    np.testing.assert_array_equal(s_q, s)
    np.testing.assert_array_equal(e4m3_decode(codes), v)


def test_zero_query_row_gives_zero_scores():
    p = synth.decode(batch=1, ctx=64, q_per_seq=1, seed=8)
    p.q_idx[0, 5:9] = 0
    p.w[0, :5] = 0
    p.w[0, 9:] = 0
    s = _scores(p)
    assert np.all(s[0] == 0.0)


def test_paged_equals_contiguous():
    p = synth.paged_decode(batch=3, q_per_seq=2, min_ctx=100, max_ctx=400, page_size=64, seed=9)
    a = oracle_args(p)
    paged = indexer_scores(a["q_idx"], a["w"], a["k_idx"], a["k_scale"], a["q_seq"], a["q_pos"],
                           ld=p.max_ctx, block_table=a["block_table"], page_size=64)
    # rebuild each sequence contiguously by walking its block table
    B, ctx = p.batch, p.max_ctx
    kc = np.zeros((B, ctx, 128), np.uint8)
    ks = np.zeros((B, ctx), np.float32)
    bt = a["block_table"]
    for b in range(B):
        for s in range(int(p.seqlens[b])):
            kc[b, s] = a["k_idx"][bt[b, s // 64], s % 64]
            ks[b, s] = a["k_scale"][bt[b, s // 64], s % 64]
    contig = indexer_scores(a["q_idx"], a["w"], kc, ks, a["q_seq"], a["q_pos"], ld=ctx)
    np.testing.assert_array_equal(paged, contig)


def test_tiny_config_runs_and_is_causal():
    p = synth.tiny()
    s = _scores(p)
    assert s.shape == (256, 256)
    assert np.all(np.isneginf(s[np.triu_indices(256, 1)]))
    assert np.all(s[np.tril_indices(256)] >= 0)
