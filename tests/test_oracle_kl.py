"""Pins of the oracle's indexer KL loss term ([TR] §2.1): closed forms, Gibbs'
inequality, library routines (torch softmax / log_softmax / kl_div in fp64) and
set invariances."""

import math

import numpy as np
import torch

from oracle import dense_indexer_kl, indexer_kl_token, sparse_indexer_kl


def test_closed_form_uniform_attention_two_keys():
    # q = 0: every head attends uniformly, p = (1/2, 1/2); I = (0, ln 2) gives
    # softmax(I) = (1/3, 2/3), KL = 1/2 ln(3/2) + 1/2 ln(3/4) = 1/2 ln(9/8)
    got = indexer_kl_token(np.zeros((4, 3)), np.ones((2, 3)), np.array([0.0, math.log(2.0)]), 0.3)
    assert abs(got - 0.5 * math.log(9.0 / 8.0)) < 1e-14


def test_single_key_and_empty_set_give_zero():
    rng = np.random.default_rng(1)
    assert indexer_kl_token(rng.normal(size=(8, 5)), rng.normal(size=(1, 5)), np.array([3.0]),
                            0.4) == 0.0
    assert indexer_kl_token(rng.normal(size=(8, 5)), np.zeros((0, 5)), np.zeros(0), 0.4) == 0.0


def _library_kl(q_t, kv_rows, scores, scale):
    """The same quantity from library routines: per-head softmax, head mean,
    log_softmax of the scores and torch's KL divergence (sum p (ln p - ln q))."""
    q_t = torch.as_tensor(q_t, dtype=torch.float64)
    c = torch.as_tensor(kv_rows, dtype=torch.float64)
    a = torch.softmax(scale * q_t @ c.T, dim=1)
    p = a.mean(dim=0)
    log_q = torch.log_softmax(torch.as_tensor(scores, dtype=torch.float64), dim=0)
    return float(torch.nn.functional.kl_div(log_q, p, reduction="sum"))


def test_matches_library_routines_and_is_nonnegative():
    rng = np.random.default_rng(2)
    for n in (2, 7, 64, 300):
        q_t = rng.normal(size=(16, 24))
        kv = rng.normal(size=(n, 24)) * 0.7
        scores = rng.normal(size=n) * 3.0
        got = indexer_kl_token(q_t, kv, scores, 24 ** -0.5)
        ref = _library_kl(q_t, kv, scores, 24 ** -0.5)
        assert got >= 0.0                      # Gibbs' inequality
        assert abs(got - ref) <= 1e-12 * max(1.0, abs(ref))


def test_zero_when_scores_are_log_target_plus_constant():
    rng = np.random.default_rng(3)
    q_t = rng.normal(size=(8, 16))
    kv = rng.normal(size=(40, 16))
    a = torch.softmax(torch.as_tensor(0.25 * q_t @ kv.T), dim=1)
    p = a.mean(dim=0).numpy()
    got = indexer_kl_token(q_t, kv, np.log(p) + 5.0, 0.25)
    assert abs(got) < 1e-13


def _rows_problem(seed):
    rng = np.random.default_rng(seed)
    T, H, D, L = 3, 4, 10, 50
    q = rng.normal(size=(T, H, D))
    kv = rng.normal(size=(1, L, D))
    q_seq = np.zeros(T, np.int64)
    q_pos = np.array([9, 30, 49])
    scores = rng.normal(size=(T, 64))
    return q, kv, q_seq, q_pos, scores, rng


def test_set_invariances_permutation_padding_and_dense():
    q, kv, q_seq, q_pos, scores, rng = _rows_problem(4)
    idx = np.stack([np.sort(rng.choice(int(p) + 1, 8, replace=False)) for p in q_pos])
    base = sparse_indexer_kl(q, kv, q_seq, q_pos, idx, scores, 0.3)
    perm = np.stack([rng.permutation(r) for r in idx])
    assert np.allclose(sparse_indexer_kl(q, kv, q_seq, q_pos, perm, scores, 0.3), base,
                       rtol=1e-12, atol=1e-15)
    padded = np.concatenate([idx, np.full((3, 4), -1), np.full((3, 2), 999)], axis=1)
    assert np.allclose(sparse_indexer_kl(q, kv, q_seq, q_pos, padded, scores, 0.3), base,
                       rtol=1e-12, atol=1e-15)
    full = [np.arange(int(p) + 1) for p in q_pos]
    assert np.allclose(dense_indexer_kl(q, kv, q_seq, q_pos, scores, 0.3),
                       sparse_indexer_kl(q, kv, q_seq, q_pos, full, scores, 0.3), rtol=0, atol=0)
    # each row's term is the per-token function on that row's own keys and scores
    for r, t in enumerate(range(3)):
        ref = _library_kl(q[t], kv[0, idx[r]], scores[r, idx[r]], 0.3)
        assert abs(base[r] - ref) <= 1e-12 * max(1.0, ref)
