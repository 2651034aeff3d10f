"""Pins for the oracle's top-k selection: hand-worked cases and brute force
with Python's sort on tiny, tie-heavy rows."""

import json
import os

import numpy as np
import pytest

from oracle import topk_rows, topk_select

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _brute(row, n, k):
    cand = sorted(range(n), key=lambda s: (-float(row[s]), s))[:k]
    out = sorted(cand) + [-1] * (k - min(k, n))
    return out


def test_golden_cases():
    g = json.load(open(os.path.join(GOLDEN, "topk_hand.json")))
    for c in g["cases"]:
        row = np.array([float(v) for v in c["scores"]], np.float32)
        got = topk_select(row, c["n"], c["k"]).tolist()
        assert got == c["expected"], (c, got)


@pytest.mark.parametrize("seed", range(20))
def test_bruteforce_tie_heavy(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 60))
    k = int(rng.integers(1, 70))
    pool = np.array([0.0, -0.0, 1.0, 2.5, -1.0, 7.0, 1e-30, -np.inf], np.float32)
    row = rng.choice(pool[: int(rng.integers(2, 9))], size=n + 5).astype(np.float32)
    got = topk_select(row, n, k).tolist()
    assert got == _brute(row, n, k)


def test_all_equal_row_takes_lowest_positions():
    row = np.full(100, 3.25, np.float32)
    assert topk_select(row, 100, 10).tolist() == list(range(10))


def test_n_equal_k_and_n_below_k():
    row = np.arange(16, dtype=np.float32)
    assert topk_select(row, 8, 8).tolist() == list(range(8))
    assert topk_select(row, 5, 8).tolist() == list(range(5)) + [-1] * 3
    assert topk_select(row, 9, 8).tolist() == list(range(1, 9))


def test_rows_use_their_own_positions():
    scores = np.array([[5, 1, 9, 9], [5, 1, 9, 9]], np.float32)
    got = topk_rows(scores, np.array([1, 3]), 2)
    assert got.tolist() == [[0, 1], [2, 3]]
