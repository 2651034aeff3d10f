"""GPU parity of dsa_topk against the oracle's selection: exact match on
seeded score rows (tie-heavy, signed zeros, negatives, rows shorter than k,
rows longer than the kernel's shared-memory row cache)."""

import numpy as np
import pytest
import torch

from oracle import topk_rows

pytestmark = pytest.mark.gpu


def _dsa():
    from sparse_attention_05_b200 import dsa
    return dsa


def _run(scores_np, seqlens, q_per_seq, k):
    """dsa_topk (one CTA per row) and dsa_topk_ws (long rows split across CTAs) on
    the same rows: both must equal the oracle's selection; returns the one-CTA
    result (and checks the split one inside)."""
    dsa = _dsa()
    T, ld = scores_np.shape
    B = len(seqlens)
    kv = dsa.KvLayout(batch=B, max_ctx=ld,
                      seqlens=torch.tensor(seqlens, dtype=torch.int32, device="cuda"))
    s = torch.from_numpy(scores_np).cuda()
    idx = dsa.dsa_topk(s, kv, q_per_seq, k)
    idx_split = dsa.dsa_topk_ws(s, kv, q_per_seq, k)
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == 0
    pos = np.array([seqlens[t // q_per_seq] - q_per_seq + t % q_per_seq for t in range(T)])
    want = topk_rows(scores_np, pos, k)
    np.testing.assert_array_equal(idx_split.cpu().numpy(), want)
    return idx.cpu().numpy(), want


def _rows(rng, T, ld, kind):
    if kind == "normal":
        return rng.standard_normal((T, ld)).astype(np.float32)
    if kind == "ties":
        pool = np.array([0.0, -0.0, 1.0, 1.5, 2.0, -3.0, 7.25], np.float32)
        return rng.choice(pool, size=(T, ld)).astype(np.float32)
    if kind == "narrow":  # all values within one binade: stresses the top radix digit
        return (1.0 + rng.random((T, ld)) * 0.5).astype(np.float32)
    if kind == "quantized":  # few distinct values, many exact ties at the threshold
        return (rng.integers(0, 300, (T, ld)) / 64.0).astype(np.float32)
    raise ValueError(kind)


@pytest.mark.parametrize("kind", ["normal", "ties", "narrow", "quantized"])
def test_decode_rows(kind):
    rng = np.random.default_rng(hash(kind) % 2**32)
    ld = 32768
    seqlens = [32768, 2048, 2049, 100, 1, 30001, 4097, 16384]
    s = _rows(rng, len(seqlens), ld, kind)
    got, want = _run(s, seqlens, 1, 2048)
    np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("k", [1, 7, 64, 2047, 2048])
def test_various_k(k):
    rng = np.random.default_rng(k)
    seqlens = [5000, 3, 2048, 9000]
    s = _rows(rng, 4, 9216, "quantized")
    got, want = _run(s, seqlens, 1, k)
    np.testing.assert_array_equal(got, want)


def test_long_rows_beyond_row_cache():
    rng = np.random.default_rng(7)
    seqlens = [131072, 40961, 65536, 99999]
    s = _rows(rng, 4, 131072, "ties")
    s[1] = rng.standard_normal(131072).astype(np.float32)
    got, want = _run(s, seqlens, 1, 2048)
    np.testing.assert_array_equal(got, want)


def test_prefill_rows_two_queries_per_sequence_and_causal_rows():
    rng = np.random.default_rng(9)
    # paged-decode geometry: 2 query rows per sequence
    seqlens = [4096, 70000, 2049, 2050]
    s = _rows(rng, 8, 70016, "normal")
    got, want = _run(s, seqlens, 2, 2048)
    np.testing.assert_array_equal(got, want)
    # prefill geometry: one sequence, every row its own causal length
    L = 3000
    s = _rows(rng, L, L, "quantized")
    got, want = _run(s, [L], L, 2048)
    np.testing.assert_array_equal(got, want)


def test_masked_tail_is_never_read():
    rng = np.random.default_rng(10)
    s = rng.standard_normal((2, 8192)).astype(np.float32)
    s[0, 5000:] = np.inf  # beyond pos: must be ignored
    s[1, 3000:] = np.nan
    got, want = _run(s, [5000, 3000], 1, 2048)
    np.testing.assert_array_equal(got, want)


def test_split_rows_whose_sample_misjudges_take_the_full_row_path():
    """Rows built so that the strided sample's threshold is useless: the sampled
    positions hold the row's largest scores (fewer than k candidates pass), or its
    smallest (nearly every key passes, more than the candidate list holds). The
    split selection must still be exact (it falls back to the whole row)."""
    rng = np.random.default_rng(11)
    n = 131072
    rows = np.empty((3, n), np.float32)
    sampled = (np.arange(2048, dtype=np.int64) * n) // 2048
    rows[0] = rng.standard_normal(n).astype(np.float32)
    rows[0][sampled] = 100.0 + rng.random(2048).astype(np.float32)  # threshold too high
    rows[1] = 10.0 + rng.random(n).astype(np.float32)
    rows[1][sampled] = -100.0                                         # threshold too low
    rows[2] = rng.standard_normal(n).astype(np.float32)               # a plain row
    got, want = _run(rows, [n, n, 70001], 1, 2048)
    np.testing.assert_array_equal(got, want)


def test_split_chunk_edges_and_hot_ties():
    """Rows whose lengths end just past, at and before chunk edges (16384 keys), with
    the top scores tied across chunk boundaries."""
    rng = np.random.default_rng(12)
    ld = 65536
    seqlens = [16384, 16385, 32767, 8193, 49153, 65536]
    s = (rng.integers(0, 40, (len(seqlens), ld)) / 8.0).astype(np.float32)
    s[:, 16380:16390] = 9.0  # ties straddling the first chunk edge
    got, want = _run(s, seqlens, 1, 2048)
    np.testing.assert_array_equal(got, want)


def test_rows_longer_than_the_position_bitmaps():
    """Rows of more than 131072 keys keep their candidates in position order (the
    bitmap selection covers shorter rows only): plain, tie-heavy and sample-misjudged
    rows must still match the oracle exactly."""
    rng = np.random.default_rng(13)
    ld = 200000
    seqlens = [200000, 150001, 131073, 199999]
    s = rng.standard_normal((4, ld)).astype(np.float32)
    pool = np.array([0.0, -0.0, 1.0, 1.5, 2.0, -3.0, 7.25], np.float32)
    s[1] = rng.choice(pool, size=ld)
    sampled = (np.arange(2048, dtype=np.int64) * seqlens[3]) // 2048
    s[3][sampled] = 100.0 + rng.random(2048).astype(np.float32)  # threshold too high
    got, want = _run(s, seqlens, 1, 2048)
    np.testing.assert_array_equal(got, want)
