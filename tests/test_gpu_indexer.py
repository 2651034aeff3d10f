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


_BF16_POS = (np.arange(1, 0x7F80, dtype=np.uint32) << 16).view(np.float32)  # positive finite bf16


def _midpoint_distance(x: np.ndarray, amax) -> np.ndarray:
    """fp32 ulps between RN(x / s_q) (s_q = RN(amax / 448)) and the nearest
    E4M3 rounding midpoint, for quotients in the normal E4M3 range."""
    s_q = np.float32(amax) / np.float32(448.0)
    quot = (x / s_q).astype(np.float32)
    rem = (quot.view(np.uint32) & 0xFFFFF).astype(np.int64)
    return np.where(quot >= np.float32(2.0 ** -6), np.abs(rem - 0x80000), 1 << 30)


def _near_midpoint_row(rng) -> np.ndarray:
    """128 bf16 values, the hardest inputs for the query quantization: amax is
    chosen among bf16 values in [0.5, 8) so that many values below it have a
    fp32 quotient RN(x / s_q) within a few ulps of an E4M3 rounding midpoint
    (or exactly on one, where ties-to-even decides); the row is amax plus the
    127 values closest to midpoints, with random signs, in random order."""
    amaxes = _BF16_POS[(_BF16_POS >= 0.5) & (_BF16_POS < 8.0)]
    best = []
    for amax in rng.choice(amaxes, 48, replace=False):
        d = _midpoint_distance(_BF16_POS[_BF16_POS < amax], amax)
        best.append((int(d.min()), -int((d <= 16).sum()), float(amax)))
    amax = np.float32(min(best)[2])
    x = _BF16_POS[_BF16_POS < amax]
    pick = x[np.argsort(_midpoint_distance(x, amax), kind="stable")[:127]]
    row = np.concatenate([[amax], pick * rng.choice([-1.0, 1.0], 127)])
    return rng.permutation(row).astype(np.float32)


def test_query_codes_exact_via_one_hot_keys():
    """Every E4M3 query code is checked exactly: keys are +-e_i (scale 1) and
    each row weights one head by 1, so score(row, key +-e_i) = RN(s_q * ReLU(
    +-q_hat_i)) on both sides; the GPU must equal the oracle bit for bit.
    Half the rows hold values whose quotients sit next to E4M3 midpoints."""
    B, H, D = 64, 64, 128
    p = synth.decode(batch=B, ctx=2 * D, q_per_seq=1, seed=36)
    rng = np.random.default_rng(36)
    q = p.q_idx.float().numpy().copy()
    for b in range(B):
        if b % 2 == 0:
            q[b, b % H] = _near_midpoint_row(rng)
    p.q_idx = torch.from_numpy(q).to(torch.bfloat16)
    assert torch.equal(p.q_idx.float(), torch.from_numpy(q))  # values are bf16-exact
    w = np.zeros((B, H), np.float32)
    w[np.arange(B), np.arange(B) % H] = 1.0
    p.w = torch.from_numpy(w)
    codes = np.zeros((B, 2 * D, D), np.uint8)
    for i in range(D):
        codes[:, i, i] = 0x38        # +1.0 in E4M3
        codes[:, D + i, i] = 0xB8    # -1.0
    p.k_idx = torch.from_numpy(codes)
    p.k_scale = torch.ones(B, 2 * D)
    got = _gpu_scores(p)
    a = oracle_args(p)
    ref = indexer_scores(a["q_idx"], a["w"], a["k_idx"], a["k_scale"], a["q_seq"], a["q_pos"],
                         ld=got.shape[1], block_table=None)
    bad = got[:, :2 * D] != ref[:, :2 * D]
    assert not bad.any(), f"{bad.sum()} scores differ; first at {np.argwhere(bad)[0]}"
