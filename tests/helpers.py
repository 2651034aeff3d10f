"""Shared test helpers: turn a seeded synthetic problem into oracle arguments and
compare results with the tolerances the parity tests use."""

from __future__ import annotations

import numpy as np
import torch

# Tolerances of the parity contract (written here, used by every parity test).
SCORE_RTOL = 5e-3        # indexer scores vs the FP8-emulated fp64 oracle
SCORE_FLOOR = 1e-3       # relative error measured against max(|ref|, floor * max|row|)
OUT_ATOL = 2e-2          # bf16 attention output, max abs
OUT_RTOL = 1e-2          # bf16 attention output, relative
LSE_ATOL = 1e-4          # fp32 log-sum-exp
TIE_RTOL = 1e-3          # index-set differences allowed only within this of the k-th score


def np32(x: torch.Tensor) -> np.ndarray:
    return x.detach().cpu().float().numpy()


def oracle_args(p):
    """numpy views of a synth.Problem in the form the oracle takes."""
    args = dict(
        q_idx=np32(p.q_idx), w=np32(p.w),
        k_idx=(p.k_idx.cpu().numpy() if p.fp8 else np32(p.k_idx)),
        k_scale=(np32(p.k_scale) if p.k_scale is not None else None),
        q=np32(p.q), kv=np32(p.kv),
        q_seq=p.q_seq().numpy(), q_pos=p.q_pos().numpy(),
        block_table=(p.block_table.cpu().numpy() if p.paged else None),
        page_size=p.page_size, fp8=p.fp8,
    )
    return args


def check_scores(gpu_rows: np.ndarray, ref_rows: np.ndarray, q_pos_rows: np.ndarray):
    """Scores on [0, pos] within SCORE_RTOL of the oracle; masked tail -inf."""
    worst = 0.0
    for r in range(ref_rows.shape[0]):
        n = int(q_pos_rows[r]) + 1
        ref = ref_rows[r, :n].astype(np.float64)
        got = gpu_rows[r, :n].astype(np.float64)
        denom = np.maximum(np.abs(ref), SCORE_FLOOR * np.max(np.abs(ref)))
        err = np.max(np.abs(got - ref) / denom) if n else 0.0
        worst = max(worst, float(err))
    assert worst <= SCORE_RTOL, f"indexer score rel err {worst:.3e} > {SCORE_RTOL}"
    return worst


def check_index_sets(gpu_idx: np.ndarray, ref_idx: np.ndarray, ref_scores: np.ndarray,
                     q_pos_rows: np.ndarray, k: int):
    """Index sets equal, except members of the symmetric difference whose oracle
    score lies within TIE_RTOL of the oracle's k-th score. Also checks the GPU
    list is ascending, unique, in range and padded with -1."""
    n_diff_total = 0
    for r in range(ref_idx.shape[0]):
        n = int(q_pos_rows[r]) + 1
        g = gpu_idx[r]
        valid = g[g >= 0]
        assert np.all(g[len(valid):] == -1), "padding must be -1 after the valid entries"
        assert len(valid) == min(k, n), f"row {r}: {len(valid)} selected, want {min(k, n)}"
        assert np.all(np.diff(valid) > 0), "indices must be ascending and unique"
        assert valid.min(initial=0) >= 0 and valid.max(initial=0) < n
        a, b = set(valid.tolist()), set(ref_idx[r][ref_idx[r] >= 0].tolist())
        diff = a ^ b
        if diff:
            row = ref_scores[r, :n].astype(np.float64)
            tau = np.sort(row)[::-1][min(k, n) - 1]
            for s in diff:
                assert abs(row[s] - tau) <= TIE_RTOL * abs(tau), \
                    f"row {r}: index {s} (score {row[s]}) differs, k-th score {tau}"
            n_diff_total += len(diff)
    return n_diff_total


def check_attention(o_gpu: np.ndarray, lse_gpu: np.ndarray, o_ref: np.ndarray, lse_ref: np.ndarray,
                    lse_tol=None, lse_bulk: float = 0.99):
    """bf16 output within OUT_ATOL abs and OUT_RTOL rel (per element, either
    bound suffices); LSE within LSE_ATOL. With ``lse_tol`` (an array shaped like
    lse_ref) each LSE is held to its own bound instead, and at least ``lse_bulk``
    of them must still be within LSE_ATOL."""
    o_gpu = o_gpu.astype(np.float64)
    err = np.abs(o_gpu - o_ref)
    bad = (err > OUT_ATOL) & (err > OUT_RTOL * np.abs(o_ref))
    assert not bad.any(), f"{bad.sum()} output elements out of tolerance; max abs err {err.max():.3e}"
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse_gpu), fin)
    lerr = np.abs(lse_gpu[fin].astype(np.float64) - lse_ref[fin])
    if lse_tol is None:
        assert lerr.max(initial=0.0) <= LSE_ATOL, f"LSE max abs err {lerr.max():.3e}"
    else:
        over = lerr > np.asarray(lse_tol)[fin]
        assert not over.any(), f"{over.sum()} LSE values beyond their bound; max err {lerr.max():.3e}"
        frac = float(np.mean(lerr <= LSE_ATOL)) if lerr.size else 1.0
        assert frac >= lse_bulk, f"only {frac:.4f} of LSE values within {LSE_ATOL}"
    return float(err.max(initial=0.0)), float(lerr.max(initial=0.0))


# fp32 accumulation of the 512-term up-projection dot products: at most 512 additions,
# each adding one rounding of at most 2^-24 relative (doubled: the tensor core's
# summation order and internal rounding are not specified)
UP_PROJ_GAMMA = 2 * 512 * 2.0 ** -24


def mha_lse_tolerance(q_mha, kv, q_seq, q_pos, sets, w_uk, scale, rows, *, block_table=None,
                      page_size=64):
    """Per (row, head) bound on |LSE_gpu - LSE_oracle| for MHA mode.

    The oracle rounds the exact fp64 keys W^UK c to bf16; the GPU rounds an fp32
    sum of the same 512 products, which lies within UP_PROJ_GAMMA * sum|c_i w_i|
    of the exact value, so a key element may land one bf16 step away only where
    its exact value is that close to a rounding midpoint. Such an element moves
    logit s by at most scale * |q_d| * (its bf16 step): delta_s. LSE(z + dz) -
    LSE(z) = ln sum_s p_s e^{dz_s}, so |dLSE| <= ln sum_s p_s e^{delta_s} with the
    oracle's weights p_s. Adds LSE_ATOL for the remaining fp32 arithmetic."""
    from oracle import bf16_round, resolve_kv_rows
    R, H = len(rows), q_mha.shape[1]
    tol = np.zeros((R, H))
    d_n = w_uk.shape[1]
    for b in sorted({int(q_seq[t]) for t in rows}):
        mine = [r for r, t in enumerate(rows) if int(q_seq[t]) == b]
        n = max(int(q_pos[rows[r]]) for r in mine) + 1
        c = np.asarray(resolve_kv_rows(kv, b, list(range(n)), block_table, page_size), np.float64)
        cl, ca = c[:, :512], np.abs(c[:, :512])
        for h in range(H):
            w = np.asarray(w_uk[h], np.float64)
            k_ex = cl @ w.T
            eps = UP_PROJ_GAMMA * (ca @ np.abs(w).T)
            step = np.abs(bf16_round(k_ex + eps).astype(np.float64) -
                          bf16_round(k_ex - eps).astype(np.float64))
            k_r = np.concatenate([bf16_round(k_ex).astype(np.float64), c[:, 512:]], axis=1)
            for r in mine:
                s = np.asarray(sets[r], np.int64)
                qv = np.asarray(q_mha[rows[r], h], np.float64)
                z = scale * (k_r[s] @ qv)
                pw = np.exp(z - (z.max() + np.log(np.sum(np.exp(z - z.max())))))
                delta = scale * (step[s] @ np.abs(qv[:d_n]))
                tol[r, h] = np.log(np.sum(pw * np.exp(delta))) + LSE_ATOL
    return tol
