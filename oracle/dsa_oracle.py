"""Plain, slow, fp64 CPU oracle of the DeepSeek Sparse Attention (DSA) forward.

TEST INFRASTRUCTURE ONLY: used by ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py``. The CUDA library never imports it and it never
imports the CUDA library; the two share nothing but the seeded inputs.

Sources (web pages on DeepSeek-V3.2-Exp, cited by page and section):

* [TR]  "DeepSeek-V3.2-Exp ... 附完整论文中文翻译" (m.163.com), the Chinese
        translation of the DeepSeek-V3.2-Exp technical report.
        §1 "Architecture": lightning indexer (Eq. 1, image missing in the text),
        fine-grained token selection, attention output u_t (Eq. 2, image
        missing), MLA in MQA mode (Fig. 1). §2.1: the selected set
        S_t = {s | I_{t,s} in Top-k(I_{t,:})}, k = 2048.
* [OSR] "DeepSeek-V3.2开源技术报告" (nsmao.com), "DeepSeek稀疏注意力机制（DSA）原理":
        128-d indexer key cache per token, 512-d latent key cache, the four-step
        flow (projections -> indexer scores -> top-k -> sparse MLA).

Readings where the pages are silent:

* Indexer score, [TR] §1 Eq. 1 (missing image; the prose names H^I heads,
  q^I_{t,j} in R^{d_I}, a scalar weight w^I_{t,j}, keys k^I_s, ReLU):
  I_{t,s} = sum_j w_{t,j} * ReLU(q^I_{t,j} . k^I_s), no extra scale.
* FP8 ([TR] §1: "can be implemented in FP8"): keys arrive as E4M3 codes with one
  fp32 scale per token; the query row of each (token, head) is quantized to E4M3
  with scale s_q = max(amax, 2^-120) / 448 (fp32), codes = RNE-satfinite(q / s_q)
  with the division in fp32. Then
  I_{t,s} = s_k[s] * sum_j (w_{t,j} * s_q[t,j]) * ReLU(q_hat_{t,j} . k_hat_s),
  exact because ReLU(c x) = c ReLU(x) for c > 0.
* Causality: keys s <= pos(t) are visible (inclusive).
* Top-k ties: equal fp32 scores keep the lower position; -0.0 == +0.0. Output
  ascending by position, padded with -1 when fewer than k keys are visible.
* Attention ([TR] §1 Eq. 2 and Fig. 1, MQA mode): every head attends over the
  same selected latent rows c_s (576-d key = 512 latent + 64 rope), value =
  c_s[:512]; softmax with the given scale; LSE = ln sum_s exp(scale q.c_s).
  Entries of the index list outside [0, pos(t)] are ignored; an empty set gives
  o = 0 and LSE = -inf.
* Indexer training target ([TR] §2.1, loss equations missing): the main
  attention scores summed over the heads and L1-normalised along the sequence
  are read as the head-mean of the per-head softmax over the set (a
  distribution); the loss term of a row is KL(p || softmax(I)) over the set
  (all visible keys in the dense warm-up, S_t in the sparse stage).
* MLA in MHA mode ([TR] Appendix A, Fig. 4 missing) and its masked form for
  short prefill ([TR] §3): per head h the key is [W^UK_h c_s[:512] ; c_s[512:]]
  (the 64 rope dims shared by all heads) and the value W^UV_h c_s[:512], with
  128 nope query/key dims and 128 value dims per head (the pages give no
  per-head sizes); the decompressed keys and values are held in bf16. The mask
  of row t is its selected set S_t (plain causal when every visible key is
  selected); the softmax scale is the one MQA mode uses, so that both modes
  compute the same logits.

Parity pins live in tests/test_oracle_*.py. Parity with values printed by the
pages: unpinned (the pages print no worked values).
"""

from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
QSCALE_FLOOR = 2.0 ** -120

# --------------------------------------------------------------------------------------
# Number formats
# --------------------------------------------------------------------------------------


def bf16_round(x) -> np.ndarray:
    """Round fp32 values to the nearest bfloat16 (ties to even); returns fp32.

    bfloat16 keeps the top 16 bits of the IEEE binary32 pattern. Rounding to
    nearest-even on the dropped 16 bits: add 0x7FFF plus the lowest kept bit,
    then truncate. NaNs are passed through as a quiet NaN.
    """
    x = np.asarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    out = r.view(np.float32).copy()
    out[np.isnan(x)] = np.nan
    return out


def e4m3_decode(codes) -> np.ndarray:
    """Decode FP8 E4M3 (the "fn" variant: bias 7, no infinities) to fp64.

    Bit layout s eeee mmm. e == 0: subnormal m * 2^-9. Otherwise
    (1 + m/8) * 2^(e-7). Code 0x7F / 0xFF (e = 15, m = 7) is NaN; the largest
    finite magnitude is 1.75 * 2^8 = 448.
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (c & 0x7 == 7), np.nan, mag)
    return sign * mag


def e4m3_encode(x) -> np.ndarray:
    """Encode fp32 values as FP8 E4M3 codes, round-to-nearest-even, saturating.

    Magnitudes that round above 448 saturate to 448 (code 0x7E); infinities
    saturate too. Normal range: the quantum for a value in [2^E, 2^(E+1)) is
    2^(E-3) (3 stored mantissa bits); below 2^-6 the quantum is fixed at 2^-9
    (subnormals). A mantissa that rounds up to 2 moves to the next binade.
    NaN maps to 0x7F.
    """
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    out = np.zeros(x.shape, dtype=np.uint8)
    neg = np.signbit(x)
    a = np.abs(x)
    nan = np.isnan(a)
    a = np.where(nan, 0.0, a)
    # binade exponent of |x| (frexp gives a = f * 2^ex with f in [0.5, 1))
    _, ex = np.frexp(a)
    E = ex.astype(np.int64) - 1
    E = np.maximum(E, -6)  # below 2^-6 the grid is the subnormal grid 2^-9
    quantum = np.exp2((E - 3).astype(np.float64))
    q = np.rint(a / quantum)  # numpy rint: round half to even; a/quantum is exact
    val = q * quantum
    val = np.minimum(val, E4M3_MAX)  # satfinite
    # re-derive the fields of the rounded value
    is_sub = val < 2.0 ** -6
    m_sub = np.rint(val / 2.0 ** -9).astype(np.int64)
    _, ex2 = np.frexp(np.where(is_sub, 1.0, val))
    E2 = ex2.astype(np.int64) - 1
    m_norm = np.rint((val / np.exp2(E2.astype(np.float64)) - 1.0) * 8.0).astype(np.int64)
    code = np.where(is_sub, m_sub, ((E2 + 7) << 3) | m_norm)
    code = np.where(nan, 0x7F, code)
    code = code | np.where(neg & ~nan, 0x80, 0)
    out[...] = code.astype(np.uint8)
    return out


# --------------------------------------------------------------------------------------
# Key-value cache addressing ([OSR] "dynamic KV cache"; paged with a block table)
# --------------------------------------------------------------------------------------


def resolve_kv_rows(cache, b, positions, block_table=None, page_size=64):
    """Rows of a per-token cache for logical token positions of sequence ``b``.

    Contiguous layout: cache[b, s]. Paged layout: the logical token s lives in
    physical page block_table[b, s // page_size] at row s % page_size.
    """
    positions = np.asarray(positions, dtype=np.int64)
    if block_table is None:
        return cache[b, positions]
    pages = np.asarray(block_table)[b, positions // page_size]
    return cache[pages, positions % page_size]


# --------------------------------------------------------------------------------------
# Lightning indexer ([TR] §1 Eq. 1)
# --------------------------------------------------------------------------------------


def quantize_indexer_query(q_idx):
    """FP8 E4M3 quantization of each (token, head) indexer query row.

    q_idx: [..., d_I] fp32 holding bf16 values. Returns (codes uint8 [..., d_I],
    s_q fp32 [...]) with s_q = max(amax, 2^-120) / 448 computed in fp32 and
    codes = E4M3(q / s_q), the quotient taken in fp32.
    """
    q = np.asarray(q_idx, dtype=np.float32)
    amax = np.max(np.abs(q), axis=-1)
    s_q = np.maximum(amax, np.float32(QSCALE_FLOOR)).astype(np.float32) / np.float32(E4M3_MAX)
    s_q = s_q.astype(np.float32)
    quot = (q / s_q[..., None]).astype(np.float32)
    return e4m3_encode(quot), s_q


def indexer_scores(q_idx, w, k_idx, k_scale, q_seq, q_pos, *, ld, rows=None,
                   fp8=True, block_table=None, page_size=64):
    """Index scores I_{t,s} for query rows ``rows`` (default: all), fp32 [R, ld].

    fp8=True: q_idx [T, H^I, d_I] (bf16 values as fp32), w [T, H^I] fp32,
    k_idx uint8 E4M3 codes ([B, ctx, d_I] or paged [P, page, d_I]) and k_scale
    fp32 ([B, ctx] or [P, page]). The score is evaluated in fp64 on the decoded
    FP8 values and rounded once to fp32:
        I = s_k[s] * sum_j (w_{t,j} * s_q[t,j]) * max(0, q_hat_{t,j} . k_hat_s)
    fp8=False: q_idx, k_idx are plain fp32 values and no scales apply:
        I = sum_j w_{t,j} * max(0, q_{t,j} . k_s)
    Entries s > pos(t) (and s >= ld) are -inf.
    """
    T = q_idx.shape[0]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    out = np.full((len(rows), ld), -np.inf, dtype=np.float32)
    if fp8:
        codes, s_q = quantize_indexer_query(q_idx)
        q_hat = e4m3_decode(codes)
        head_w = np.asarray(w, np.float64) * s_q.astype(np.float64)
    else:
        q_hat = np.asarray(q_idx, np.float64)
        head_w = np.asarray(w, np.float64)
    # a sequence's visible keys are resolved and decoded once for a run of its rows,
    # up to the last position those rows see (decoding is elementwise: the same values
    # as decoding each row's keys separately); one sequence is held at a time
    n_seq = {}
    for t in rows:
        b = int(q_seq[t])
        n_seq[b] = max(n_seq.get(b, 0), int(q_pos[t]) + 1)
    held_b, held = None, None
    for r, t in enumerate(rows):
        b = int(q_seq[t])
        n = int(q_pos[t]) + 1
        if b != held_b:
            pos_b = np.arange(n_seq[b])
            keys = resolve_kv_rows(k_idx, b, pos_b, block_table, page_size)
            if fp8:  # all 256 codes decoded once, then looked up (the same values)
                held = (e4m3_decode(np.arange(256, dtype=np.uint8))[np.asarray(keys, np.uint8)],
                        resolve_kv_rows(k_scale, b, pos_b, block_table,
                                        page_size).astype(np.float64))
            else:
                held = (np.asarray(keys, np.float64), np.ones(n_seq[b]))
            held_b = b
        k_hat, s_k = held[0][:n], held[1][:n]
        dots = q_hat[t] @ k_hat.T  # [H^I, n]
        score = s_k * (head_w[t] @ np.maximum(dots, 0.0))
        out[r, :n] = score.astype(np.float32)
    return out


# --------------------------------------------------------------------------------------
# Fine-grained token selection ([TR] §1 and §2.1: S_t = Top-k(I_{t,:}))
# --------------------------------------------------------------------------------------


def topk_select(score_row, n_valid, k):
    """The k highest of score_row[0:n_valid]; ties keep the lower position.

    Returns int32 [k]: the selected positions in ascending order, padded with
    -1. When n_valid <= k every visible position is selected.
    """
    n = int(n_valid)
    out = np.full(k, -1, dtype=np.int32)
    if n <= k:
        out[:n] = np.arange(n, dtype=np.int32)
        return out
    vals = np.asarray(score_row[:n], dtype=np.float64)
    pos = np.arange(n)
    order = np.lexsort((pos, -vals))  # primary: score descending; secondary: position
    chosen = np.sort(order[:k])
    out[:] = chosen.astype(np.int32)
    return out


def topk_rows(scores, q_pos, k, rows=None):
    """Apply topk_select to each row r of ``scores`` with n_valid = pos + 1."""
    q_pos = np.asarray(q_pos)
    rows = np.arange(scores.shape[0]) if rows is None else np.asarray(rows)
    return np.stack([topk_select(scores[r], int(q_pos[t]) + 1, k)
                     for r, t in enumerate(rows)]) if len(rows) else np.zeros((0, k), np.int32)


# --------------------------------------------------------------------------------------
# Sparse MLA in MQA mode ([TR] §1 Eq. 2, Fig. 1; Appendix A)
# --------------------------------------------------------------------------------------


def sparse_mla_token(q_t, kv_rows, scale, d_v):
    """Softmax attention of all heads of one query over shared latent rows.

    q_t: [H, D]; kv_rows: [n, D] (key = full D dims, value = first d_v dims).
    z_{h,s} = scale * q_{h} . c_s;  LSE_h = ln sum_s exp(z_{h,s});
    o_h = sum_s exp(z_{h,s} - LSE_h) c_s[:d_v]. All in fp64.
    n == 0 gives o = 0 and LSE = -inf.
    """
    q64 = np.asarray(q_t, np.float64)
    H = q64.shape[0]
    if len(kv_rows) == 0:
        return np.zeros((H, d_v)), np.full(H, -np.inf)
    c = np.asarray(kv_rows, np.float64)
    z = scale * (q64 @ c.T)  # [H, n]
    m = np.max(z, axis=1, keepdims=True)
    lse = m[:, 0] + np.log(np.sum(np.exp(z - m), axis=1))
    p = np.exp(z - lse[:, None])
    return p @ c[:, :d_v], lse


def sparse_mla(q, kv, q_seq, q_pos, idx, scale, d_v, *, rows=None, block_table=None,
               page_size=64):
    """Sparse MLA for query rows ``rows``: each row attends over the entries of
    idx[r] that fall in [0, pos(t)]. Returns (o fp64 [R, H, d_v], lse fp64 [R, H]).

    ``idx`` is indexed by the position of the row within ``rows``.
    """
    T = q.shape[0]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    H = q.shape[1]
    o = np.zeros((len(rows), H, d_v))
    lse = np.zeros((len(rows), H))
    for r, t in enumerate(rows):
        b, pos = int(q_seq[t]), int(q_pos[t])
        sel = [int(s) for s in idx[r] if 0 <= int(s) <= pos]
        kv_rows = resolve_kv_rows(kv, b, sel, block_table, page_size) if sel else []
        o[r], lse[r] = sparse_mla_token(q[t], kv_rows, scale, d_v)
    return o, lse


def dense_causal_mqa(q, kv, q_seq, q_pos, scale, d_v, *, rows=None, block_table=None,
                     page_size=64):
    """Dense causal MQA: every row attends over all positions 0..pos(t)."""
    T = q.shape[0]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    idx = [np.arange(int(q_pos[t]) + 1) for t in rows]
    return sparse_mla(q, kv, q_seq, q_pos, idx, scale, d_v, rows=rows,
                      block_table=block_table, page_size=page_size)


# --------------------------------------------------------------------------------------
# The whole forward: indexer -> top-k -> sparse MLA ([OSR] four-step flow)
# --------------------------------------------------------------------------------------


def dsa_forward(q_idx, w, k_idx, k_scale, q, kv, q_seq, q_pos, *, k, scale, d_v, ld,
                rows=None, fp8=True, block_table=None, page_size=64):
    """Returns dict(scores, idx, o, lse) for the query rows ``rows``."""
    T = q.shape[0]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    scores = indexer_scores(q_idx, w, k_idx, k_scale, q_seq, q_pos, ld=ld, rows=rows,
                            fp8=fp8, block_table=block_table, page_size=page_size)
    idx = topk_rows(scores, q_pos, k, rows=rows)
    o, lse = sparse_mla(q, kv, q_seq, q_pos, idx, scale, d_v, rows=rows,
                        block_table=block_table, page_size=page_size)
    return {"scores": scores, "idx": idx, "o": o, "lse": lse}


# --------------------------------------------------------------------------------------
# Indexer training target and KL loss ([TR] §2.1, both continued-pretraining stages)
# --------------------------------------------------------------------------------------


def indexer_kl_token(q_t, kv_rows, scores_sel, scale):
    """KL loss term of one query token over a set of keys ([TR] §2.1).

    q_t: [H, D]; kv_rows: [n, D] latent rows of the keys in the set; scores_sel:
    [n] indexer scores I_{t,s} of the same keys. Reading of the pages (the loss
    equations are missing images): the main attention of each head over the set
    is a_h(s) = softmax_s(scale * q_h . c_s); the target p(s) sums a_h(s) over the
    heads and L1-normalises over the set, i.e. p(s) = mean_h a_h(s); the model
    distribution is softmax_s(I_{t,s}); the term is KL(p || softmax(I)) =
    sum_s p(s) (ln p(s) - ln softmax(I)(s)), with 0 ln 0 = 0. All in fp64. An
    empty set gives 0.
    """
    n = len(kv_rows)
    if n == 0:
        return 0.0
    q64 = np.asarray(q_t, np.float64)
    c = np.asarray(kv_rows, np.float64)
    z = scale * (q64 @ c.T)                                  # [H, n]
    z = z - np.max(z, axis=1, keepdims=True)
    a = np.exp(z)
    a = a / np.sum(a, axis=1, keepdims=True)                 # per-head softmax over the set
    p = np.sum(a, axis=0)
    p = p / np.sum(p)                                        # head-sum, L1-normalised
    i64 = np.asarray(scores_sel, np.float64)
    log_q = i64 - (np.max(i64) + np.log(np.sum(np.exp(i64 - np.max(i64)))))
    nz = p > 0
    return float(np.sum(p[nz] * (np.log(p[nz]) - log_q[nz])))


def sparse_indexer_kl(q, kv, q_seq, q_pos, idx, scores, scale, *, rows=None, block_table=None,
                      page_size=64):
    """Sparse-stage KL term per query row ([TR] §2.1, sparse training stage): the
    set is S_t, the entries of idx[r] inside [0, pos(t)] (as listed); scores[r]
    is row t's indexer score row. Returns fp64 [R]; ``idx`` and ``scores`` are
    indexed by the position of the row within ``rows``."""
    T = q.shape[0]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    out = np.zeros(len(rows))
    for r, t in enumerate(rows):
        b, pos = int(q_seq[t]), int(q_pos[t])
        sel = [int(s) for s in idx[r] if 0 <= int(s) <= pos]
        kv_rows = resolve_kv_rows(kv, b, sel, block_table, page_size) if sel else []
        out[r] = indexer_kl_token(q[t], kv_rows, np.asarray(scores[r])[sel], scale)
    return out


def dense_indexer_kl(q, kv, q_seq, q_pos, scores, scale, *, rows=None, block_table=None,
                     page_size=64):
    """Dense warm-up KL term per query row ([TR] §2.1, dense warm-up stage): the
    set is every visible key 0..pos(t)."""
    T = q.shape[0]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    idx = [np.arange(int(q_pos[t]) + 1) for t in rows]
    return sparse_indexer_kl(q, kv, q_seq, q_pos, idx, scores, scale, rows=rows,
                             block_table=block_table, page_size=page_size)


# --------------------------------------------------------------------------------------
# MLA in MHA mode and the masked-MHA emulation of DSA ([TR] Appendix A, Fig. 4;
# [TR] §3 "Inference cost": short-sequence prefill runs a masked MHA mode)
# --------------------------------------------------------------------------------------


def mla_up_project(c_rows, w_uk_h, w_uv_h, *, round_kv=True):
    """MHA-mode key and value of one head for latent rows ``c_rows`` [n, d_c + d_r].

    k_{h,s} = [W^UK_h c_s[:d_c] ; c_s[d_c:]] (the rope part is shared by all
    heads: it does not pass through the up-projection) and v_{h,s} =
    W^UV_h c_s[:d_c], with w_uk_h [d_n, d_c] and w_uv_h [d_hv, d_c]. Computed in
    fp64; with ``round_kv`` both are rounded to bf16, the format in which the
    MHA mode holds its decompressed keys and values. Returns (k [n, d_n + d_r],
    v [n, d_hv]) as fp64.
    """
    c = np.asarray(c_rows, np.float64)
    uk = np.asarray(w_uk_h, np.float64)
    uv = np.asarray(w_uv_h, np.float64)
    d_c = uk.shape[1]
    k = np.concatenate([c[:, :d_c] @ uk.T, c[:, d_c:]], axis=1)
    v = c[:, :d_c] @ uv.T
    if round_kv:
        k = bf16_round(k).astype(np.float64)
        v = bf16_round(v).astype(np.float64)
    return k, v


def mha_head_attention(q_th, k, v, scale):
    """Softmax attention of one head's query ``q_th`` [d_qk] over keys k [n, d_qk]
    and values v [n, d_hv]: (o [d_hv], lse) in fp64; n == 0 gives (0, -inf)."""
    if len(k) == 0:
        return np.zeros(v.shape[1]), -np.inf
    z = scale * (k @ np.asarray(q_th, np.float64))
    m = np.max(z)
    lse = m + np.log(np.sum(np.exp(z - m)))
    return np.exp(z - lse) @ v, lse


def masked_mha(q, kv, q_seq, q_pos, idx, scale, w_uk, w_uv, *, rows=None, block_table=None,
               page_size=64, round_kv=True):
    """Masked MHA emulation of DSA for query rows ``rows`` (default: all).

    q: [T, H, d_n + d_r] MHA-mode queries (q^C_{t,h} ; q^R_{t,h}); kv: the latent
    cache; w_uk: [H, d_n, d_c]; w_uv: [H, d_hv, d_c]. Row t of head h attends,
    with softmax scale ``scale``, over the set {s in idx[r] : 0 <= s <= pos(t)}
    (a set: an entry listed twice counts once) or, when ``idx`` is None, over every
    visible key 0..pos(t) (plain causal MHA). Keys and values come from
    mla_up_project. Returns (o fp64 [R, H, d_hv], lse fp64 [R, H]); ``idx`` is
    indexed by the position of the row within ``rows``.

    Heads are independent, so the loop runs head by head over the rows of each
    sequence, up-projecting the sequence's visible latent rows once per head.
    """
    T, H = q.shape[0], q.shape[1]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    d_hv = np.asarray(w_uv).shape[1]
    o = np.zeros((len(rows), H, d_hv))
    lse = np.full((len(rows), H), -np.inf)
    sets = []
    for r, t in enumerate(rows):
        pos = int(q_pos[t])
        if idx is None:
            sets.append(np.arange(pos + 1))
        else:
            sets.append(np.unique([int(s) for s in idx[r] if 0 <= int(s) <= pos]).astype(np.int64))
    for b in sorted({int(q_seq[t]) for t in rows}):
        mine = [r for r, t in enumerate(rows) if int(q_seq[t]) == b]
        n_keys = max(int(q_pos[rows[r]]) for r in mine) + 1
        c = resolve_kv_rows(kv, b, list(range(n_keys)), block_table, page_size)
        for h in range(H):
            k_h, v_h = mla_up_project(c, w_uk[h], w_uv[h], round_kv=round_kv)
            for r in mine:
                s = sets[r]
                o[r, h], lse[r, h] = mha_head_attention(q[rows[r], h], k_h[s], v_h[s], scale)
    return o, lse


def absorb_mha_query(q_mha, w_uk):
    """The MHA-to-MQA conversion of a query ([TR] Appendix A): per head,
    q~_h = [W^UK_h^T q^C_h ; q^R_h], so that q~_h . c_s = q_h . k_{h,s} for the
    unrounded MHA-mode key. q_mha: [T, H, d_n + d_r]; w_uk: [H, d_n, d_c]."""
    q64 = np.asarray(q_mha, np.float64)
    uk = np.asarray(w_uk, np.float64)
    d_n = uk.shape[1]
    nope = np.einsum("thn,hnc->thc", q64[:, :, :d_n], uk)
    return np.concatenate([nope, q64[:, :, d_n:]], axis=2)
