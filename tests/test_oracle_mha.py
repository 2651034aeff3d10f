"""Pins of the oracle's MLA MHA mode and its masked form ([TR] Appendix A, Fig. 4;
[TR] §3 "Inference cost"): the MHA/MQA conversion against the separately pinned
MQA-mode oracle, torch's scaled_dot_product_attention in fp64 (causal and with an
explicit boolean mask), a closed form for one key, and set semantics of the mask."""

import numpy as np
import torch

from oracle import (absorb_mha_query, bf16_round, masked_mha, mha_head_attention,
                    mla_up_project, sparse_mla)


def _problem(seed, T=12, H=3, d_c=16, d_r=4, d_n=6, d_hv=5):
    """One sequence whose query rows are its positions 0..T-1 (prefill)."""
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(T, H, d_n + d_r))
    kv = rng.normal(size=(1, T, d_c + d_r)) * 0.5
    w_uk = rng.normal(size=(H, d_n, d_c)) / np.sqrt(d_c)
    w_uv = rng.normal(size=(H, d_hv, d_c)) / np.sqrt(d_c)
    q_seq = np.zeros(T, np.int64)
    q_pos = np.arange(T)
    return q, kv, w_uk, w_uv, q_seq, q_pos, rng


def _keys_values(kv, w_uk, w_uv):
    """Decompressed keys/values per head by plain einsum (no rounding)."""
    c = kv[0]
    d_c = w_uk.shape[2]
    kn = np.einsum("hnc,sc->hsn", w_uk, c[:, :d_c])
    kr = np.broadcast_to(c[None, :, d_c:], (w_uk.shape[0],) + c[:, d_c:].shape)
    return np.concatenate([kn, kr], axis=2), np.einsum("hvc,sc->hsv", w_uv, c[:, :d_c])


def test_conversion_to_mqa_mode_is_exact():
    """Appendix A's conversion: attention in MHA mode equals MQA-mode attention of
    the absorbed query over the latent rows, followed by W^UV on the output."""
    q, kv, w_uk, w_uv, q_seq, q_pos, rng = _problem(1)
    T, H = q.shape[:2]
    idx = [np.sort(rng.choice(int(p) + 1, min(int(p) + 1, 5), replace=False)) for p in q_pos]
    o, lse = masked_mha(q, kv, q_seq, q_pos, idx, 0.37, w_uk, w_uv, round_kv=False)
    qa = absorb_mha_query(q, w_uk)
    o_lat, lse_mqa = sparse_mla(qa, kv, q_seq, q_pos, idx, 0.37, w_uk.shape[2])
    o_mqa = np.einsum("hvc,thc->thv", w_uv, o_lat)
    assert np.allclose(lse, lse_mqa, rtol=0, atol=1e-12)
    assert np.allclose(o, o_mqa, rtol=1e-11, atol=1e-12)


def test_causal_matches_torch_sdpa():
    q, kv, w_uk, w_uv, q_seq, q_pos, _ = _problem(2)
    o, lse = masked_mha(q, kv, q_seq, q_pos, None, 0.41, w_uk, w_uv, round_kv=False)
    k, v = _keys_values(kv, w_uk, w_uv)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q.transpose(1, 0, 2).copy()), torch.from_numpy(k.copy()),
        torch.from_numpy(v.copy()), is_causal=True, scale=0.41)
    assert np.allclose(o, ref.numpy().transpose(1, 0, 2), rtol=1e-11, atol=1e-12)
    # LSE: logsumexp of the causal logits, by torch
    z = 0.41 * torch.einsum("thd,hsd->hts", torch.from_numpy(q), torch.from_numpy(k.copy()))
    z = z.masked_fill(torch.triu(torch.ones(12, 12, dtype=torch.bool), 1), float("-inf"))
    assert np.allclose(lse, torch.logsumexp(z, dim=2).numpy().T, rtol=0, atol=1e-12)


def test_selection_mask_matches_torch_sdpa_with_boolean_mask():
    q, kv, w_uk, w_uv, q_seq, q_pos, rng = _problem(3, T=20)
    T = q.shape[0]
    mask = np.zeros((T, T), bool)
    idx = []
    for t in range(T):
        sel = rng.choice(t + 1, min(t + 1, 6), replace=False)
        mask[t, sel] = True
        idx.append(sel)
    o, _ = masked_mha(q, kv, q_seq, q_pos, idx, 0.3, w_uk, w_uv, round_kv=False)
    k, v = _keys_values(kv, w_uk, w_uv)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q.transpose(1, 0, 2).copy()), torch.from_numpy(k.copy()),
        torch.from_numpy(v.copy()), attn_mask=torch.from_numpy(mask), scale=0.3)
    assert np.allclose(o, ref.numpy().transpose(1, 0, 2), rtol=1e-11, atol=1e-12)


def test_single_key_closed_form():
    rng = np.random.default_rng(4)
    k = rng.normal(size=(1, 7))
    v = rng.normal(size=(1, 3))
    q = rng.normal(size=7)
    o, lse = mha_head_attention(q, k, v, 0.5)
    assert np.array_equal(o, v[0])
    assert abs(lse - 0.5 * float(k[0] @ q)) < 1e-15


def test_mask_is_a_set_and_ignores_invisible_entries():
    q, kv, w_uk, w_uv, q_seq, q_pos, rng = _problem(5)
    T = q.shape[0]
    idx = [np.sort(rng.choice(int(p) + 1, min(int(p) + 1, 4), replace=False)) for p in q_pos]
    base = masked_mha(q, kv, q_seq, q_pos, idx, 0.3, w_uk, w_uv)
    noisy = [np.concatenate([r, r[:2], [-1, -1, int(p) + 1, 10 ** 6]])
             for r, p in zip(idx, q_pos)]
    again = masked_mha(q, kv, q_seq, q_pos, noisy, 0.3, w_uk, w_uv)
    assert np.array_equal(base[0], again[0]) and np.array_equal(base[1], again[1])
    # selecting every visible key is plain causal attention
    full = [np.arange(int(p) + 1) for p in q_pos]
    a = masked_mha(q, kv, q_seq, q_pos, full, 0.3, w_uk, w_uv)
    b = masked_mha(q, kv, q_seq, q_pos, None, 0.3, w_uk, w_uv)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_up_projection_rounds_to_bf16_and_shares_rope():
    rng = np.random.default_rng(6)
    c = rng.normal(size=(9, 20))
    uk = rng.normal(size=(6, 16))
    uv = rng.normal(size=(5, 16))
    k, v = mla_up_project(c, uk, uv)
    k0, v0 = mla_up_project(c, uk, uv, round_kv=False)
    assert np.array_equal(k, bf16_round(k0)) and np.array_equal(v, bf16_round(v0))
    assert np.array_equal(k0[:, 6:], c[:, 16:])              # rope dims pass through
    assert np.allclose(k0[:, :6], c[:, :16] @ uk.T, rtol=1e-14)
    assert np.max(np.abs(k - k0) / np.maximum(np.abs(k0), 1e-30)) <= 2.0 ** -8  # bf16: 8 significant bits


def test_rows_of_several_sequences_and_paged_cache():
    """Rows of two sequences through a block table equal the contiguous result."""
    rng = np.random.default_rng(7)
    H, d_c, d_r, d_n, d_hv, L = 2, 8, 4, 3, 3, 10
    kv = rng.normal(size=(2, L, d_c + d_r))
    q = rng.normal(size=(4, H, d_n + d_r))
    w_uk = rng.normal(size=(H, d_n, d_c))
    w_uv = rng.normal(size=(H, d_hv, d_c))
    q_seq = np.array([0, 0, 1, 1])
    q_pos = np.array([8, 9, 8, 9])
    ref = masked_mha(q, kv, q_seq, q_pos, None, 0.2, w_uk, w_uv)
    # pages of 5 tokens, physical order shuffled
    pages = kv.reshape(4, 5, d_c + d_r)
    perm = np.array([2, 0, 3, 1])
    phys = np.empty_like(pages)
    phys[perm] = pages
    bt = perm.reshape(2, 2)
    got = masked_mha(q, phys, q_seq, q_pos, None, 0.2, w_uk, w_uv, block_table=bt, page_size=5)
    assert np.array_equal(ref[0], got[0]) and np.array_equal(ref[1], got[1])
