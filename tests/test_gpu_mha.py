"""GPU parity of MLA's MHA mode ([TR] Appendix A; the masked-MHA emulation of DSA
for short prefill, [TR] §3): the up-projection, the selection mask and the masked
flash attention, each through the C ABI, against the oracle (fp64, keys/values
rounded to bf16 as the MHA mode holds them). Causal and selected masks, ragged
tails, several sequences, row windows, paged caches, large logits (the lazy
rescale path) and sampled rows of the 8K prefill through dsa_mha_prefill."""

import numpy as np
import pytest
import torch

from oracle import indexer_scores, masked_mha, mla_up_project, resolve_kv_rows, topk_rows
from sparse_attention_05_b200 import synth
from tests.helpers import check_attention, check_index_sets, mha_lse_tolerance, oracle_args

pytestmark = pytest.mark.gpu


def _dsa():
    from sparse_attention_05_b200 import dsa
    return dsa


def _np(x):
    return x.detach().cpu().float().numpy()


def _mha_args(p, m):
    a = oracle_args(p)
    a.update(q_mha=_np(m.q_mha), w_uk=_np(m.w_uk), w_uv=_np(m.w_uv))
    return a


def _oracle(p, m, idx_rows, rows, scale=None):
    a = _mha_args(p, m)
    return masked_mha(a["q_mha"], a["kv"], a["q_seq"], a["q_pos"], idx_rows,
                      p.scale if scale is None else scale, a["w_uk"], a["w_uv"], rows=rows,
                      block_table=a["block_table"], page_size=p.page_size)


def _check(p, m, o_gpu, lse_gpu, idx_rows, rows, scale=None, bulk=0.99):
    """Oracle parity of the given rows: outputs within the bf16 attention
    tolerance, each LSE within its derived bound (bf16 rounding of the
    decompressed keys, see mha_lse_tolerance) and 99% of them within 1e-4."""
    scale = p.scale if scale is None else scale
    o_r, l_r = _oracle(p, m, idx_rows, rows, scale)
    a = _mha_args(p, m)
    pos = a["q_pos"]
    if idx_rows is None:
        sets = [np.arange(int(pos[t]) + 1) for t in rows]
    else:
        sets = [np.unique([s for s in idx_rows[r] if 0 <= s <= pos[t]]) for r, t in enumerate(rows)]
    tol = mha_lse_tolerance(a["q_mha"], a["kv"], a["q_seq"], pos, sets, a["w_uk"], scale, rows,
                            block_table=a["block_table"], page_size=p.page_size)
    return check_attention(o_gpu, lse_gpu, o_r, l_r, lse_tol=tol, lse_bulk=bulk)


def _gpu_mha(p, m, idx=None, k=2048, scale=None, rows=None):
    """Up-projection, (selection mask), masked MHA through the C ABI."""
    dsa = _dsa()
    g, gm = p.to("cuda"), m.to("cuda")
    kv = dsa.KvLayout.of(g)
    kn, kr, v = dsa.dsa_mla_up_project(g.kv, gm.w_uk, gm.w_uv, kv)
    mask = None
    if idx is not None:
        idx_t = torch.from_numpy(np.ascontiguousarray(idx, np.int32)).cuda()
        mask = dsa.dsa_selection_mask(idx_t, kv, p.q_per_seq, rows=rows)
    out, lse = dsa.dsa_masked_mha(gm.q_mha, kn, kr, v, kv, p.q_per_seq,
                                  p.scale if scale is None else scale, mask=mask, k=k,
                                  rows=rows)
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == 0
    return _np(out), lse.cpu().numpy(), (kn, kr, v)


def _random_idx(p, k, seed):
    rng = np.random.default_rng(seed)
    pos = p.q_pos().numpy()
    out = np.full((p.num_q, k), -1, np.int32)
    for t in range(p.num_q):
        n = min(k, int(pos[t]) + 1)
        out[t, :n] = np.sort(rng.choice(int(pos[t]) + 1, n, replace=False))
    return out


# ---- up-projection -----------------------------------------------------------------


def _check_up_projection(p, m, kn, kr, v):
    a = _mha_args(p, m)
    kn, kr, v = _np(kn), _np(kr), _np(v)
    seqlens = p.seqlens.cpu().numpy()
    for b in range(p.batch):
        n = int(seqlens[b])
        c = resolve_kv_rows(a["kv"], b, list(range(n)), a["block_table"], p.page_size)
        for h in (0, 1, 63, 127):
            k0, v0 = mla_up_project(c, a["w_uk"][h], a["w_uv"][h], round_kv=False)
            # bf16 of an fp32-accumulated product: at most one rounding (2^-8
            # relative) plus the fp32 sum over 512 terms
            for got, ref in ((kn[b, h, :n], k0[:, :128]), (v[b, h, :n], v0)):
                tol = 2.0 ** -8 * np.abs(ref) + 1e-5 * np.max(np.abs(ref))
                assert np.all(np.abs(got - ref) <= tol)
            pad = (n + 127) // 128 * 128
            assert not kn[b, h, n:pad].any() and not v[b, h, n:pad].any()
        assert np.array_equal(kr[b, :n], c[:, 512:].astype(np.float32))  # bf16 copied exactly
        assert not kr[b, n:(n + 127) // 128 * 128].any()


def test_up_projection_contiguous_ragged():
    p = synth.prefill(L=300, seed=80)
    m = synth.mha_inputs(p, 81)
    _, _, (kn, kr, v) = _gpu_mha(p, m)
    _check_up_projection(p, m, kn, kr, v)


def test_up_projection_paged_varlen():
    p = synth.paged_decode(batch=3, q_per_seq=2, min_ctx=200, max_ctx=520, page_size=64, seed=82)
    m = synth.mha_inputs(p, 83)
    dsa = _dsa()
    g, gm = p.to("cuda"), m.to("cuda")
    kn, kr, v = dsa.dsa_mla_up_project(g.kv, gm.w_uk, gm.w_uv, dsa.KvLayout.of(g))
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == 0
    _check_up_projection(p, m, kn, kr, v)


# ---- selection mask ------------------------------------------------------------------


def test_selection_mask_bits_exact():
    p = synth.prefill(L=600, seed=84)
    k = 100
    idx = _random_idx(p, k, 85)
    idx[300, :5] = idx[300, 5]          # duplicates
    idx[301, 0] = 10 ** 6               # out of range
    idx[302, 1] = 590                   # beyond the row's position
    dsa = _dsa()
    g = p.to("cuda")
    kv = dsa.KvLayout.of(g)
    mask = dsa.dsa_selection_mask(torch.from_numpy(idx).cuda(), kv, p.q_per_seq)
    torch.cuda.synchronize()
    got = mask.cpu().numpy().view(np.uint32)
    pos = p.q_pos().numpy()
    for t in range(p.num_q):
        want = np.zeros(got.shape[1], np.uint32)
        if pos[t] + 1 > k:
            for s in idx[t]:
                if 0 <= s <= pos[t]:
                    want[s >> 5] |= np.uint32(1) << np.uint32(s & 31)
        assert np.array_equal(got[t], want), f"row {t}"


# ---- masked MHA ------------------------------------------------------------------------


def test_causal_prefill_all_rows_ragged():
    p = synth.prefill(L=300, seed=86)
    m = synth.mha_inputs(p, 87)
    o_g, l_g, _ = _gpu_mha(p, m)
    _check(p, m, o_g, l_g, None, np.arange(p.num_q))


def test_selected_rows_random_sets():
    p = synth.prefill(L=700, seed=88)
    m = synth.mha_inputs(p, 89)
    k = 256
    idx = _random_idx(p, k, 90)
    o_g, l_g, _ = _gpu_mha(p, m, idx=idx, k=k)
    rows = synth.sample_rows(p.num_q, 40, seed=91, must=(0, 127, 255, 256, 257, 699)).numpy()
    _check(p, m, o_g[rows], l_g[rows], idx[rows], rows)


def test_large_logits_exercise_the_lazy_rescale():
    p = synth.prefill(L=640, seed=92)
    m = synth.mha_inputs(p, 93)
    idx = _random_idx(p, 128, 94)
    o_g, l_g, _ = _gpu_mha(p, m, idx=idx, k=128, scale=1.0)
    rows = synth.sample_rows(p.num_q, 32, seed=95, must=(0, 639)).numpy()
    # at scale 1 one key dominates each softmax, so a bf16 step of one of its
    # elements shows in full in the LSE: a looser bulk criterion (95%)
    _check(p, m, o_g[rows], l_g[rows], idx[rows], rows, scale=1.0, bulk=0.95)


def test_several_sequences_and_a_row_window():
    """Rows are the last 200 tokens of two 700-token sequences; only window rows
    [50, 150) are computed, the others stay untouched."""
    p = synth.decode(batch=2, ctx=700, q_per_seq=200, seed=96)
    m = synth.mha_inputs(p, 97)
    idx = _random_idx(p, 300, 98)
    dsa = _dsa()
    g, gm = p.to("cuda"), m.to("cuda")
    kv = dsa.KvLayout.of(g)
    kn, kr, v = dsa.dsa_mla_up_project(g.kv, gm.w_uk, gm.w_uv, kv)
    idx_t = torch.from_numpy(idx).cuda()
    mask = dsa.dsa_selection_mask(idx_t, kv, p.q_per_seq, rows=(50, 100))
    out = torch.full((p.num_q, 128, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((p.num_q, 128), 7.0, device="cuda")
    dsa.dsa_masked_mha(gm.q_mha, kn, kr, v, kv, p.q_per_seq, p.scale, mask=mask, k=300,
                       out=out, lse=lse, rows=(50, 100))
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == 0
    win = np.array([b * 200 + i for b in range(2) for i in range(50, 150)])
    rows = win[::7]
    _check(p, m, _np(out)[rows], lse.cpu().numpy()[rows], idx[rows], rows)
    others = np.setdiff1d(np.arange(p.num_q), win)
    assert np.all(_np(out)[others] == 7.0) and np.all(lse.cpu().numpy()[others] == 7.0)


def test_paged_varlen_causal():
    p = synth.paged_decode(batch=3, q_per_seq=150, min_ctx=300, max_ctx=520, page_size=64,
                           seed=99)
    m = synth.mha_inputs(p, 100)
    o_g, l_g, _ = _gpu_mha(p, m)
    rows = synth.sample_rows(p.num_q, 30, seed=101, must=(0, 149, 150, 449)).numpy()
    _check(p, m, o_g[rows], l_g[rows], None, rows)


# ---- the composed call ---------------------------------------------------------------


def _prefill_end_to_end(L, k, n_rows, seed, must):
    dsa = _dsa()
    p = synth.prefill(L=L, seed=seed)
    m = synth.mha_inputs(p, seed + 1)
    g, gm = p.to("cuda"), m.to("cuda")
    idx = torch.empty(p.num_q, k, dtype=torch.int32, device="cuda")
    out, lse, _ = dsa.dsa_mha_prefill(g.q_idx, g.w, g.k_idx, g.k_scale, gm.q_mha, g.kv, gm.w_uk,
                                      gm.w_uv, dsa.KvLayout.of(g), p.q_per_seq, k, p.scale,
                                      idx_out=idx)
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == 0
    rows = synth.sample_rows(p.num_q, n_rows, seed=seed + 2, must=must).numpy()
    a = oracle_args(p)
    ld = (L + 127) // 128 * 128
    sc = indexer_scores(a["q_idx"], a["w"], a["k_idx"], a["k_scale"], a["q_seq"], a["q_pos"],
                        ld=ld, rows=rows)
    idx_g = idx.cpu().numpy()[rows]
    check_index_sets(idx_g, topk_rows(sc, a["q_pos"], k, rows=rows), sc, a["q_pos"][rows], k)
    # attention parity on the GPU's own (checked) selection
    _check(p, m, _np(out)[rows], lse.cpu().numpy()[rows], idx_g, rows)


def test_mha_prefill_composed_ragged():
    _prefill_end_to_end(L=1100, k=512, n_rows=24, seed=102, must=(0, 511, 512, 1099))


def test_mha_prefill_full_size_sampled_rows():
    """The 8K prefill (k = 2048), sampled rows through the composed call."""
    _prefill_end_to_end(L=8192, k=2048, n_rows=6, seed=2, must=(0, 2047, 2048, 8191))


def test_host_argument_checks():
    dsa = _dsa()
    p = synth.prefill(L=256, seed=103).to("cuda")
    m = synth.mha_inputs(p, 104).to("cuda")
    kv = dsa.KvLayout.of(p)
    kn = torch.empty(1, 128, 128, 128, dtype=torch.bfloat16, device="cuda")  # ctx_pad too small
    kr = torch.empty(1, 256, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(dsa.DSAError) as e:
        dsa.dsa_mla_up_project(p.kv, m.w_uk, m.w_uv, kv, k_nope=kn, k_rope=kr, v=kn)
    assert e.value.status == 1
    idx = torch.zeros(256, 16, dtype=torch.int32, device="cuda")
    bad = torch.zeros(256, 6, dtype=torch.int32, device="cuda")  # mask_ld not a multiple of 4
    with pytest.raises(dsa.DSAError) as e:
        dsa.dsa_selection_mask(idx, kv, 256, mask=bad)
    assert e.value.status == 1


# ---- degenerate cases ------------------------------------------------------------------


def test_one_token_sequences_attend_to_themselves():
    """Sequences of one token: the row's only key is itself, so o = v and LSE = z
    (the oracle's closed form for one key)."""
    p = synth.decode(batch=3, ctx=1, q_per_seq=1, seed=105)
    m = synth.mha_inputs(p, 106)
    o_g, l_g, _ = _gpu_mha(p, m)
    _check(p, m, o_g, l_g, None, np.arange(p.num_q))


def test_k_one_every_row_selects_a_single_key():
    p = synth.prefill(L=300, seed=107)
    m = synth.mha_inputs(p, 108)
    idx = _random_idx(p, 1, 109)
    o_g, l_g, _ = _gpu_mha(p, m, idx=idx, k=1)
    rows = np.arange(0, 300, 7)
    _check(p, m, o_g[rows], l_g[rows], idx[rows], rows)


def test_paged_cache_with_selection_masks():
    p = synth.paged_decode(batch=2, q_per_seq=160, min_ctx=400, max_ctx=640, page_size=64,
                           seed=111)
    m = synth.mha_inputs(p, 112)
    idx = _random_idx(p, 200, 113)
    o_g, l_g, _ = _gpu_mha(p, m, idx=idx, k=200)
    rows = synth.sample_rows(p.num_q, 30, seed=114, must=(0, 159, 160, 319)).numpy()
    _check(p, m, o_g[rows], l_g[rows], idx[rows], rows)
