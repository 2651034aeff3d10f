"""dsa_forward_noalloc: the forward for callers that cannot allocate device
memory (a plugin given only its input and output buffers, a runtime whose whole
device memory belongs to its own pool). It runs on the library's fixed scratch
array instead of a caller workspace; its results must match dsa_forward's on
two calls in a row (the second call finds the first call's data still in the
shared array). This file is collected last on purpose.

Every call here passes real device buffers, so that a regression in the size
check can never hand the kernels an address that does not exist."""

import numpy as np
import pytest
import torch

from sparse_attention_05_b200 import synth
from tests.helpers import LSE_ATOL, OUT_ATOL, OUT_RTOL

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 128 << 20  # the size include/dsa.h states for the static array


def _run_both(p, kv_override=None):
    from sparse_attention_05_b200 import dsa
    g = p.to("cuda")
    kv = kv_override(g) if kv_override else dsa.KvLayout.of(g)
    idx_a = torch.empty(p.num_q, 2048, dtype=torch.int32, device="cuda")
    out_a, lse_a, _ = dsa.dsa_forward(g.q_idx, g.w, g.k_idx, g.k_scale, g.q, g.kv, kv,
                                      p.q_per_seq, 2048, p.scale, idx_out=idx_a)
    # no idx_out: the indices live in the static scratch array too
    out_b, lse_b, _ = dsa.dsa_forward_noalloc(g.q_idx, g.w, g.k_idx, g.k_scale, g.q, g.kv, kv,
                                              p.q_per_seq, 2048, p.scale)
    idx_c = torch.empty_like(idx_a)
    out_c, lse_c, _ = dsa.dsa_forward_noalloc(g.q_idx, g.w, g.k_idx, g.k_scale, g.q, g.kv, kv,
                                              p.q_per_seq, 2048, p.scale, idx_out=idx_c)
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == 0
    return (idx_a, out_a, lse_a), (out_b, lse_b), (idx_c, out_c, lse_c)


def _close(o, l, o_ref, l_ref):
    o, o_ref = o.float().cpu().numpy(), o_ref.float().cpu().numpy()
    err = np.abs(o - o_ref)
    assert np.all((err <= OUT_ATOL) | (err <= OUT_RTOL * np.abs(o_ref)))
    l, l_ref = l.cpu().numpy(), l_ref.cpu().numpy()
    assert np.array_equal(np.isfinite(l), np.isfinite(l_ref))
    fin = np.isfinite(l_ref)
    assert np.abs(l[fin] - l_ref[fin]).max(initial=0.0) <= LSE_ATOL


def test_noalloc_matches_workspace_forward_on_two_calls():
    first = synth.decode(batch=4, ctx=5000, q_per_seq=1, seed=60)
    second = synth.paged_decode(batch=3, q_per_seq=2, min_ctx=3000, max_ctx=9000, seed=61)
    for p in (first, second):
        (idx_a, out_a, lse_a), (out_b, lse_b), (idx_c, out_c, lse_c) = _run_both(p)
        assert torch.equal(idx_c, idx_a)
        _close(out_b, lse_b, out_a, lse_a)
        _close(out_c, lse_c, out_a, lse_a)


def _wide_paged(batch):
    """A paged geometry whose block table admits 131072 tokens per sequence (so one
    score row is 512 KiB) while every sequence holds only 130 to 300 tokens."""
    from sparse_attention_05_b200 import dsa
    p = synth.paged_decode(batch=batch, q_per_seq=1, min_ctx=130, max_ctx=300, seed=62)
    max_ctx = 131072

    def kv_of(g):
        bt = torch.zeros(batch, max_ctx // g.page_size, dtype=torch.int32, device="cuda")
        bt[:, : g.block_table.shape[1]] = g.block_table.clamp(min=0)
        return dsa.KvLayout(batch=batch, max_ctx=max_ctx, seqlens=g.seqlens, block_table=bt,
                            page_size=g.page_size, num_pages=g.k_idx.shape[0])
    return p, kv_of


def test_noalloc_geometry_at_the_scratch_limit_runs():
    """256 score rows of 512 KiB fill the 128 MiB array exactly when the indices go to
    idx_out: the call is accepted, twice in a row, and matches dsa_forward."""
    from sparse_attention_05_b200 import dsa
    p, kv_of = _wide_paged(256)
    assert 256 * 131072 * 4 == SCRATCH_BYTES
    g = p.to("cuda")
    kv = kv_of(g)
    idx_a = torch.empty(p.num_q, 2048, dtype=torch.int32, device="cuda")
    out_a, lse_a, _ = dsa.dsa_forward(g.q_idx, g.w, g.k_idx, g.k_scale, g.q, g.kv, kv, 1, 2048,
                                      p.scale, idx_out=idx_a)
    for _ in range(2):
        idx_b = torch.full_like(idx_a, 7)
        out_b, lse_b, _ = dsa.dsa_forward_noalloc(g.q_idx, g.w, g.k_idx, g.k_scale, g.q, g.kv,
                                                  kv, 1, 2048, p.scale, idx_out=idx_b)
        torch.cuda.synchronize()
        assert dsa.dsa_get_device_error() == 0
        assert torch.equal(idx_b, idx_a)
        _close(out_b, lse_b, out_a, lse_a)


def test_noalloc_rejects_geometry_beyond_the_scratch_array():
    """Past the limit the call returns DSA_ERR_WORKSPACE and launches nothing: 256
    sequences whose indices must also live in the array, and 257 sequences with
    idx_out given (one score row more than fits)."""
    from sparse_attention_05_b200 import dsa
    for batch, with_idx_out in ((256, False), (257, True)):
        p, kv_of = _wide_paged(batch)
        g = p.to("cuda")
        kv = kv_of(g)
        out = torch.full((p.num_q, 128, 512), 7.0, dtype=torch.bfloat16, device="cuda")
        lse = torch.full((p.num_q, 128), 7.0, dtype=torch.float32, device="cuda")
        idx = torch.full((p.num_q, 2048), 7, dtype=torch.int32, device="cuda")
        with pytest.raises(dsa.DSAError) as e:
            dsa.dsa_forward_noalloc(g.q_idx, g.w, g.k_idx, g.k_scale, g.q, g.kv, kv, 1, 2048,
                                    p.scale, idx_out=idx if with_idx_out else None, out=out,
                                    lse=lse)
        assert e.value.status == 6  # DSA_ERR_WORKSPACE
        torch.cuda.synchronize()
        assert dsa.dsa_get_device_error() == 0
        assert bool((out == 7.0).all()) and bool((lse == 7.0).all())
        assert bool((idx == 7).all())
