"""dsa_forward_noalloc: the forward for callers that cannot allocate device
memory (a plugin given only its input and output buffers, a runtime whose whole
device memory belongs to its own pool). It runs on the library's fixed scratch
array instead of a caller workspace; its results must match dsa_forward's on
two calls in a row (the second call finds the first call's data still in the
shared array). This file is collected last on purpose."""

import ctypes

import numpy as np
import pytest
import torch

from sparse_attention_05_b200 import synth
from tests.helpers import LSE_ATOL, OUT_ATOL, OUT_RTOL

pytestmark = pytest.mark.gpu


def _run_both(p):
    from sparse_attention_05_b200 import dsa
    g = p.to("cuda")
    kv = dsa.KvLayout.of(g)
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


def test_noalloc_rejects_geometry_beyond_the_scratch_array():
    from sparse_attention_05_b200 import dsa
    kv = dsa.KvDescC()
    kv.layout, kv.batch, kv.max_ctx = 0, 1, 20000
    q = dsa.QDescC(20000, 20000, 0, 0)  # 20000 x 2048 int32 indices = 164 MB > 128 MiB
    fake = ctypes.c_void_p(0x1000)      # never dereferenced: the size check comes first
    st = dsa.lib().dsa_forward_noalloc(fake, fake, fake, fake, fake, fake, ctypes.byref(kv),
                                       ctypes.byref(q), 2048, 0.04, None, fake, fake, None)
    assert st == 6  # DSA_ERR_WORKSPACE
