"""Context-parallel prefill through the library on one GPU (one rank: the
all-gather is a copy and the zigzag windows cover every row): the gathered caches
and dsa_forward over the rank's row windows must reproduce dsa_forward over all
rows bit for bit. The multi-rank collective itself is covered on the host with gloo
ranks (tests/test_cp.py); this pool gives one GPU per run."""

import numpy as np
import pytest
import torch

from sparse_attention_05_b200 import cp, synth

pytestmark = pytest.mark.gpu


def test_one_rank_windows_reproduce_the_single_gpu_forward():
    from sparse_attention_05_b200 import dsa
    L, k = 1100, 512
    p = synth.prefill(L=L, seed=110).to("cuda")
    kv = dsa.KvLayout.of(p)
    out0, lse0, _ = dsa.dsa_forward(p.q_idx, p.w, p.k_idx, p.k_scale, p.q, p.kv, kv,
                                    p.q_per_seq, k, p.scale)
    b, e = cp.token_shard(L, 1, 0)
    shards = {n: getattr(p, n)[0, b:e].clone() for n in ("k_idx", "k_scale", "kv")}
    out = torch.empty_like(out0)
    lse = torch.empty_like(lse0)

    def compute(c, wins):
        for r0, rc in wins:
            dsa.dsa_forward(p.q_idx, p.w, c["k_idx"][None], c["k_scale"][None], p.q,
                            c["kv"][None], kv, p.q_per_seq, k, p.scale, out=out, lse=lse,
                            rows=(r0, rc))
        return None

    wins, _ = cp.cp_prefill(L, 1, 0, shards, compute)
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == 0
    assert wins == [(0, L)]
    assert torch.equal(out, out0) and torch.equal(lse, lse0)
