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


@pytest.mark.parametrize("world", [2, 3])
def test_rank_windows_match_the_oracle(world):
    """Every rank's zigzag row windows, computed by dsa_forward on the caches that the
    all-gather assembles from the ranks' token shards (assembled here on the one GPU),
    against the oracle: index sets up to near-ties, outputs and LSE within the
    parity tolerances. The ranks' windows together cover every row exactly once."""
    from oracle import dsa_forward as oracle_forward
    from sparse_attention_05_b200 import dsa
    from tests.helpers import check_attention, check_index_sets, oracle_args
    L, k = 2600, 512
    p = synth.prefill(L=L, seed=111 + world)
    g = p.to("cuda")
    kv = dsa.KvLayout.of(g)
    names = ("k_idx", "k_scale", "kv")
    shards = [{n: getattr(g, n)[0, b:e].clone() for n in names}
              for b, e in (cp.token_shard(L, world, r) for r in range(world))]
    full = {n: torch.cat([s[n] for s in shards])[None] for n in names}
    for n in names:  # the gathered caches are the original ones
        assert torch.equal(full[n], getattr(g, n))
    idx = torch.full((L, k), -7, dtype=torch.int32, device="cuda")
    out = torch.full((L, 128, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((L, 128), float("nan"), dtype=torch.float32, device="cuda")
    covered = np.zeros(L, np.int64)
    edges = []
    for r in range(world):
        for r0, rc in cp.zigzag_windows(L, world, r):
            covered[r0:r0 + rc] += 1
            edges += [r0, r0 + rc - 1]
            dsa.dsa_forward(g.q_idx, g.w, full["k_idx"], full["k_scale"], g.q, full["kv"], kv,
                            L, k, p.scale, idx_out=idx, out=out, lse=lse, rows=(r0, rc))
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == 0
    assert np.all(covered == 1)
    rows = synth.sample_rows(L, 40, seed=112, must=edges + [k - 1, k]).numpy()
    a = oracle_args(p)
    ref = oracle_forward(a["q_idx"], a["w"], a["k_idx"], a["k_scale"], a["q"], a["kv"],
                         a["q_seq"], a["q_pos"], k=k, scale=p.scale, d_v=512, ld=L, rows=rows)
    gi = idx.cpu().numpy()[rows]
    check_index_sets(gi, ref["idx"], ref["scores"], a["q_pos"][rows], k)
    o_ref, l_ref = _oracle_attention_over(a, rows, gi, p.scale)
    check_attention(out.float().cpu().numpy()[rows], lse.cpu().numpy()[rows], o_ref, l_ref)


def _oracle_attention_over(a, rows, idx_rows, scale):
    from oracle import sparse_mla
    return sparse_mla(a["q"], a["kv"], a["q_seq"], a["q_pos"], idx_rows, scale, 512, rows=rows)
