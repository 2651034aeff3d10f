"""Context-parallel prefill ("DeepSeek-V3.2开源技术报告", DSA principle section: context
parallelism across GPUs): the zigzag row partition and the token shards, and, with
two gloo ranks on the host, the all-gather of the per-token caches followed by the
forward on each rank's rows. The compute there is the oracle (the GPU kernels need
a GPU); each rank's rows must equal the single-process oracle on the same rows bit
for bit, and the gathered caches must equal the whole caches."""

import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_attention_05_b200 import cp, synth


@pytest.mark.parametrize("L", [300, 1100, 8192, 131072])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_zigzag_rows_cover_once_and_balance(L, world):
    wins = [cp.zigzag_windows(L, world, r) for r in range(world)]
    rows = np.concatenate([np.arange(b, b + c) for w in wins for b, c in w]) if L else []
    assert np.array_equal(np.sort(rows), np.arange(L))           # every row exactly once
    for w in wins:
        assert all(b % cp.CHUNK_ALIGN == 0 for b, _ in w)          # tile-aligned starts
    pairs = np.array([cp.causal_pairs(w) for w in wins])
    assert pairs.sum() == L * (L + 1) // 2
    # balance: within one 128-row chunk's pairs of the mean, beyond the tiny cases
    if L >= 8192:
        assert pairs.max() - pairs.mean() <= 2 * cp.CHUNK_ALIGN * L


@pytest.mark.parametrize("L,world", [(300, 2), (8192, 3), (131072, 8)])
def test_token_shards_are_contiguous_and_cover(L, world):
    sh = [cp.token_shard(L, world, r) for r in range(world)]
    assert sh[0][0] == 0 and sh[-1][1] == L
    for (b0, e0), (b1, _) in zip(sh, sh[1:]):
        assert e0 == b1 and b0 % cp.CHUNK_ALIGN == 0


def _rank(rank, world, port, results):
    from oracle import dsa_forward
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    p = synth.tiny(L=256, seed=0)
    L, D = 256, p.dims
    b, e = cp.token_shard(L, world, rank)
    shards = {"k_idx": p.k_idx[0, b:e].clone(), "kv": p.kv[0, b:e].clone()}
    q_seq = np.zeros(L, np.int64)
    q_pos = np.arange(L)

    def compute(caches, wins):
        rows = np.concatenate([np.arange(r0, r0 + rc) for r0, rc in wins])
        got = dsa_forward(p.q_idx.numpy(), p.w.numpy(), caches["k_idx"].numpy()[None],
                          None, p.q.numpy(), caches["kv"].numpy()[None], q_seq, q_pos,
                          k=D.topk, scale=p.scale, d_v=D.d_v, ld=L, rows=rows, fp8=False)
        return rows, got

    wins, (rows, got) = cp.cp_prefill(L, world, rank, shards, compute)
    # the gathered caches are the whole caches
    full = {n: cp.allgather_cache(t, L, world) for n, t in shards.items()}
    same = torch.equal(full["k_idx"], p.k_idx[0]) and torch.equal(full["kv"], p.kv[0])
    results[rank] = (rows, got["idx"], got["o"], got["lse"], same)
    dist.destroy_process_group()


def test_gloo_two_ranks_gather_then_forward_equals_single_process():
    from oracle import dsa_forward
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, results)) for r in range(2)]
    for pr in procs:
        pr.start()
    for pr in procs:
        pr.join(300)
        assert pr.exitcode == 0
    p = synth.tiny(L=256, seed=0)
    D = p.dims
    allrows = []
    for r in range(2):
        rows, idx, o, lse, same = results[r]
        assert same
        ref = dsa_forward(p.q_idx.numpy(), p.w.numpy(), p.k_idx.numpy(), None, p.q.numpy(),
                          p.kv.numpy(), np.zeros(256, np.int64), np.arange(256), k=D.topk,
                          scale=p.scale, d_v=D.d_v, ld=256, rows=rows, fp8=False)
        assert np.array_equal(idx, ref["idx"])
        assert np.array_equal(o, ref["o"]) and np.array_equal(lse, ref["lse"])
        allrows.append(rows)
    assert np.array_equal(np.sort(np.concatenate(allrows)), np.arange(256))
