"""Row geometry of the seeded inputs: every query row's sequence and position, for
uniform and ragged batches (the geometry the oracle receives in the parity tests)."""

import torch

from sparse_attention_05_b200 import synth


def test_uniform_rows_are_each_sequence_last_tokens():
    p = synth.decode(batch=3, ctx=100, q_per_seq=2, seed=1)
    assert p.q_seq().tolist() == [0, 0, 1, 1, 2, 2]
    assert p.q_pos().tolist() == [98, 99] * 3


def test_ragged_rows_follow_q_start():
    p = synth.ragged([70, 130, 65, 300], [70, 0, 3, 1], page_size=64, seed=5)
    assert p.q_start.tolist() == [0, 70, 70, 73, 74]
    assert p.num_q == 74 and p.q_per_seq == 70
    seq, pos = p.q_seq().tolist(), p.q_pos().tolist()
    assert seq == [0] * 70 + [2] * 3 + [3]
    assert pos == list(range(70)) + [62, 63, 64] + [299]
    # the block table covers exactly each sequence's pages with distinct physical pages
    used = [int(x) for b, n in enumerate([2, 3, 2, 5]) for x in p.block_table[b, :n]]
    assert sorted(used) == list(range(12))
    assert bool((p.block_table[0, 2:] == -1).all())
    assert p.q_idx.shape[0] == 74 and p.q.shape[0] == 74 and p.w.shape[0] == 74


def test_ragged_problem_moves_its_offsets_with_it():
    p = synth.ragged([100, 200], [10, 20], seed=6)
    assert p.to("cpu").q_start is not None
    assert torch.equal(p.to("cpu").q_start, p.q_start)
