"""CPU tests of bench.py's host logic: the algorithmic work per kernel, the
roofline classification, the whole-job throughput and, with two gloo ranks,
the max-over-ranks timing reduction the multi-GPU run uses."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from sparse_attention_05_b200 import synth


def test_algorithmic_work_counts():
    p = synth.decode(batch=2, ctx=3000, q_per_seq=2, seed=1)
    w = bench.algorithmic_work(p, k=2048)
    # rows at positions 2998 and 2999 of each sequence: 2999 + 3000 visible keys per sequence
    n_vis = 2 * (2999 + 3000)
    n_sel = 4 * 2048
    assert w["indexer"]["flop"] == 16384 * n_vis
    assert w["indexer"]["bytes"] == 132 * 6000 + 4 * (64 * 128 * 2 + 64 * 4) + 4 * n_vis
    assert w["topk"]["bytes"] == 4 * n_vis + 4 * 4 * 2048
    assert w["sparse_mla"]["flop"] == 278528 * n_sel
    assert w["sparse_mla"]["bytes"] == 4 * (128 * 576 * 2 + 128 * 512 * 2 + 512 + 8192) + 1152 * n_sel


def test_roofline_classification():
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1400.0,
             "source": "measured"}
    work = {"a": {"bytes": 6e9, "flop": 1e12, "flop_dtype": "bf16"},      # 1 ms vs 0.67 ms
            "b": {"bytes": 1e9, "flop": 3e13, "flop_dtype": "fp8"}}       # 0.17 ms vs 10 ms
    ra = bench.roofline("a", work, 2e-3, peaks, long_step=False)
    assert ra["bound"] == "hbm" and abs(ra["frac"] - 0.5) < 1e-12 and ra["unit"] == "GB/s"
    rb = bench.roofline("b", work, 20e-3, peaks, long_step=True)
    assert rb["bound"] == "tensor" and rb["peak"] == 2 * 1400.0
    assert abs(rb["achieved"] - 1500.0) < 1e-9


def test_job_throughput():
    assert bench.job_throughput(4, 256, 10, 2.0) == 4 * 256 * 10 / 2.0


def test_step_roofline_sums_every_kernel():
    peaks = {"hbm_gbs": 5000.0, "bf16_tflops": 1000.0, "bf16_tflops_sustained": 800.0}
    work = {"a": {"bytes": 5e9, "flop": 0, "flop_dtype": None},          # 1 ms of HBM
            "b": {"bytes": 5e9, "flop": 2e12, "flop_dtype": "bf16"},     # 1 ms, 2 ms of BF16
            "c": {"bytes": 0, "flop": 4e12, "flop_dtype": "fp8"}}        # 2 ms of FP8
    r = bench.step_roofline(work, ("a", "b", "c"), 8e-3, peaks, long_step=False)
    assert abs(r["hbm_ms"] - 2.0) < 1e-9 and abs(r["tensor_ms"] - 4.0) < 1e-9
    assert r["bound"] == "tensor" and abs(r["frac"] - 0.5) < 1e-12
    r = bench.step_roofline(work, ("a", "b"), 4e-3, peaks, long_step=True)
    assert abs(r["tensor_ms"] - 2.5) < 1e-9 and r["bound"] == "tensor"


def test_end_to_end_staging_layout():
    """The end-to-end run packs a step's inputs (and its outputs) into one buffer:
    every tensor sits at a 256-byte boundary, views round-trip the data, and the
    packed size is what one copy moves."""
    t = {"q": torch.randn(3, 5).to(torch.bfloat16), "seqlens": torch.arange(7, dtype=torch.int32),
         "w": torch.rand(2, 3), "table": torch.arange(12, dtype=torch.int32).view(3, 4)}
    offs, total = bench._packed(t)
    assert all(o % 256 == 0 for o in offs.values())
    sizes = {n: v.numel() * v.element_size() for n, v in t.items()}
    spans = sorted((offs[n], offs[n] + sizes[n]) for n in t)
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))  # no overlap
    assert total >= spans[-1][1] and total % 256 == 0
    blob = torch.zeros(total, dtype=torch.uint8)
    for n, v in bench._views(blob, t, offs).items():
        assert v.is_contiguous() and v.dtype == t[n].dtype and v.shape == t[n].shape
        v.copy_(t[n])
    back = bench._views(blob, t, offs)
    assert all(torch.equal(back[n], t[n]) for n in t)


def _worker(rank, world, port, results):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    secs = [0.5, 1.25][rank]
    m = bench.max_over_ranks(secs, world, device="cpu")
    results[rank] = (m, bench.job_throughput(world, 256, 10, m))
    dist.destroy_process_group()


def test_max_over_ranks_gloo_world_two():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, results)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert results[0] == results[1] == (1.25, 2 * 256 * 10 / 1.25)
