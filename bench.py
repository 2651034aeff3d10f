#!/usr/bin/env python
"""Benchmark of the B200 DSA forward hot path (lightning indexer -> top-k ->
sparse MLA) on synthetic inputs, one JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole path over the workload's query rows with all
inputs resident in device memory. The timed region (K steps) is bracketed by a
barrier and a device synchronize, timed with CUDA events on the launching
stream, and reduced as the max over ranks. Every rank runs the full workload
on its own seeded inputs (independent sequences: weak scaling, no data-path
collective). Per-kernel durations come from CUDA events around each launch
inside the timed region. ``--impl reference`` times the CPU oracle on host
cores on a bounded sample of the same workload instead.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_attention_05_b200 import synth  # noqa: E402

METRIC = "DSA fwd query tokens/s at 128K ctx (decode & prefill); % of HBM / tensor roofline"
UNIT = "query tokens/s"
K_SEL = 2048

WORKLOADS = {
    # 128K-context decode: varlen paged cache, 2 query tokens per sequence
    "paged_decode_128k": dict(kind="paged", batch=128, q_per_seq=2, min_ctx=4096,
                              max_ctx=131072, page_size=64, seed=4),
    "decode_32k": dict(kind="decode", batch=64, ctx=32768, q_per_seq=1, seed=1),
    "prefill_8k": dict(kind="prefill", L=8192, seed=2),
    "prefill_128k": dict(kind="prefill", L=131072, seed=3, n_hot=64),
}
DEFAULT_WORKLOAD = "paged_decode_128k"
MHA_MAX_L = 16384  # MHA mode is the short-prefill path (dense causal cost grows as L^2)

SCORE_BUDGET = 2 << 30  # bytes of fp32 score rows per chunk (as the library's own plan)


# ----------------------------------------------------------------------------------------
# workload and algorithmic work
# ----------------------------------------------------------------------------------------
def make_problem(name: str, device, seed_offset: int = 0, batch=None) -> synth.Problem:
    w = dict(WORKLOADS[name])
    kind = w.pop("kind")
    w["seed"] = w["seed"] + 1000 * seed_offset
    if batch is not None:  # smaller decode batches for profiler captures
        if "batch" not in w:
            raise SystemExit(f"--batch applies to decode workloads, not {name}")
        w["batch"] = batch
    if kind == "paged":
        return synth.paged_decode(device=device, **w)
    if kind == "decode":
        return synth.decode(device=device, latent_std=0.5, **w)
    return synth.prefill(device=device, **w)


def algorithmic_work(p: synth.Problem, k: int = K_SEL, rows=None) -> dict:
    """Bytes and FLOPs the method must move or compute per step, per kernel.

    indexer: 132 B per visible key per sequence (128 B E4M3 + 4 B scale), the
             query rows (bf16) and weights, one fp32 score per (row, visible key);
             16384 FP8 FLOP per (row, visible key).
    top-k:   one read of each visible score, k int32 written per row.
    sparse MLA: Q (bf16), out (bf16), LSE, indices, 1152 B per selected latent
             row per query row; 278528 BF16 FLOP per (row, selected key).
    """
    seqlens = p.seqlens.cpu().long()
    pos = p.q_pos().long()
    if rows is not None:  # a subset of the query rows (context-parallel ranks)
        pos = pos[torch.as_tensor(rows)]
    n_vis = pos + 1
    n_sel = torch.clamp(n_vis, max=k)
    T = len(pos)
    keys = int(seqlens.sum())  # every sequence's keys are read once
    idx_bytes = 132 * keys + T * (64 * 128 * 2 + 64 * 4) + 4 * int(n_vis.sum())
    idx_flop = 16384 * int(n_vis.sum())
    topk_bytes = 4 * int(n_vis.sum()) + 4 * T * k
    mla_bytes = T * (128 * 576 * 2 + 128 * 512 * 2 + 128 * 4 + 4 * k) + 1152 * int(n_sel.sum())
    mla_flop = 278528 * int(n_sel.sum())
    return {
        "indexer": {"bytes": idx_bytes, "flop": idx_flop, "flop_dtype": "fp8"},
        "topk": {"bytes": topk_bytes, "flop": 0, "flop_dtype": None},
        "sparse_mla": {"bytes": mla_bytes, "flop": mla_flop, "flop_dtype": "bf16"},
        # indexer KL loss term: Q, LSE, idx, the score and latent row of every
        # selected key per row; the 128-head score of every selected key
        "indexer_kl": {"bytes": T * (128 * 576 * 2 + 128 * 4 + 4 * k + 4) +
                       (1152 + 4) * int(n_sel.sum()),
                       "flop": 2 * 128 * 576 * int(n_sel.sum()), "flop_dtype": "bf16"},
    }


def algorithmic_work_mha(p: synth.Problem, k: int = K_SEL) -> dict:
    """Bytes and FLOPs of a short-prefill step in MHA mode, per kernel.

    indexer / top-k: as in MQA mode, for the rows with more than k visible keys
             (the other rows select every visible key and need no scores).
    mask:    the selected indices of those rows read, their bit rows written.
    up-projection: per key the latent row (1152 B) read and 128 heads x (128 key
             + 128 value) bf16 written, plus both weight tensors once (32 MiB);
             2 * 512 * 256 * 128 BF16 FLOP per key.
    masked MHA: Q (128 x 192 bf16), out (128 x 128 bf16) and LSE per row, the
             decompressed keys/values once, the mask bits; 2 * 128 * (192 + 128)
             = 81920 BF16 FLOP per visible (row, key) pair: the mode computes the
             causal triangle and the mask only removes weight.
    """
    seqlens = p.seqlens.cpu().long()
    pos = p.q_pos().long()
    n_vis = pos + 1
    sel = n_vis > k
    T, T_sel = p.num_q, int(sel.sum())
    keys = int(seqlens.sum())
    idx_bytes = (132 * keys if T_sel else 0) + T_sel * (64 * 128 * 2 + 64 * 4) + \
        4 * int(n_vis[sel].sum())
    return {
        "indexer": {"bytes": idx_bytes, "flop": 16384 * int(n_vis[sel].sum()),
                    "flop_dtype": "fp8"},
        "topk": {"bytes": 4 * int(n_vis[sel].sum()) + 4 * T_sel * k, "flop": 0,
                 "flop_dtype": None},
        "mask": {"bytes": 4 * T_sel * k + int(((n_vis[sel] + 127) // 128).sum()) * 16,
                 "flop": 0, "flop_dtype": None},
        "up_proj": {"bytes": keys * (1152 + 128 * 256 * 2 + 128) + 2 * 128 * 128 * 512 * 2,
                    "flop": 2 * 512 * 256 * 128 * keys, "flop_dtype": "bf16"},
        "masked_mha": {"bytes": T * (128 * 192 * 2 + 128 * 128 * 2 + 128 * 4) +
                       keys * (128 * 256 * 2 + 128) +
                       int(((n_vis[sel] + 127) // 128).sum()) * 16,
                       "flop": 81920 * int(n_vis.sum()), "flop_dtype": "bf16"},
    }


def load_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        m = json.load(open(path))
        return {"hbm_gbs": m["hbm_gbs"], "bf16_tflops": m["bf16_tflops"],
                "bf16_tflops_sustained": m.get("bf16_tflops_sustained", m["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def roofline(kernel: str, work: dict, avg_s: float, peaks: dict, long_step: bool) -> dict:
    """Roofline of one kernel from its algorithmic work and average launch time."""
    w = work[kernel]
    bf16 = peaks["bf16_tflops_sustained"] if long_step else peaks["bf16_tflops"]
    tflops = {"bf16": bf16, "fp8": 2.0 * bf16}  # FP8 = BF16 measured x nominal 4.5/2.25
    t_mem = w["bytes"] / (peaks["hbm_gbs"] * 1e9)
    t_cmp = w["flop"] / (tflops[w["flop_dtype"]] * 1e12) if w["flop"] else 0.0
    if t_cmp > t_mem:
        achieved = w["flop"] / avg_s / 1e12
        peak = tflops[w["flop_dtype"]]
        r = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
             "dtype": w["flop_dtype"]}
    else:
        achieved = w["bytes"] / avg_s / 1e9
        peak = peaks["hbm_gbs"]
        r = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s"}
    r["frac"] = achieved / peak
    if r["unit"] == "TFLOP/s" and w["flop_dtype"] == "fp8" and peaks.get("fp8_tflops"):
        r["frac_of_measured_fp8"] = achieved / peaks["fp8_tflops"]
    r["peak_source"] = peaks["source"] + ("" if r["unit"] == "GB/s" else
                                          (" sustained" if long_step else " burst") +
                                          (" x2 (fp8 from bf16)" if w["flop_dtype"] == "fp8" else ""))
    return r


def step_roofline(work: dict, kernels, step_s: float, peaks: dict, long_step: bool) -> dict:
    """Roofline of the whole step: T_roof = max(all bytes / HBM, FP8 FLOP / FP8 peak +
    BF16 FLOP / BF16 peak) over the step's kernels, against the measured step time."""
    bf16 = peaks["bf16_tflops_sustained"] if long_step else peaks["bf16_tflops"]
    tflops = {"bf16": bf16, "fp8": 2.0 * bf16}
    nbytes = sum(work[k]["bytes"] for k in kernels)
    t_mem = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_cmp = sum(work[k]["flop"] / (tflops[work[k]["flop_dtype"]] * 1e12)
                for k in kernels if work[k]["flop"])
    t_roof = max(t_mem, t_cmp)
    return {"bound": "tensor" if t_cmp > t_mem else "hbm", "roofline_ms": 1e3 * t_roof,
            "ms_per_step": 1e3 * step_s, "frac": t_roof / step_s,
            "hbm_ms": 1e3 * t_mem, "tensor_ms": 1e3 * t_cmp, "bytes": nbytes,
            "kernels": list(kernels)}


def measure_fp8_peak() -> dict:
    """Dense FP8 (E4M3 x E4M3 -> bf16) throughput of cuBLASLt through torch._scaled_mm,
    8192^3, best of 10 bursts of 10: the measured FP8 figure that sits next to the
    2 x BF16 denominator (context, not the product path)."""
    n = 8192
    try:
        a = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn).t()
        one = torch.ones((), device="cuda")
        for _ in range(3):
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        best = float("inf")
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(10):
                torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1) / 1e3 / 10)
        del a, b
        torch.cuda.empty_cache()
        return {"fp8_tflops": 2 * n ** 3 / best / 1e12,
                "fp8_source": "torch._scaled_mm e4m3 x e4m3 -> bf16, 8192^3, best of 10 "
                              "bursts of 10, measured in this run (cuBLASLt)"}
    except Exception as e:  # noqa: BLE001 - context only
        return {"fp8_tflops": None, "fp8_source": f"not measured: {type(e).__name__}"}


def dram_traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes from a committed ncu summary, if it matches the
    kernel's source as built now (its header and the PTX helpers; else null)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    try:
        d = json.load(open(path))
        e = d.get(workload, {}).get(kernel)
        if not e:
            return None
        from sparse_attention_05_b200.build import source_digest
        if e.get("source_digest") != source_digest(kernel):
            return None
        return e["bytes_per_launch"]
    except Exception:
        return None


# ----------------------------------------------------------------------------------------
# clocks
# ----------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.path = None
        try:
            # select this process's GPU by UUID: nvidia-smi ignores CUDA_VISIBLE_DEVICES
            gpu = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) == 6 and parts[0].isdigit():
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[2 + i] == "Active"})
        return {"sm_mhz": statistics.median(float(r[0]) for r in rows),
                "sm_max_mhz": float(rows[0][1]), "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------------------
MLA_PART_BYTES = 128 * 512 * 4 + 128 * 4  # one segment's fp32 output and LSE


def mla_split_plan(rows: int, k: int, scratch_bytes: int, sms=None):
    """(split rows, segments per split row) of one dsa_sparse_mla_fwd_ws call under
    the library's rule: the rows of a last wave (clusters of 2 SMs) that is at most
    half full run as 2..8 segments of >= 6 blocks of 48 keys, as many as the scratch
    holds. Used for the launch count; tests pin it to the library's workspace sizes."""
    if sms is None:
        sms = torch.cuda.get_device_properties(0).multi_processor_count
    wave = sms // 2
    tail = rows % wave if wave >= 2 and rows > 0 else 0
    if tail == 0:
        return 0, 1
    nb = -(-k // 48)
    s = min(wave // tail, 8, nb // 6)
    while s >= 2 and tail * s * MLA_PART_BYTES > scratch_bytes:
        s -= 1
    if s < 2:
        return 0, 1
    bps = -(-nb // s)
    nseg = -(-nb // bps)
    return (tail, nseg) if nseg >= 2 else (0, 1)


def mla_split_launches(rows: int, k: int, scratch_bytes: int) -> int:
    """Kernel launches of one dsa_sparse_mla_fwd_ws call: the attention, plus the
    segment merge when rows are split."""
    return 2 if mla_split_plan(rows, k, scratch_bytes)[0] else 1


class Runner:
    """Holds the device buffers of one workload and runs one step of the path
    through the library's stage calls (the same launches dsa_forward makes)."""

    def __init__(self, p: synth.Problem, k: int = K_SEL, with_kl: bool = False,
                 split_topk: bool = False):
        from sparse_attention_05_b200 import dsa
        self.dsa = dsa
        self.p = p
        self.k = k
        self.kv = dsa.KvLayout.of(p)
        T, B = p.num_q, p.batch
        self.ld = dsa.round_up(p.max_ctx, 128)
        rows = max(1, SCORE_BUDGET // (self.ld * 4 * B))
        if rows >= p.q_per_seq:
            rows = p.q_per_seq
        elif rows >= 4:
            rows &= ~3
        self.chunks = [(r0, min(rows, p.q_per_seq - r0)) for r0 in range(0, p.q_per_seq, rows)]
        # the score rows, whose space the sparse MLA then uses as its split scratch
        # (as in dsa_forward's workspace)
        nscore = B * rows * self.ld * 4
        self.ws = torch.empty(max(nscore, dsa.dsa_sparse_mla_workspace_size()), dtype=torch.uint8,
                              device=p.q.device)
        self.scores = self.ws[:nscore].view(torch.float32).view(B * rows, self.ld)
        self.idx = torch.empty(T, k, dtype=torch.int32, device=p.q.device)
        self.out = torch.empty(T, 128, 512, dtype=torch.bfloat16, device=p.q.device)
        self.lse = torch.empty(T, 128, dtype=torch.float32, device=p.q.device)
        self.mla_ws = self.ws
        # the selection dsa_forward makes: one CTA per row (dsa_topk); with --split-topk
        # the split path of dsa_topk_ws (threshold, chunk sweep, per-row selection)
        tk = (dsa.dsa_topk_workspace_size(self.kv, T, p.q_per_seq, k, rows=(0, rows))
              if split_topk else 0)
        self.topk_ws = torch.empty(max(tk, 256), dtype=torch.uint8, device=p.q.device)
        self.topk_launches = 3 if tk else 1
        self.with_kl = with_kl
        if with_kl:
            if len(self.chunks) > 1:
                raise SystemExit("--kl needs every score row in one chunk (not this workload)")
            self.kl = torch.empty(T, dtype=torch.float32, device=p.q.device)
            # the KL term reads the score rows after the attention: keep them intact
            self.mla_ws = torch.empty(dsa.dsa_sparse_mla_workspace_size(), dtype=torch.uint8,
                                      device=p.q.device)
        self.launches_per_step = ((1 + self.topk_launches) * len(self.chunks) +
                                  mla_split_launches(T, k, self.mla_ws.numel()) +
                                  (1 if with_kl else 0))

    def step(self, ev=None):
        d, p = self.dsa, self.p
        for r0, rc in self.chunks:
            if ev is not None:
                ev["indexer"].append(_record())
            d.dsa_indexer_scores(p.q_idx, p.w, p.k_idx, p.k_scale, self.kv, p.q_per_seq,
                                 scores=self.scores[: p.batch * rc], rows=(r0, rc))
            if ev is not None:
                ev["indexer"].append(_record())
                ev["topk"].append(_record())
            self.topk(r0, rc)
            if ev is not None:
                ev["topk"].append(_record())
        if ev is not None:
            ev["sparse_mla"].append(_record())
        d.dsa_sparse_mla_fwd_ws(p.q, p.kv, self.kv, p.q_per_seq, self.idx, p.scale,
                                workspace=self.mla_ws, out=self.out, lse=self.lse)
        if ev is not None:
            ev["sparse_mla"].append(_record())
        if self.with_kl:  # the indexer's KL loss term over the selected sets
            if ev is not None:
                ev["indexer_kl"].append(_record())
            d.dsa_indexer_kl(p.q, p.kv, self.kv, p.q_per_seq, self.idx, p.scale, self.lse,
                             self.scores, kl=self.kl)
            if ev is not None:
                ev["indexer_kl"].append(_record())

    def topk(self, r0, rc):
        d, p = self.dsa, self.p
        if self.topk_launches > 1:
            d.dsa_topk_ws(self.scores[: p.batch * rc], self.kv, p.q_per_seq, self.k,
                          workspace=self.topk_ws, idx=self.idx, rows=(r0, rc))
        else:
            d.dsa_topk(self.scores[: p.batch * rc], self.kv, p.q_per_seq, self.k, idx=self.idx,
                       rows=(r0, rc))

    # end-to-end through the public call dsa_forward
    def e2e_host_inputs(self):
        p = self.p
        h = {"q_idx": p.q_idx, "w": p.w, "q": p.q, "seqlens": p.seqlens}
        if p.paged:
            h["block_table"] = p.block_table
        return h

    def e2e_workspace(self):
        d, p = self.dsa, self.p
        return max(256, d.dsa_workspace_size(self.kv, p.num_q, p.q_per_seq, self.k))

    def e2e_call(self, g, kv, ws, out, lse, stream):
        d, p = self.dsa, self.p
        d.dsa_forward(g["q_idx"], g["w"], p.k_idx, p.k_scale, g["q"], p.kv, kv, p.q_per_seq,
                      self.k, p.scale, workspace=ws, out=out, lse=lse, stream=stream)


class CpRunner(Runner):
    """Context-parallel prefill on this rank: the rank owns a contiguous token shard
    of the per-token caches; every step all-gathers them (NCCL) and runs the stage
    calls on the rank's zigzag query rows (row windows of the library calls)."""

    def __init__(self, p: synth.Problem, world: int, rank: int, k: int = K_SEL):
        from sparse_attention_05_b200 import cp
        super().__init__(p, k)
        self.cp, self.world = cp, world
        L = p.max_ctx
        b, e = cp.token_shard(L, world, rank)
        self.shards = {n: getattr(p, n)[0, b:e].clone() for n in ("k_idx", "k_scale", "kv")}
        self.windows = cp.zigzag_windows(L, world, rank)
        self.rows = [i for r0, rc in self.windows for i in range(r0, r0 + rc)]
        # score chunks inside each window (the same budget as the single-GPU plan)
        per = max(1, SCORE_BUDGET // (self.ld * 4 * p.batch))
        if per >= 4:
            per &= ~3
        self.chunks = [(r0 + c, min(per, rc - c)) for r0, rc in self.windows
                       for c in range(0, rc, per)]
        self.launches_per_step = (1 + self.topk_launches) * len(self.chunks) + len(self.windows)

    def step(self, ev=None):
        d, p = self.dsa, self.p
        if ev is not None:
            ev["allgather"].append(_record())
        full = {n: self.cp.allgather_cache(t, p.max_ctx, self.world)
                for n, t in self.shards.items()}
        k_idx, k_scale, kv = full["k_idx"][None], full["k_scale"][None], full["kv"][None]
        if ev is not None:
            ev["allgather"].append(_record())
        for r0, rc in self.chunks:
            if ev is not None:
                ev["indexer"].append(_record())
            d.dsa_indexer_scores(p.q_idx, p.w, k_idx, k_scale, self.kv, p.q_per_seq,
                                 scores=self.scores[: p.batch * rc], rows=(r0, rc))
            if ev is not None:
                ev["indexer"].append(_record())
                ev["topk"].append(_record())
            self.topk(r0, rc)
            if ev is not None:
                ev["topk"].append(_record())
        for r0, rc in self.windows:
            if ev is not None:
                ev["sparse_mla"].append(_record())
            d.dsa_sparse_mla_fwd(p.q, kv, self.kv, p.q_per_seq, self.idx, p.scale, out=self.out,
                                 lse=self.lse, rows=(r0, rc))
            if ev is not None:
                ev["sparse_mla"].append(_record())


class FusedRunner(Runner):
    """The fused indexer -> top-k selection (no stored score rows; one host sync per
    chunk of rows inside the call) followed by the sparse MLA."""

    def __init__(self, p: synth.Problem, k: int = K_SEL):
        super().__init__(p, k)
        d = self.dsa
        nbytes = d.dsa_fused_workspace_size(self.kv, p.num_q, p.q_per_seq, k)
        self.ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=p.q.device)
        self.scores = None  # never materialised
        self.mla_ws = self.ws  # dead once the selection is done (as in dsa_forward_fused)
        # per chunk: sampled indexer, threshold top-k, filtering indexer, selection
        per = max(1, (2 << 30) // (p.batch * (self.ld // 8 * 4 + 12 + 8192 * 8)))
        self.launches_per_step = (4 * (-(-p.q_per_seq // per))
                                  + mla_split_launches(p.num_q, k, self.ws.numel()))

    def step(self, ev=None):
        d, p = self.dsa, self.p
        if ev is not None:
            ev["select_fused"].append(_record())
        d.dsa_select_fused(p.q_idx, p.w, p.k_idx, p.k_scale, self.kv, p.q_per_seq, self.k,
                           idx=self.idx, workspace=self.ws)
        if ev is not None:
            ev["select_fused"].append(_record())
            ev["sparse_mla"].append(_record())
        d.dsa_sparse_mla_fwd_ws(p.q, p.kv, self.kv, p.q_per_seq, self.idx, p.scale,
                                workspace=self.mla_ws, out=self.out, lse=self.lse)
        if ev is not None:
            ev["sparse_mla"].append(_record())


class MhaRunner:
    """Short-prefill step in MHA mode through the library's stage calls (the same
    launches dsa_mha_prefill makes): indexer + top-k for the rows with more than
    k visible keys, their selection masks, the up-projection of the latent cache
    and the masked MHA."""

    STAGES = ("indexer", "topk", "mask", "up_proj", "masked_mha")

    def __init__(self, p: synth.Problem, k: int = K_SEL, seed: int = 0):
        from sparse_attention_05_b200 import dsa
        if p.q_per_seq != p.max_ctx:
            raise SystemExit("--mode mha runs the prefill workloads")
        self.dsa, self.p, self.k = dsa, p, k
        self.m = synth.mha_inputs(p, seed + 500, device=p.q.device)
        self.kv = dsa.KvLayout.of(p)
        T, B, dev = p.num_q, p.batch, p.q.device
        self.ld = dsa.round_up(p.max_ctx, 128)
        sel_begin = min(p.q_per_seq, max(0, k))   # row i selects all of 0..i when i < k
        n_sel = p.q_per_seq - sel_begin
        rows = max(1, SCORE_BUDGET // (self.ld * 4 * B))
        if rows >= n_sel:
            rows = max(1, n_sel)
        elif rows >= 4:
            rows &= ~3
        self.sel = (sel_begin, n_sel)
        self.chunks = [(r0, min(rows, p.q_per_seq - r0)) for r0 in range(sel_begin, p.q_per_seq, rows)]
        self.scores = torch.empty(B * rows, self.ld, dtype=torch.float32, device=dev)
        self.idx = torch.empty(T, k, dtype=torch.int32, device=dev)
        cp = dsa.mha_ctx_pad(self.kv)
        self.mask = torch.zeros(T, cp // 32, dtype=torch.int32, device=dev)
        self.kn = torch.empty(B, 128, cp, 128, dtype=torch.bfloat16, device=dev)
        self.kr = torch.empty(B, cp, 64, dtype=torch.bfloat16, device=dev)
        self.vv = torch.empty(B, 128, cp, 128, dtype=torch.bfloat16, device=dev)
        self.out = torch.empty(T, 128, 128, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(T, 128, dtype=torch.float32, device=dev)
        self.launches_per_step = 2 * len(self.chunks) + (1 if n_sel else 0) + 2

    def step(self, ev=None):
        d, p, m = self.dsa, self.p, self.m

        def mark(name):
            if ev is not None:
                ev[name].append(_record())
        for r0, rc in self.chunks:
            mark("indexer")
            d.dsa_indexer_scores(p.q_idx, p.w, p.k_idx, p.k_scale, self.kv, p.q_per_seq,
                                 scores=self.scores[: p.batch * rc], rows=(r0, rc))
            mark("indexer")
            mark("topk")
            d.dsa_topk(self.scores[: p.batch * rc], self.kv, p.q_per_seq, self.k, idx=self.idx,
                       rows=(r0, rc))
            mark("topk")
        if self.sel[1]:
            mark("mask")
            d.dsa_selection_mask(self.idx, self.kv, p.q_per_seq, mask=self.mask, rows=self.sel)
            mark("mask")
        mark("up_proj")
        d.dsa_mla_up_project(p.kv, m.w_uk, m.w_uv, self.kv, self.kn, self.kr, self.vv)
        mark("up_proj")
        mark("masked_mha")
        d.dsa_masked_mha(m.q_mha, self.kn, self.kr, self.vv, self.kv, p.q_per_seq, p.scale,
                         mask=self.mask if self.sel[1] else None, k=self.k, out=self.out,
                         lse=self.lse)
        mark("masked_mha")

    # end-to-end through the public composed call
    def e2e_host_inputs(self):
        return {"q_idx": self.p.q_idx, "w": self.p.w, "q_mha": self.m.q_mha,
                "seqlens": self.p.seqlens}

    def e2e_workspace(self):
        d, p = self.dsa, self.p
        return max(256, d.dsa_mha_workspace_size(self.kv, p.num_q, p.q_per_seq, self.k))

    def e2e_call(self, g, kv, ws, out, lse, stream):
        d, p, m = self.dsa, self.p, self.m
        d.dsa_mha_prefill(g["q_idx"], g["w"], p.k_idx, p.k_scale, g["q_mha"], p.kv, m.w_uk,
                          m.w_uv, kv, p.q_per_seq, self.k, p.scale, workspace=ws, out=out,
                          lse=lse, stream=stream)


def _record():
    e = torch.cuda.Event(enable_timing=True)
    e.record()
    return e


def _pairs_ms(evs):
    return [evs[i].elapsed_time(evs[i + 1]) for i in range(0, len(evs), 2)]


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device="cuda") -> float:
    """Slowest rank's time: the whole job is as fast as its slowest GPU."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, rows_per_rank: int, steps: int, max_secs: float) -> float:
    """Whole-job query tokens/s: every rank processed rows_per_rank rows per step."""
    return world * rows_per_rank * steps / max_secs


def _packed(tensors: dict, align: int = 256):
    """Byte offsets of the tensors packed one after another (each at a multiple of
    ``align``) and the packed size."""
    offs, tot = {}, 0
    for n, v in tensors.items():
        offs[n] = tot
        tot += (v.numel() * v.element_size() + align - 1) // align * align
    return offs, tot


def _views(blob, like: dict, offs: dict) -> dict:
    """Tensors shaped like ``like``'s, viewing ``blob`` (uint8) at ``offs``."""
    return {n: blob[offs[n]:offs[n] + v.numel() * v.element_size()].view(v.dtype).view(v.shape)
            for n, v in like.items()}


def e2e_run(r, steps: int, warmup: int, world: int):
    """Through the public call (dsa_forward; dsa_mha_prefill in MHA mode), with
    the step's query-side inputs copied from pinned host memory and the result
    read back every step.

    The step's inputs sit packed in one pinned host staging buffer and go up as
    one copy into a device buffer the calls read through views; the outputs (out
    and LSE) are views of one device buffer that comes down as one copy (a copy
    engine pays a fixed cost per transfer: five uploads per step instead of one
    cost 0.14 ms per step on the default workload). Copies and compute overlap
    across steps the way a serving loop would run them: step i's inputs go up on
    an upload stream while earlier steps compute, and finished steps' outputs come
    down on a download stream while step i computes (NBUF device buffers for each,
    so an upload or a download never waits for the step right before it). Every
    step still makes its own full host->device and device->host copies inside the
    timed region."""
    d, p = r.dsa, r.p
    NBUF = 3
    hin = {n: v.cpu().contiguous() for n, v in r.e2e_host_inputs().items()}
    in_offs, in_bytes = _packed(hin)
    host_in = torch.zeros(in_bytes, dtype=torch.uint8).pin_memory()
    for n, v in _views(host_in, hin, in_offs).items():
        v.copy_(hin[n])
    dev_in = [torch.empty(in_bytes, dtype=torch.uint8, device="cuda") for _ in range(NBUF)]
    dev = [_views(blob, hin, in_offs) for blob in dev_in]
    olike = {"out": r.out, "lse": r.lse}
    out_offs, out_bytes = _packed(olike)
    dev_out = [torch.empty(out_bytes, dtype=torch.uint8, device="cuda") for _ in range(NBUF)]
    outs = [_views(blob, olike, out_offs) for blob in dev_out]
    host_out = [torch.empty(out_bytes, dtype=torch.uint8).pin_memory() for _ in range(NBUF)]
    ws = torch.empty(r.e2e_workspace(), dtype=torch.uint8, device="cuda")
    kvs = [d.KvLayout(batch=p.batch, max_ctx=p.max_ctx, seqlens=dev[b]["seqlens"],
                      block_table=dev[b].get("block_table"), page_size=p.page_size,
                      num_pages=r.kv.num_pages) for b in range(NBUF)]
    s_up, s_cmp, s_down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = {n: [torch.cuda.Event() for _ in range(NBUF)]
          for n in ("in_ready", "in_free", "done", "out_free")}

    def one(i):
        b = i % NBUF
        with torch.cuda.stream(s_up):
            if i >= NBUF:
                s_up.wait_event(ev["in_free"][b])
            dev_in[b].copy_(host_in, non_blocking=True)
            ev["in_ready"][b].record(s_up)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev["in_ready"][b])
            if i >= NBUF:
                s_cmp.wait_event(ev["out_free"][b])
            r.e2e_call(dev[b], kvs[b], ws, outs[b]["out"], outs[b]["lse"], s_cmp)
            ev["in_free"][b].record(s_cmp)
            ev["done"][b].record(s_cmp)
        with torch.cuda.stream(s_down):
            s_down.wait_event(ev["done"][b])
            host_out[b].copy_(dev_out[b], non_blocking=True)
            ev["out_free"][b].record(s_down)

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize()
    barrier(world)
    t0 = _record()
    for st in (s_up, s_cmp, s_down):
        st.wait_event(t0)
    for i in range(warmup, warmup + steps):
        one(i)
    torch.cuda.current_stream().wait_stream(s_down)
    t1 = _record()
    torch.cuda.synchronize()
    barrier(world)
    secs = max_over_ranks(t0.elapsed_time(t1) / 1e3, world)
    return {"value": job_throughput(world, p.num_q, steps, secs), "unit": UNIT,
            "h2d_bytes_per_step": in_bytes,
            "d2h_bytes_per_step": out_bytes, "ms_per_step": 1e3 * secs / steps,
            "overlap": "uploads of later steps and downloads of earlier ones overlap the compute "
                       "of step i (%d buffers each); one packed copy each way per step" % NBUF}


# ----------------------------------------------------------------------------------------
# CPU oracle (baseline and reference arm)
# ----------------------------------------------------------------------------------------
def oracle_sample_inputs(p: synth.Problem, rows):
    """numpy inputs for the oracle restricted to the sequences of ``rows``,
    each rebuilt contiguously on the host (pages resolved through the block
    table), plus the rows' indices in that reduced problem."""
    seqs = sorted({int(t) // p.q_per_seq for t in rows})
    seqlens = p.seqlens.cpu().long()
    ctx = int(max(seqlens[s] for s in seqs))
    kc = np.zeros((len(seqs), ctx, 128), np.uint8)
    ks = np.zeros((len(seqs), ctx), np.float32)
    kvc = np.zeros((len(seqs), ctx, 576), np.float32)
    for i, s in enumerate(seqs):
        n = int(seqlens[s])
        if p.paged:
            pages = p.block_table[s, : (n + p.page_size - 1) // p.page_size].long()
            kc[i, :n] = p.k_idx[pages].reshape(-1, 128)[:n].cpu().numpy()
            ks[i, :n] = p.k_scale[pages].reshape(-1)[:n].cpu().numpy()
            kvc[i, :n] = p.kv[pages].reshape(-1, 576)[:n].float().cpu().numpy()
        else:
            kc[i, :n] = p.k_idx[s, :n].cpu().numpy()
            ks[i, :n] = p.k_scale[s, :n].cpu().numpy()
            kvc[i, :n] = p.kv[s, :n].float().cpu().numpy()
    trows = torch.as_tensor(list(rows))
    q_seq = np.array([seqs.index(int(t) // p.q_per_seq) for t in rows])
    q_pos = p.q_pos()[trows].numpy()
    return dict(q_idx=p.q_idx[trows].float().cpu().numpy(), w=p.w[trows].cpu().numpy(),
                k_idx=kc, k_scale=ks, q=p.q[trows].float().cpu().numpy(), kv=kvc,
                q_seq=q_seq, q_pos=q_pos, ld=ctx)


def oracle_step(inp, scale, k=K_SEL):
    from oracle import dsa_forward as oracle_forward
    return oracle_forward(inp["q_idx"], inp["w"], inp["k_idx"], inp["k_scale"], inp["q"],
                          inp["kv"], inp["q_seq"], inp["q_pos"], k=k, scale=scale, d_v=512,
                          ld=inp["ld"])


def oracle_step_mha(p: synth.Problem, m: synth.MhaInputs, rows, k=K_SEL):
    """The oracle's MHA-mode prefill for ``rows``: indexer + top-k for the rows with
    more than k visible keys, then the masked MHA (every visible key otherwise)."""
    from oracle import indexer_scores, masked_mha, topk_rows
    inp = oracle_sample_inputs(p, rows)
    trows = torch.as_tensor(list(rows))
    q_mha = m.q_mha[trows].float().cpu().numpy()
    local = np.arange(len(rows))
    need = [r for r in local if inp["q_pos"][r] + 1 > k]
    idx = [np.arange(int(inp["q_pos"][r]) + 1) for r in local]
    if need:
        sc = indexer_scores(inp["q_idx"], inp["w"], inp["k_idx"], inp["k_scale"], inp["q_seq"],
                            inp["q_pos"], ld=inp["ld"], rows=need)
        for r, sel in zip(need, topk_rows(sc, inp["q_pos"], k, rows=need)):
            idx[r] = sel
    return masked_mha(q_mha, inp["kv"], inp["q_seq"], inp["q_pos"], idx, p.scale,
                      m.w_uk.float().cpu().numpy(), m.w_uv.float().cpu().numpy())


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


def host_cpu() -> dict:
    """The host the oracle ran on: CPU model and logical core count."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "nproc": os.cpu_count() or 1}


def cpu_baseline(p: synth.Problem, name: str, budget_s: float = 12.0, seed: int = 0,
                 mha=None) -> dict:
    """The oracle on a bounded sample: two query rows of a random sequence per call
    (their last rows in MQA mode; two random rows in MHA mode, whose cost is the
    up-projection of every visible key per head), until ``budget_s`` of host time."""
    rng = np.random.default_rng(seed)
    rows_done, elapsed, seqs = 0, 0.0, []
    while elapsed < budget_s and rows_done < p.num_q:
        b = int(rng.integers(0, p.batch))
        r0 = b * p.q_per_seq
        if mha is None:
            rows = list(range(r0, r0 + min(p.q_per_seq, 2)))
            inp = oracle_sample_inputs(p, rows)
            t0 = time.perf_counter()
            oracle_step(inp, p.scale)
        else:
            rows = sorted(r0 + int(i) for i in rng.choice(p.q_per_seq, 2, replace=False))
            t0 = time.perf_counter()
            oracle_step_mha(p, mha, rows)
        elapsed += time.perf_counter() - t0
        rows_done += len(rows)
        seqs.append(b)
    what = ("indexer+top-k (rows past k)+masked MHA per row" if mha is not None
            else "full indexer+top-k+attention per row")
    nt = blas_threads()
    return {"value": rows_done / elapsed, "unit": UNIT, "cores": nt, "processes": 1,
            "parallelism": f"1 process; numpy's BLAS on {nt} threads (matmuls), the rest "
                           f"single-threaded", **host_cpu(),
            "kind": "oracle",
            "sample": f"{rows_done} query rows of {name} (sequences {seqs[:8]}"
                      f"{'...' if len(seqs) > 8 else ''}), {what}, "
                      f"{elapsed:.1f} s of host time, 1 process with {nt} BLAS threads"}


def reference_arm(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    p = make_problem(args.workload, dev)
    rng = np.random.default_rng(123)
    per_step_rows = min(p.q_per_seq, 2)
    m = synth.mha_inputs(p, 500, device=dev) if args.mode == "mha" else None

    def one():
        b = int(rng.integers(0, p.batch))
        if m is not None:
            rows = sorted(b * p.q_per_seq + int(i)
                          for i in rng.choice(p.q_per_seq, per_step_rows, replace=False))
            t0 = time.perf_counter()
            oracle_step_mha(p, m, rows)
            return time.perf_counter() - t0
        rows = list(range(b * p.q_per_seq, b * p.q_per_seq + per_step_rows))
        inp = oracle_sample_inputs(p, rows)
        t0 = time.perf_counter()
        oracle_step(inp, p.scale)
        return time.perf_counter() - t0

    for _ in range(args.warmup):
        one()
    secs = sum(one() for _ in range(args.steps))
    value = args.steps * per_step_rows / secs
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, **WORKLOADS[args.workload],
                       **({"mode": "mha (masked MHA emulation of DSA)"} if m is not None else {}),
                       "sample_rows_per_step": per_step_rows},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(),
                             "processes": 1, **host_cpu(), "kind": "oracle",
                             "sample": f"{per_step_rows} query rows of one random sequence per "
                                       f"step, {args.steps} steps, 1 process with "
                                       f"{blas_threads()} BLAS threads"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ----------------------------------------------------------------------------------------
def measure(r, work: dict, workload: str, steps: int, warmup: int, world: int, local: int,
            soak_s: float, ev_names, peaks: dict) -> dict:
    """Warm-up, a short untimed soak (clock samples start), then exactly ``steps``
    steps bracketed by a barrier and a device synchronize on both sides, timed with
    CUDA events on the launching stream (max over ranks); per-kernel CUDA events
    inside the same region give each stage's time and roofline."""
    for _ in range(warmup):
        r.step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    t_soak = time.perf_counter()
    while time.perf_counter() - t_soak < soak_s:
        r.step()
        torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ev = {n: [] for n in ev_names}
    start = _record()
    for _ in range(steps):
        r.step(ev)
    stop = _record()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    secs = max_over_ranks(start.elapsed_time(stop) / 1e3, world)

    per_kernel = {kname: _pairs_ms(e) for kname, e in ev.items() if e}
    launches = {kname: len(v) for kname, v in per_kernel.items()}
    total_ms = {kname: sum(v) for kname, v in per_kernel.items()}
    # the dominant kernel (the all-gather of the context-parallel mode is a collective)
    dominant = max((k for k in total_ms if k != "allgather"), key=total_ms.get)
    long_step = secs / steps > 0.05
    avg_s = total_ms[dominant] / 1e3 / steps  # one step's worth of that kernel
    roof = roofline(dominant, work, avg_s, peaks, long_step)
    roof["kernel"] = dominant
    roof["launches_per_step"] = launches[dominant] // steps
    roof["traffic"] = dram_traffic(dominant, workload)
    roof["step"] = step_roofline(work, [k for k in per_kernel if k != "allgather"],
                                 secs / steps, peaks, long_step)
    stages = {}
    for kname in per_kernel:
        a = total_ms[kname] / 1e3 / steps
        rf = roofline(kname, work, a, peaks, long_step)
        stages[kname] = {"ms_per_step": 1e3 * a, "share": total_ms[kname] / sum(total_ms.values()),
                         "bound": rf["bound"], "frac": rf["frac"],
                         "achieved": rf["achieved"], "unit": rf["unit"]}
        if "frac_of_measured_fp8" in rf:
            stages[kname]["frac_of_measured_fp8"] = rf["frac_of_measured_fp8"]
    return {"secs": secs, "clocks": clk, "roofline": roof, "stages": stages,
            "launches": launches}


def secondary_prefill(args, world: int, local: int, rank: int, peaks: dict) -> dict:
    """The metric's other half: the 128K causal prefill step (MQA mode) measured in the
    same run as the decode line, with the same protocol (3 warm-up, 3 timed steps)."""
    name = "prefill_128k"
    p = make_problem(name, "cuda", seed_offset=rank)
    r = Runner(p)
    work = algorithmic_work(p)
    steps, warmup = 3, 3
    m = measure(r, work, name, steps, warmup, world, local, 0.0,
                ("indexer", "topk", "sparse_mla"), peaks)
    out = {"workload": name, **WORKLOADS[name], "value": world * p.num_q * steps / m["secs"],
           "unit": UNIT, "ms_per_step": 1e3 * m["secs"] / steps, "steps": steps,
           "warmup": warmup, "roofline": m["roofline"], "stages": m["stages"],
           "clocks": m["clocks"], "gpu_launches": r.launches_per_step * steps,
           "query_rows_per_gpu": p.num_q}
    del r, p
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--kl", action="store_true",
                    help="also run the indexer KL loss term (training target) every step")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the decode batch (small cases for profiler captures)")
    ap.add_argument("--cp", action="store_true",
                    help="context-parallel prefill: caches sharded by token, all-gathered "
                         "every step, query rows split zigzag across the ranks")
    ap.add_argument("--fused", action="store_true",
                    help="fused indexer -> top-k selection (no stored score rows)")
    ap.add_argument("--mode", default="mqa", choices=["mqa", "mha"],
                    help="mha: short-prefill DSA in MLA's MHA mode (masked MHA; prefill_8k)")
    ap.add_argument("--split-topk", action="store_true",
                    help="time the split selection of dsa_topk_ws (long rows swept by several "
                         "CTAs) instead of dsa_forward's one CTA per row")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the 128K prefill half of the metric in the default run")
    ap.add_argument("--no-fp8-peak", action="store_true",
                    help="skip the live FP8 GEMM measurement (context for the FP8 fractions)")
    ap.add_argument("--soak-s", type=float, default=1.0,
                    help="untimed seconds of steps right before the timed region (clock samples)")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)

    if args.mode == "mha":
        w = WORKLOADS[args.workload]
        if w["kind"] != "prefill" or w["L"] > MHA_MAX_L:
            raise SystemExit(f"--mode mha is the short-prefill path: prefill workloads with "
                             f"L <= {MHA_MAX_L} (not {args.workload})")
        if args.kl:
            raise SystemExit("--kl runs with the MQA-mode path")
    if args.impl == "reference":
        return reference_arm(args)

    if args.cp and (WORKLOADS[args.workload]["kind"] != "prefill" or args.mode != "mqa"
                    or args.kl):
        raise SystemExit("--cp runs the prefill workloads in MQA mode")
    world, rank, local = dist_setup(args.gpus)
    # context parallel: one sequence shared by all ranks (same seed everywhere)
    p = make_problem(args.workload, "cuda", seed_offset=0 if args.cp else rank,
                     batch=args.batch)
    if args.fused and (args.cp or args.mode != "mqa" or args.kl):
        raise SystemExit("--fused runs the MQA-mode path alone")
    if args.fused:
        r = FusedRunner(p)
        work = algorithmic_work(p)
        # the fused selection does the indexer's work (plus a 1/8 sample) and the top-k's
        work["select_fused"] = dict(work["indexer"])
    elif args.cp:
        r = CpRunner(p, world, rank)
        work = algorithmic_work(p, rows=r.rows)
        L = p.max_ctx
        work["allgather"] = {"bytes": L * (128 + 4 + 1152) * (world - 1) // max(world, 1),
                             "flop": 0, "flop_dtype": None}
    elif args.mode == "mha":
        r = MhaRunner(p, seed=rank)
        work = algorithmic_work_mha(p)
    else:
        r = Runner(p, with_kl=args.kl, split_topk=args.split_topk)
        work = algorithmic_work(p)
    peaks = load_peaks()

    if args.mode == "mha":
        ev_names = MhaRunner.STAGES
    elif args.cp:
        ev_names = ("allgather", "indexer", "topk", "sparse_mla")
    elif args.fused:
        ev_names = ("select_fused", "sparse_mla")
    else:
        ev_names = ("indexer", "topk", "sparse_mla")
    if args.kl:
        ev_names = ev_names + ("indexer_kl",)
    peaks["fp8_tflops"] = None
    if not args.no_fp8_peak:
        peaks.update(measure_fp8_peak())
    m = measure(r, work, args.workload, args.steps, args.warmup, world, local, args.soak_s,
                ev_names, peaks)
    secs, clk, roof, stages = m["secs"], m["clocks"], m["roofline"], m["stages"]

    # context parallel: the end-to-end arm of the public call is the single-GPU one
    e2e = None if (args.no_e2e or args.cp or args.fused) else \
        e2e_run(r, max(3, args.steps // 2), 3, world)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(p, args.workload, mha=r.m if args.mode == "mha" else None)

    # the metric's other half, measured in the same run: the default (decode) line
    # also carries the 128K prefill step
    secondary = None
    run_secondary = (args.workload == DEFAULT_WORKLOAD and not args.no_secondary and
                     not (args.cp or args.fused or args.kl or args.batch) and args.mode == "mqa")
    n_launch = r.launches_per_step * args.steps
    rows_primary = len(r.rows) if args.cp else p.num_q
    rows_problem = p.num_q
    if run_secondary:
        del r, p
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        secondary = secondary_prefill(args, world, local, rank, peaks)

    if rank == 0:
        cfg = {"workload": args.workload, **WORKLOADS[args.workload],
               **({"batch": args.batch} if args.batch else {}),
               **({"indexer_kl": True} if args.kl else {}),
               **({"selection": "fused indexer -> top-k"} if args.fused else {}), "k": K_SEL,
               **({"mode": "mha (masked MHA emulation of DSA)", "heads": 128, "d_qk": 192,
                   "d_v": 128, "d_latent": 576} if args.mode == "mha" else
                  {"heads": 128, "d_qk": 576, "d_v": 512}),
               "h_idx": 64, "d_idx": 128,
               "query_rows_per_gpu": rows_primary,
               "l2": "inputs larger than L2 (no flush)",
               "parallelism": (f"cp{world} (caches sharded by token and all-gathered every "
                               f"step, query rows zigzag across GPUs)" if args.cp else
                               f"dp{world} (independent sequences per GPU)")}
        # context parallel: the job processes one sequence's L rows per step
        rows_job = rows_problem if args.cp else world * rows_problem
        line = {
            "metric": METRIC, "value": rows_job * args.steps / secs,
            "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True,
            "scaling": "strong" if args.cp else "weak",
            "vs_baseline": None, "dtype": "e4m3+bf16", "data": "synthetic", "config": cfg,
            "roofline": roof, "stages": stages, "clocks": clk,
            # our kernels launched in the timed region (the fused selection's event
            # pair spans its four launches per chunk of rows)
            "gpu_launches": n_launch,
            "e2e": e2e, "cpu_baseline": cpu, "peaks": peaks,
        }
        if secondary is not None:
            line["secondary"] = secondary
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
