"""Seeded synthetic inputs for the DSA forward (decode, paged decode, prefill).

This module only draws random numbers and stores them in the input formats the
path consumes; it holds none of the method's arithmetic. The E4M3 key codes are
produced with PyTorch's own float8 conversion (the keys arrive already
quantized, one fp32 scale per token, as the 128-d FP8 indexer key cache of
"DeepSeek-V3.2开源技术报告", DSA principle section, describes).

Every generator is deterministic for a given (seed, device): it uses a private
``torch.Generator`` and draws tensors in a fixed order.

Shapes (production dims; ``dims`` overrides them):
  q_idx   [T, H^I, d_I]  bf16     indexer queries
  w       [T, H^I]       fp32     indexer head weights
  k_idx   [B, ctx, d_I]  uint8    E4M3 key codes (paged: [P, page, d_I])
  k_scale [B, ctx]       fp32     per-token key scale (paged: [P, page])
  q       [T, H, D]      bf16     absorbed MLA queries (D = 512 latent + 64 rope)
  kv      [B, ctx, D]    bf16     latent cache (paged: [P, page, D])
  seqlens [B]            int32    visible tokens per sequence (incl. the queries)
  block_table [B, max_pages] int32 (paged only)
Query row t belongs to sequence t // q_per_seq and sits at position
seqlen - q_per_seq + t % q_per_seq; in a ragged batch (``q_start``) sequence b owns
rows q_start[b] .. q_start[b+1]-1, its last q_start[b+1] - q_start[b] tokens.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

E4M3_MAX = 448.0


@dataclasses.dataclass
class Dims:
    h_idx: int = 64      # H^I indexer heads
    d_idx: int = 128     # d_I indexer head dim
    heads: int = 128     # H query heads
    d_qk: int = 576      # latent key dim (512 latent + 64 rope)
    d_v: int = 512       # value dim (first d_v dims of the latent)
    topk: int = 2048     # k


PRODUCTION = Dims()
TINY = Dims(h_idx=4, d_idx=32, heads=8, d_qk=80, d_v=64, topk=32)


@dataclasses.dataclass
class Problem:
    dims: Dims
    batch: int
    q_per_seq: int
    max_ctx: int
    q_idx: torch.Tensor
    w: torch.Tensor
    k_idx: torch.Tensor
    k_scale: Optional[torch.Tensor]
    q: torch.Tensor
    kv: torch.Tensor
    seqlens: torch.Tensor
    scale: float
    fp8: bool = True
    paged: bool = False
    page_size: int = 64
    block_table: Optional[torch.Tensor] = None
    hot: Optional[torch.Tensor] = None
    name: str = ""
    # ragged batch: int32 [batch + 1] row offsets (sequence b owns query rows
    # q_start[b] .. q_start[b+1]-1, its last tokens); q_per_seq is then the largest count
    q_start: Optional[torch.Tensor] = None

    @property
    def num_q(self) -> int:
        if self.q_start is not None:
            return int(self.q_start[-1])
        return self.batch * self.q_per_seq

    def q_lens(self) -> torch.Tensor:
        if self.q_start is not None:
            qs = self.q_start.cpu().long()
            return qs[1:] - qs[:-1]
        return torch.full((self.batch,), self.q_per_seq, dtype=torch.int64)

    def q_seq(self) -> torch.Tensor:
        return torch.repeat_interleave(torch.arange(self.batch), self.q_lens()).int()

    def q_pos(self) -> torch.Tensor:
        lens = self.q_lens()
        b = torch.repeat_interleave(torch.arange(self.batch), lens)
        first = torch.cumsum(lens, 0) - lens  # the sequence's first row
        i = torch.arange(int(lens.sum())) - first[b]
        return (self.seqlens.cpu().long()[b] - lens[b] + i).int()

    def to(self, device) -> "Problem":
        def mv(x):
            return None if x is None else x.to(device)
        return dataclasses.replace(
            self, q_idx=mv(self.q_idx), w=mv(self.w), k_idx=mv(self.k_idx),
            k_scale=mv(self.k_scale), q=mv(self.q), kv=mv(self.kv), seqlens=mv(self.seqlens),
            block_table=mv(self.block_table), hot=mv(self.hot), q_start=mv(self.q_start))


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal(shape, g, device, std=1.0) -> torch.Tensor:
    return torch.randn(*shape, generator=g, device=device, dtype=torch.float32) * std


def _uniform(shape, g, device, lo=0.0, hi=1.0) -> torch.Tensor:
    return torch.rand(*shape, generator=g, device=device, dtype=torch.float32) * (hi - lo) + lo


def _fp8_keys(rows: int, d: int, g, device, chunk: int = 1 << 20):
    """k ~ N(0,1); per-token scale s = amax/448; codes = E4M3(k / s) (library cast)."""
    codes = torch.empty(rows, d, dtype=torch.uint8, device=device)
    scale = torch.empty(rows, dtype=torch.float32, device=device)
    for r0 in range(0, rows, chunk):
        r1 = min(rows, r0 + chunk)
        k = _normal((r1 - r0, d), g, device)
        s = k.abs().amax(dim=1) / E4M3_MAX
        codes[r0:r1] = (k / s[:, None]).to(torch.float8_e4m3fn).view(torch.uint8)
        scale[r0:r1] = s
    return codes, scale


def _bf16(shape, g, device, std=1.0, chunk_rows: int = 1 << 14) -> torch.Tensor:
    out = torch.empty(*shape, dtype=torch.bfloat16, device=device)
    flat = out.view(shape[0], -1)
    for r0 in range(0, shape[0], chunk_rows):
        r1 = min(shape[0], r0 + chunk_rows)
        flat[r0:r1] = (_normal((r1 - r0, flat.shape[1]), g, device) * std).to(torch.bfloat16)
    return out


def decode(batch=64, ctx=32768, q_per_seq=1, seed=1, dims=PRODUCTION, device="cpu",
           latent_std=0.5, w_div=8.0) -> Problem:
    """Batched decode on a contiguous cache: every sequence holds ``ctx`` tokens
    and its ``q_per_seq`` queries are its last tokens."""
    g = _gen(seed, device)
    T = batch * q_per_seq
    q_idx = _bf16((T, dims.h_idx, dims.d_idx), g, device)
    w = _uniform((T, dims.h_idx), g, device) / w_div
    k_idx, k_scale = _fp8_keys(batch * ctx, dims.d_idx, g, device)
    q = _bf16((T, dims.heads, dims.d_qk), g, device)
    kv = _bf16((batch * ctx, dims.d_qk), g, device, std=latent_std)
    return Problem(dims=dims, batch=batch, q_per_seq=q_per_seq, max_ctx=ctx,
                   q_idx=q_idx, w=w, k_idx=k_idx.view(batch, ctx, dims.d_idx),
                   k_scale=k_scale.view(batch, ctx), q=q, kv=kv.view(batch, ctx, dims.d_qk),
                   seqlens=torch.full((batch,), ctx, dtype=torch.int32, device=device),
                   scale=dims.d_qk ** -0.5, name=f"decode_b{batch}_ctx{ctx}_tq{q_per_seq}")


def prefill(L=8192, seed=2, dims=PRODUCTION, device="cpu", latent_std=0.5, w_div=8.0,
            n_hot=0, hot_factor=4.0) -> Problem:
    """Causal prefill of one sequence of L tokens (query row i at position i).

    With ``n_hot`` > 0, that many key positions (uniform without replacement)
    get their indexer key scaled by ``hot_factor`` (stored as a scaled per-token
    key scale; the E4M3 codes are unchanged)."""
    p = decode(batch=1, ctx=L, q_per_seq=L, seed=seed, dims=dims, device=device,
               latent_std=latent_std, w_div=w_div)
    p.name = f"prefill_L{L}"
    if n_hot:
        g = _gen(seed + 1000, device)
        hot = torch.randperm(L, generator=g, device=device)[:n_hot].sort().values
        p.k_scale[0, hot] *= hot_factor
        p.hot = hot.to(torch.int32)
        p.name += f"_hot{n_hot}"
    return p


def paged_decode(batch=128, q_per_seq=2, min_ctx=4096, max_ctx=131072, page_size=64,
                 seed=4, dims=PRODUCTION, device="cpu", latent_std=1.0, w_div=8.0) -> Problem:
    """Variable-length decode on a paged cache: seqlens ~ U{min_ctx..max_ctx},
    pages of ``page_size`` tokens, block table = a random permutation of the
    physical pages."""
    g = _gen(seed, device)
    seqlens = torch.randint(min_ctx, max_ctx + 1, (batch,), generator=g, device=device,
                            dtype=torch.int64)
    pages_per_seq = (seqlens + page_size - 1) // page_size
    num_pages = int(pages_per_seq.sum().item())
    max_pages = (max_ctx + page_size - 1) // page_size
    perm = torch.randperm(num_pages, generator=g, device=device).to(torch.int32)
    block_table = torch.full((batch, max_pages), -1, dtype=torch.int32, device=device)
    off = 0
    for b, n in enumerate(pages_per_seq.tolist()):
        block_table[b, :n] = perm[off:off + n]
        off += n
    T = batch * q_per_seq
    q_idx = _bf16((T, dims.h_idx, dims.d_idx), g, device)
    w = _uniform((T, dims.h_idx), g, device) / w_div
    k_idx, k_scale = _fp8_keys(num_pages * page_size, dims.d_idx, g, device)
    q = _bf16((T, dims.heads, dims.d_qk), g, device)
    kv = _bf16((num_pages * page_size, dims.d_qk), g, device, std=latent_std)
    return Problem(dims=dims, batch=batch, q_per_seq=q_per_seq, max_ctx=max_ctx,
                   q_idx=q_idx, w=w, k_idx=k_idx.view(num_pages, page_size, dims.d_idx),
                   k_scale=k_scale.view(num_pages, page_size), q=q,
                   kv=kv.view(num_pages, page_size, dims.d_qk),
                   seqlens=seqlens.to(torch.int32), scale=dims.d_qk ** -0.5, paged=True,
                   page_size=page_size, block_table=block_table,
                   name=f"paged_b{batch}_tq{q_per_seq}_ctx{min_ctx}-{max_ctx}")


def ragged(seqlens, q_lens, page_size=64, seed=5, dims=PRODUCTION, device="cpu",
           latent_std=1.0, w_div=8.0) -> Problem:
    """A ragged batch on a paged cache: sequence b holds seqlens[b] tokens and its
    query rows are its last q_lens[b] tokens (q_lens[b] = seqlens[b]: a whole prompt;
    fewer: a chunk of prefill appended to tokens already cached, or a decode step).
    Pages are a random permutation of the physical pages; inputs N(0,1) as in the
    paged decode."""
    seqlens = torch.as_tensor(seqlens, dtype=torch.int64)
    q_lens = torch.as_tensor(q_lens, dtype=torch.int64)
    assert len(seqlens) == len(q_lens) and bool((q_lens <= seqlens).all())
    g = _gen(seed, device)
    batch = len(seqlens)
    max_ctx = int(seqlens.max())
    pages_per_seq = (seqlens + page_size - 1) // page_size
    num_pages = int(pages_per_seq.sum())
    max_pages = (max_ctx + page_size - 1) // page_size
    perm = torch.randperm(num_pages, generator=g, device=device).to(torch.int32)
    block_table = torch.full((batch, max_pages), -1, dtype=torch.int32, device=device)
    off = 0
    for b, n in enumerate(pages_per_seq.tolist()):
        block_table[b, :n] = perm[off:off + n]
        off += n
    q_start = torch.zeros(batch + 1, dtype=torch.int32)
    q_start[1:] = torch.cumsum(q_lens, 0).to(torch.int32)
    T = int(q_start[-1])
    q_idx = _bf16((T, dims.h_idx, dims.d_idx), g, device)
    w = _uniform((T, dims.h_idx), g, device) / w_div
    k_idx, k_scale = _fp8_keys(num_pages * page_size, dims.d_idx, g, device)
    q = _bf16((T, dims.heads, dims.d_qk), g, device)
    kv = _bf16((num_pages * page_size, dims.d_qk), g, device, std=latent_std)
    return Problem(dims=dims, batch=batch, q_per_seq=int(q_lens.max()), max_ctx=max_ctx,
                   q_idx=q_idx, w=w, k_idx=k_idx.view(num_pages, page_size, dims.d_idx),
                   k_scale=k_scale.view(num_pages, page_size), q=q,
                   kv=kv.view(num_pages, page_size, dims.d_qk),
                   seqlens=seqlens.to(torch.int32).to(device), scale=dims.d_qk ** -0.5,
                   paged=True, page_size=page_size, block_table=block_table,
                   q_start=q_start.to(device), name=f"ragged_b{batch}")


def tiny(L=256, seed=0, dims=TINY, device="cpu") -> Problem:
    """The small fp32 causal prefill the oracle is exercised on (no FP8):
    q^I, k^I ~ N(0,1) fp32, w ~ U(0,1)/H^I, latents fp32 N(0,1), scale D^-1/2."""
    g = _gen(seed, device)
    q_idx = _normal((L, dims.h_idx, dims.d_idx), g, device)
    w = _uniform((L, dims.h_idx), g, device) / dims.h_idx
    k_idx = _normal((1, L, dims.d_idx), g, device)
    q = _normal((L, dims.heads, dims.d_qk), g, device)
    kv = _normal((1, L, dims.d_qk), g, device)
    return Problem(dims=dims, batch=1, q_per_seq=L, max_ctx=L, q_idx=q_idx, w=w,
                   k_idx=k_idx, k_scale=None, q=q, kv=kv,
                   seqlens=torch.full((1,), L, dtype=torch.int32, device=device),
                   scale=dims.d_qk ** -0.5, fp8=False, name=f"tiny_L{L}")


def sample_rows(T: int, n: int, seed: int, must=()) -> torch.Tensor:
    """n distinct query rows drawn uniformly (seeded), always including ``must``."""
    g = _gen(seed, "cpu")
    must = sorted({int(m) for m in must if 0 <= int(m) < T})
    rest = torch.randperm(T, generator=g)[: max(0, n)].tolist()
    rows = list(dict.fromkeys(must + rest))[: max(n, len(must))]
    return torch.tensor(sorted(rows), dtype=torch.int64)


def pages_needed(seqlens: torch.Tensor, page_size: int) -> int:
    return int(sum(math.ceil(int(s) / page_size) for s in seqlens.tolist()))


@dataclasses.dataclass
class MhaInputs:
    """Extra inputs of MLA's MHA mode for a Problem's query rows and latent cache.

    q_mha [T, H, d_n + d_r] bf16  per-head queries (128 nope dims, then the 64 rope dims)
    w_uk  [H, d_n, d_c]     bf16  key up-projection of each head (d_c = 512 latent dims)
    w_uv  [H, d_hv, d_c]    bf16  value up-projection of each head
    """
    q_mha: torch.Tensor
    w_uk: torch.Tensor
    w_uv: torch.Tensor

    def to(self, device) -> "MhaInputs":
        return MhaInputs(self.q_mha.to(device), self.w_uk.to(device), self.w_uv.to(device))


MHA_NOPE = 128   # nope query/key dims per head
MHA_ROPE = 64    # rope dims (shared key part)
MHA_DV = 128     # value dims per head


def mha_inputs(p: Problem, seed: int, device="cpu") -> MhaInputs:
    """q_mha ~ N(0,1) and random-init up-projections W ~ N(0, 1/d_c), all bf16
    (no trained weights: the kernels' cost and numerics do not depend on them)."""
    g = _gen(seed, device)
    H, d_c = p.dims.heads, p.dims.d_v
    q_mha = _bf16((p.num_q, H, MHA_NOPE + MHA_ROPE), g, device)
    w_uk = _bf16((H, MHA_NOPE, d_c), g, device, std=d_c ** -0.5)
    w_uv = _bf16((H, MHA_DV, d_c), g, device, std=d_c ** -0.5)
    return MhaInputs(q_mha, w_uk, w_uv)
