"""Context-parallel causal prefill over several GPUs ("DeepSeek-V3.2开源技术报告",
nsmao.com, DSA principle section: the indexer and sparse attention are deployed
with context parallelism across GPUs for long sequences).

Each rank owns a contiguous shard of the sequence's tokens, i.e. of its two
per-token caches (the 128-d FP8 indexer keys with their scales and the 576-d
latents). The one exchange step is an all-gather of those caches over
NCCL (NVLink / NVSwitch on a B200 node); after it every rank holds the whole
causal context and runs the unchanged single-GPU path (indexer -> top-k ->
sparse MLA, or the MHA mode) on its own query rows, which stay sharded.

Query rows are split "zigzag": the L rows form 2N chunks and rank r takes chunks
r and 2N - 1 - r, so every rank gets the same number of causal (row, key) pairs
up to one chunk's rounding (row i sees i + 1 keys).

The compute step is a callable, so this module holds only the partition and the
collective; the library's own calls (dsa_forward over row windows) are the
product path. ``cache_shard`` and ``allgather_cache`` work with any
torch.distributed backend (NCCL on GPUs, gloo for host-side checks).
"""

from __future__ import annotations

from typing import Callable, List, Sequence, Tuple

import torch

CHUNK_ALIGN = 128  # row chunks are multiples of the kernels' 128-row / 128-key tiles


def token_shard(L: int, world: int, rank: int) -> Tuple[int, int]:
    """[begin, end) of the tokens whose caches rank ``rank`` owns: contiguous,
    multiples of 128 except the last shard (which takes the remainder)."""
    per = -(-L // world)
    per = -(-per // CHUNK_ALIGN) * CHUNK_ALIGN
    b = min(L, rank * per)
    return b, min(L, b + per)


def zigzag_windows(L: int, world: int, rank: int) -> List[Tuple[int, int]]:
    """Row windows (row_begin, row_count) of rank ``rank``: chunks r and 2N-1-r of
    the 2N equal chunks of [0, L) (chunk boundaries rounded to 128 rows; empty
    windows dropped, adjacent ones merged)."""
    n = 2 * world
    edges = [min(L, -(-(L * c // n) // CHUNK_ALIGN) * CHUNK_ALIGN) for c in range(n)] + [L]
    wins = []
    for c in sorted({rank, n - 1 - rank}):
        b, e = edges[c], edges[c + 1]
        if e > b:
            if wins and wins[-1][0] + wins[-1][1] == b:
                wins[-1] = (wins[-1][0], wins[-1][1] + e - b)
            else:
                wins.append((b, e - b))
    return wins


def causal_pairs(windows: Sequence[Tuple[int, int]]) -> int:
    """(row, key) pairs of causal attention over the given row windows."""
    return sum((b + 1 + b + c) * c // 2 for b, c in windows)


def allgather_cache(shard: torch.Tensor, L: int, world: int, group=None) -> torch.Tensor:
    """The whole per-token cache [L, ...] from every rank's token shard (the ranks'
    shards of ``token_shard``). Shards are padded to one size for the collective
    and the padding is dropped afterwards."""
    import torch.distributed as dist
    per = token_shard(L, world, 0)[1]
    pad = torch.zeros((per,) + tuple(shard.shape[1:]), dtype=shard.dtype, device=shard.device)
    pad[: shard.shape[0]] = shard
    if world == 1:
        return pad[:L].clone()
    if dist.get_backend(group) == "nccl":
        full = torch.empty((world * per,) + tuple(shard.shape[1:]), dtype=shard.dtype,
                           device=shard.device)
        dist.all_gather_into_tensor(full, pad, group=group)
    else:
        parts = [torch.empty_like(pad) for _ in range(world)]
        dist.all_gather(parts, pad, group=group)
        full = torch.cat(parts)
    return full[:L]


def cp_prefill(L: int, world: int, rank: int, shards: dict, compute: Callable, group=None):
    """Gather the caches, then run ``compute(caches, windows)`` on this rank's
    zigzag rows. ``shards`` maps cache names to this rank's token-shard tensors
    (first dim = tokens); returns (windows, compute's result)."""
    caches = {name: allgather_cache(t, L, world, group) for name, t in shards.items()}
    wins = zigzag_windows(L, world, rank)
    return wins, compute(caches, wins)
