"""Row sharding of the codec across ranks (one process per GPU).

Tiles are independent, so a matrix splits into contiguous row blocks, one per
rank, each encoded into a self-contained stream (offsets start at 0) with no
communication.  Decoding a shard needs only that shard.  When one global
stream is wanted, the only exchange is an all-gather of each rank's payload
word count: rank r then adds the words of ranks < r to its offsets and its
payload lands at that base.  Signs depend only on the column tile, so for
weights a shard's stream equals the matching slice of a single-call stream
bit for bit.  The KV dither is drawn per tile index within a call, so a KV
shard carries its own dither realisation (decode it with the same shard
shape); its statistics are unchanged.

Host logic only (torch.distributed, any backend); the per-rank encode itself
is the library call.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def row_range(rows: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous, balanced row block [r0, r1) of `rank` (earlier ranks get the
    extra rows)."""
    base, extra = divmod(rows, world)
    r0 = rank * base + min(rank, extra)
    return r0, r0 + base + (1 if rank < extra else 0)


def global_word_base(local_words: int, group=None) -> tuple[int, int]:
    """All-gather the ranks' payload word counts; return (this rank's base,
    total words of the global stream)."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    t = torch.tensor([local_words], dtype=torch.int64)
    if dist.get_backend(group) == "nccl":
        t = t.cuda()
    out = [torch.zeros_like(t) for _ in range(world)]
    dist.all_gather(out, t, group=group)
    counts = [int(x.item()) for x in out]
    return sum(counts[:rank]), sum(counts)


def rebase_offsets(tile_off: torch.Tensor, base: int, last_rank: bool) -> torch.Tensor:
    """A shard's offsets (ntiles_local + 1, starting at 0) shifted to the global
    stream; every rank but the last drops its end offset, which the next rank's
    first offset repeats."""
    off = (tile_off.to(torch.int64) & 0xFFFFFFFF) + base
    if off.max().item() >= 1 << 32:
        raise OverflowError("global stream exceeds 2^32 payload words")
    return off if last_rank else off[:-1]
