"""Data-parallel layout of the hot path over ranks (one process per GPU).

Every prompt's planes depend only on that prompt's ids, and every token's
rotation only on its own planes, so the path shards by whole prompts with no
data-path collective.  Two layouts:

* weak scaling (the benchmark's): each rank owns a full batch of its own,
  seeded by rank;
* strong scaling: one packed batch split into contiguous runs of whole prompts
  with balanced token counts (a prompt is never split, so no rank needs another
  rank's image-marker index).

The only cross-rank step is timing: the slowest rank's time (max over ranks).
"""
from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Shard:
    seq_lo: int   # first prompt of this rank
    seq_hi: int   # one past the last prompt
    tok_lo: int   # first packed token
    tok_hi: int   # one past the last packed token

    @property
    def n_tokens(self) -> int:
        return self.tok_hi - self.tok_lo


def shard_sequences(cu_seqlens, world: int, rank: int) -> Shard:
    """Contiguous prompts [seq_lo, seq_hi) for `rank`: prompt b goes to the rank
    whose equal share of the token range holds the prompt's midpoint."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    n = int(cu[-1])
    mid2 = cu[:-1] + cu[1:]  # twice each prompt's midpoint
    owner = np.minimum((mid2 * world) // max(2 * n, 1), world - 1) if n else \
        np.minimum(np.arange(len(mid2)) * world // max(len(mid2), 1), world - 1)
    idx = np.flatnonzero(owner == rank)
    if idx.size == 0:
        # empty shard, placed after the prompts of lower ranks
        lo = int(np.searchsorted(owner, rank, side="left"))
        return Shard(lo, lo, int(cu[lo]), int(cu[lo]))
    lo, hi = int(idx[0]), int(idx[-1]) + 1
    return Shard(lo, hi, int(cu[lo]), int(cu[hi]))


def local_batch(ids, cu_seqlens, shard: Shard):
    """The rank's ids and cu_seqlens, rebased to start at 0."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    local_cu = (cu[shard.seq_lo:shard.seq_hi + 1] - shard.tok_lo).astype(np.int32)
    return np.ascontiguousarray(ids[shard.tok_lo:shard.tok_hi]), local_cu


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of rank's own batch under weak scaling."""
    return base_seed + 1000 * rank


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """The slowest rank's time (a host float); identity without a process group."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
