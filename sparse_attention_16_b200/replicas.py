"""Data-parallel bookkeeping for running the hot path on several GPUs.

Decode batches shard by sequence: every rank owns whole sequences (their
index keys and latent caches live on that rank's GPU) and runs the same path
with no exchange on the data path.  What needs coordination is only the
bookkeeping: which sequences a rank owns, a common start for the timed region,
and the job-wide time (the slowest rank's device time).
"""

from __future__ import annotations

import torch
import torch.distributed as dist


def shard_sequences(n_seqs: int, rank: int, world: int) -> range:
    """Contiguous block of sequences owned by ``rank`` (sizes differ by at most one)."""
    lo = n_seqs * rank // world
    hi = n_seqs * (rank + 1) // world
    return range(lo, hi)


def rank_seed(seed: int, rank: int) -> int:
    """Seed of the independent batch a rank draws when every rank runs a full batch."""
    return seed + 1000 * rank


def max_over_ranks(seconds: float, device=None) -> float:
    """Job-wide time of a timed region: the maximum of the ranks' device times."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(seconds)
    t = torch.tensor([seconds], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, world: int, steps: int, seconds: float) -> float:
    """Units processed by all ranks per second of the slowest rank."""
    return units_per_rank * world * steps / seconds
