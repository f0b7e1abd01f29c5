"""Context-parallel decode of long sequences over R ranks (reading of the
technical report, serving section, Figures 16-17: the positions of a sequence
are split over GPUs; each selects among its own positions, the candidates are
exchanged, each attends over the selected rows it holds, and the partial
outputs are combined).

Every step runs in the library's kernels; this module only keeps the
bookkeeping (which positions a rank holds, the shard-local causal bound) and
moves tensors between the steps:

  select_local    indexer over the rank's positions, local top-k, export of
                  (score, global position) candidates            [T, k] each
  exchange        all-gather of the candidates                   [R, T, k]
  attend_local    merge into the global selection (same tie rule), shard-local
                  view of it, attention of every layer over the rank's own
                  selected rows -> fp32 partial outputs and lse
  exchange        all-gather of the partials                     [R, L, T, 64, 512]
  combine         log-sum-exp merge of the partials -> bf16 output and lse

`exchange` is a callable mapping this rank's tensor to the [R, ...] stack of
every rank's: torch.distributed all_gather_into_tensor over NCCL in a
multi-GPU run; a stack of the ranks' tensors when one process plays every
rank (tests and single-GPU timing).
"""

from __future__ import annotations

from dataclasses import dataclass

import torch

from . import ops


def shard_range(length: int, rank: int, world: int) -> tuple[int, int]:
    """Positions [lo, hi) of a sequence of `length` positions held by `rank`
    (contiguous, in rank order, sizes differing by at most one tile of 128)."""
    tiles = (length + 127) // 128
    lo = min(length, (tiles * rank // world) * 128)
    hi = min(length, (tiles * (rank + 1) // world) * 128)
    return lo, hi


def local_q_pos(q_pos: torch.Tensor, lo: int, hi: int) -> torch.Tensor:
    """The causal bound inside a shard: candidates of query t on this rank are
    global positions lo..min(q_pos[t], hi - 1), i.e. local 0..(that - lo); -1
    when the shard lies entirely after the query."""
    return (torch.clamp(q_pos.to(torch.int64), max=hi - 1) - lo).clamp(min=-1).to(torch.int32)


@dataclass
class RankShard:
    """What one rank holds for a decode batch whose every sequence is sharded the
    same way: its positions [lo, hi) of every sequence, rows of sequence b at
    seq_row_start[b] .. + (hi - lo) of its index-key and latent-cache buffers."""

    rank: int
    world: int
    lo: int
    hi: int
    seq_row_start: torch.Tensor   # [B] int64, this rank's buffers
    q_seq: torch.Tensor           # [T] int32
    q_pos: torch.Tensor           # [T] int32, global positions
    k_idx: torch.Tensor           # [rows, 128] bf16 (this rank's positions)
    caches: list                  # per layer: [rows, 512 + d_rope] bf16


def select_local(sh: RankShard, q_idx, w, k=2048, stream=None):
    """Indexer + top-k over this rank's positions, exported as candidates.
    Returns (cand_score f32 [T, k], cand_pos int32 [T, k] global positions)."""
    dev = q_idx.device
    T = q_idx.shape[0]
    ld = max(4, ((sh.hi - sh.lo) + 3) // 4 * 4)
    qp = local_q_pos(sh.q_pos, sh.lo, sh.hi)
    scores = torch.empty((T, ld), dtype=torch.float32, device=dev)
    hist = torch.empty((T, 2048), dtype=torch.int32, device=dev)
    ops.index_scores(q_idx, w, sh.k_idx, sh.seq_row_start, sh.q_seq, qp, scores, hist=hist, stream=stream)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    cnt = torch.empty((T,), dtype=torch.int32, device=dev)
    ops.topk(scores, qp, k, idx, cnt, hist=hist, stream=stream)
    cand_score = torch.empty((T, k), dtype=torch.float32, device=dev)
    cand_pos = torch.empty((T, k), dtype=torch.int32, device=dev)
    ops.topk_export(scores, idx, cnt, sh.lo, cand_score, cand_pos, stream=stream)
    return cand_score, cand_pos


def attend_local(sh: RankShard, all_score, all_pos, layers, k=2048, stream=None):
    """Global selection from every rank's candidates ([R, T, k]), then every
    layer's attention over the selected rows this rank holds.  `layers`: dicts
    with q_nope, q_pe (or None), qmul, d_rope.  Returns (idx_global [T, k],
    count [T], o_parts fp32 [L, T, 64, 512], lse_parts [L, T, 64])."""
    dev = all_pos.device
    T = all_pos.shape[1]
    idx_global = torch.empty((T, k), dtype=torch.int32, device=dev)
    idx_local = torch.empty((T, k), dtype=torch.int32, device=dev)
    count = torch.empty((T,), dtype=torch.int32, device=dev)
    count_local = torch.empty((T,), dtype=torch.int32, device=dev)
    ops.topk_merge(all_score, all_pos, k, count, idx_global=idx_global, idx_local=idx_local,
                   count_local=count_local, shard=(sh.lo, sh.hi), stream=stream)
    n_l = len(layers)
    o_parts = torch.empty((n_l, T, 64, 512), dtype=torch.float32, device=dev)
    lse_parts = torch.empty((n_l, T, 64), dtype=torch.float32, device=dev)
    lay = [dict(q_nope=L["q_nope"], q_pe=L.get("q_pe"), qmul=L["qmul"], cache=c, d_rope=L["d_rope"], out=o_parts[i],
                lse=lse_parts[i]) for i, (L, c) in enumerate(zip(layers, sh.caches))]
    qp = local_q_pos(sh.q_pos, sh.lo, sh.hi)
    ops.sparse_mla_attend_layers(lay, sh.caches[0].shape[0], sh.seq_row_start, sh.q_seq, idx_local, count_local,
                                 q_pos=qp, stream=stream)
    return idx_global, count, o_parts, lse_parts


def combine(all_o, all_lse, stream=None):
    """Per layer: merge the ranks' partials ([R, L, T, 64, 512] and [R, L, T, 64]).
    Returns (out bf16 [L, T, 64, 512], lse [L, T, 64])."""
    R, n_l, T = all_lse.shape[:3]
    out = torch.empty((n_l, T, 64, 512), dtype=torch.bfloat16, device=all_o.device)
    lse = torch.empty((n_l, T, 64), dtype=torch.float32, device=all_o.device)
    for i in range(n_l):
        ops.lse_combine(all_o[:, i].contiguous(), all_lse[:, i].contiguous(), out[i], lse[i], stream=stream)
    return out, lse


def dist_exchange(group=None):
    """The all-gather of a multi-process run: this rank's tensor -> [R, ...] of
    every rank's (one all_gather_into_tensor over NCCL; a list all-gather on
    other backends, e.g. gloo on the CPU)."""
    import torch.distributed as dist

    def gather(t):
        world = dist.get_world_size(group)
        t = t.contiguous()
        out = torch.empty((world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
        if dist.get_backend(group) == "nccl":
            dist.all_gather_into_tensor(out, t, group=group)
        else:
            dist.all_gather(list(out.unbind(0)), t, group=group)
        return out

    return gather


def stack_exchange(per_rank):
    """The exchange when one process plays every rank: the ranks' tensors, stacked."""
    return torch.stack([t.contiguous() for t in per_rank])
