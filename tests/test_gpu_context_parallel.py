"""Context-parallel decode (reading of the technical report, serving section,
Figures 16-17) on one GPU: the ranks are played one after another by this
process, and the exchanges are stacks of their tensors.  Each rank holds a
contiguous slice of every sequence's positions (index keys and latent caches)
and runs the library's steps: indexer + top-k on its own positions, export of
(score, global position) candidates, merge into the global selection, attention
over its own selected rows (fp32 partials), log-sum-exp combine.

Checked against the single-GPU path and the oracle:
  * every rank's merged selection is bit-exact the top-k of the full rows (the
    scores of a position do not depend on the sharding), and equals the
    oracle's topk_merge of the exported candidates;
  * the combined output and lse match the oracle's attention over that selection
    within the attention tolerances, for a RoPE and a NoPE layer.
"""

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_16_b200 import context_parallel as cp
from sparse_attention_16_b200 import ops
from sparse_attention_16_b200.workloads import make_workload, small_case, to_numpy
from tests import parity_util as pu

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    ops.load_library()
    yield
    assert ops.check_errors() == 0


def _shard(wl, rank, world, max_len):
    """Rank `rank`'s slice [lo, hi) of every sequence (the same split for all)."""
    lo, hi = cp.shard_range(max_len, rank, world)
    starts = to_numpy(wl.seq_row_start)
    lens = [int(x) + 1 for x in to_numpy(wl.q_pos)]   # decode: the query sits at the last position
    rows, seq_start = [], []
    at = 0
    for b, L in enumerate(lens):
        a, e = min(lo, L), min(hi, L)
        seq_start.append(at)
        rows.append(torch.arange(int(starts[b]) + a, int(starts[b]) + e, device=DEV))
        at += e - a
    rows = torch.cat(rows) if at else torch.zeros(1, dtype=torch.int64, device=DEV)
    # at least one row so that the buffers are never empty
    k_idx = wl.k_idx.index_select(0, rows)
    caches = [L.cache.index_select(0, rows) for L in wl.layers]
    return cp.RankShard(rank=rank, world=world, lo=lo, hi=hi,
                        seq_row_start=torch.tensor(seq_start, dtype=torch.int64, device=DEV), q_seq=wl.q_seq,
                        q_pos=wl.q_pos, k_idx=k_idx, caches=caches)


@pytest.mark.parametrize("world", [2, 4, 8])
def test_context_parallel_decode_matches_the_single_gpu_path(world):
    lengths = (20_000, 9_000, 3_000, 1_500)
    case = small_case("cp_gpu", lengths, layers=(64, 0), seed=71 + world)
    wl = make_workload(case, DEV)
    T, k = wl.T, 2048
    shards = [_shard(wl, r, world, max(lengths)) for r in range(world)]
    # phase 1: local selection on every rank, then the exchange
    cands = [cp.select_local(sh, wl.q_idx, wl.w, k) for sh in shards]
    all_score = cp.stack_exchange([c[0] for c in cands])
    all_pos = cp.stack_exchange([c[1] for c in cands])
    # phase 2: merge + local attention on every rank, then the exchange
    layers = [dict(q_nope=L.q_nope, q_pe=L.q_pe, qmul=L.qmul, d_rope=L.d_rope) for L in wl.layers]
    parts = [cp.attend_local(sh, all_score, all_pos, layers, k) for sh in shards]
    out, lse = cp.combine(cp.stack_exchange([p[2] for p in parts]), cp.stack_exchange([p[3] for p in parts]))
    torch.cuda.synchronize()
    assert ops.check_errors() == 0

    # the selection: every rank agrees, equals the full-row top-k bit for bit ...
    full_scores = pu.gpu_scores(wl)
    idx_full, cnt_full = pu.gpu_topk(full_scores, wl.q_pos, k)
    for p in parts:
        assert torch.equal(p[0], idx_full) and torch.equal(p[1], cnt_full)
    # ... and the oracle's merge of the exported candidates
    s_np = to_numpy(all_score).astype(np.float64)
    p_np = to_numpy(all_pos).astype(np.int64)
    idx_h, cnt_h = to_numpy(idx_full), to_numpy(cnt_full)
    for t in range(T):
        want = oracle.topk_merge(s_np[:, t].reshape(-1), p_np[:, t].reshape(-1), k)
        assert idx_h[t, :cnt_h[t]].tolist() == want.tolist()
    # the combined attention against the oracle on that selection
    for i, L in enumerate(wl.layers):
        ref_o, ref_l = pu.oracle_attend(wl, L, list(range(T)), idx_h, cnt_h)
        pu.assert_attention_close(to_numpy(out[i]), to_numpy(lse[i]), ref_o, ref_l)


def test_context_parallel_decode_over_fp8_latent_caches():
    # The same sharded decode with every rank's latent caches kept as FP8 rows:
    # the combined output matches the oracle's FP8 attention over the merged
    # selection (the global rows, decoded from the same bytes).
    from sparse_attention_16_b200.workloads import quantize_latent_fp8

    world = 2
    lengths = (20_000, 9_000, 3_000, 1_500)
    case = small_case("cp_gpu_fp8", lengths, layers=(64, 0), seed=81)
    wl = make_workload(case, DEV)
    T, k = wl.T, 2048
    full8 = [quantize_latent_fp8(L.cache, L.d_rope) for L in wl.layers]
    for L, c8 in zip(wl.layers, full8):
        L.cache = c8   # the shards take their rows of the FP8 caches
    shards = [_shard(wl, r, world, max(lengths)) for r in range(world)]
    cands = [cp.select_local(sh, wl.q_idx, wl.w, k) for sh in shards]
    all_score = cp.stack_exchange([c[0] for c in cands])
    all_pos = cp.stack_exchange([c[1] for c in cands])
    layers = [dict(q_nope=L.q_nope, q_pe=L.q_pe, qmul=L.qmul, d_rope=L.d_rope) for L in wl.layers]
    parts = [cp.attend_local(sh, all_score, all_pos, layers, k) for sh in shards]
    out, lse = cp.combine(cp.stack_exchange([p[2] for p in parts]), cp.stack_exchange([p[3] for p in parts]))
    torch.cuda.synchronize()
    assert ops.check_errors() == 0
    idx_h, cnt_h = to_numpy(parts[0][0]), to_numpy(parts[0][1])
    starts, q_seq, _ = pu.host_meta(wl)
    for i, L in enumerate(wl.layers):
        c8 = full8[i].cpu().numpy()
        for t in range(T):
            sel = idx_h[t, :cnt_h[t]]
            o_ref, l_ref = oracle.sparse_mla_fp8(to_numpy(L.q_nope[t:t + 1]),
                                                 to_numpy(L.q_pe[t:t + 1]) if L.q_pe is not None else None,
                                                 to_numpy(L.qmul[t:t + 1]), pu.SOFTMAX_SCALE,
                                                 c8[int(starts[q_seq[t]]) + sel], L.d_rope, np.array([0]),
                                                 np.array([0]), np.arange(len(sel), dtype=np.int32)[None, :],
                                                 np.array([len(sel)]))
            pu.assert_attention_close(to_numpy(out[i][t:t + 1]), to_numpy(lse[i][t:t + 1]), o_ref, l_ref)
