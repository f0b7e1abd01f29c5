"""Multi-rank bookkeeping on CPU with the gloo backend (world size 2): sequence
sharding, the max-over-ranks time, the job-wide throughput, and that running the
path rank by rank on disjoint sequences reproduces the single-process result
(checked with the CPU oracle, so no GPU is needed).  Also the context-parallel
exchange for one long sequence (per-rank selection, candidate all-gather and
merge, per-rank attention, output combine), computed with the oracle: the
decomposition a context-parallel decode must reproduce."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_attention_16_b200 import replicas


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from sparse_attention_16_b200.workloads import SOFTMAX_SCALE, make_workload, small_case, to_numpy

        # max over ranks
        t = replicas.max_over_ranks(0.5 + rank)
        # the same batch on every rank; each rank processes only its own sequences
        case = small_case("dist", (700, 300, 1200, 90, 450), layers=(64,), seed=3)
        wl = make_workload(case, "cpu")
        mine = list(replicas.shard_sequences(wl.T, rank, world))
        lay = wl.layers[0]
        starts = to_numpy(wl.seq_row_start)
        res = {}
        for q in mine:   # decode: query q belongs to sequence q
            b0, n = int(starts[q]), int(to_numpy(wl.q_pos)[q]) + 1
            layers = [dict(q_nope=to_numpy(lay.q_nope[q:q + 1]), q_pe=to_numpy(lay.q_pe[q:q + 1]),
                           qmul=to_numpy(lay.qmul[q:q + 1]), cache=to_numpy(lay.cache[b0:b0 + n]), d_rope=64)]
            _, _, outs = oracle.forward(to_numpy(wl.q_idx[q:q + 1]), to_numpy(wl.w[q:q + 1]),
                                        to_numpy(wl.k_idx[b0:b0 + n]), np.array([0]), np.array([0]),
                                        np.array([n - 1]), layers, SOFTMAX_SCALE, k=256)
            res[q] = outs[0][0][0]
        gathered = [None] * world
        dist.all_gather_object(gathered, res)
        out[rank] = {"max": t, "mine": mine, "all": {k: v for g in gathered for k, v in g.items()}}
    finally:
        dist.destroy_process_group()


def test_replicas_world_size_2():
    import oracle
    from sparse_attention_16_b200.workloads import SOFTMAX_SCALE, make_workload, small_case, to_numpy

    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    r0, r1 = out[0], out[1]
    assert r0["max"] == r1["max"] == 1.5
    assert sorted(r0["mine"] + r1["mine"]) == list(range(5)) and not set(r0["mine"]) & set(r1["mine"])
    # single-process result over the whole batch
    wl = make_workload(small_case("dist", (700, 300, 1200, 90, 450), layers=(64,), seed=3), "cpu")
    lay = wl.layers[0]
    layers = [dict(q_nope=to_numpy(lay.q_nope), q_pe=to_numpy(lay.q_pe), qmul=to_numpy(lay.qmul),
                   cache=to_numpy(lay.cache), d_rope=64)]
    _, _, outs = oracle.forward(to_numpy(wl.q_idx), to_numpy(wl.w), to_numpy(wl.k_idx),
                                to_numpy(wl.seq_row_start), to_numpy(wl.q_seq), to_numpy(wl.q_pos), layers,
                                SOFTMAX_SCALE, k=256)
    for q in range(5):
        np.testing.assert_allclose(r0["all"][q], outs[0][0][q], rtol=1e-12, atol=1e-14)


def _cp_worker(rank, world, port, out):
    # Context-parallel decode of one long sequence (the exchange the technical report's
    # serving section describes): each rank scores and selects among its own positions,
    # the candidates are all-gathered and merged, each rank attends over the selected rows
    # it owns, and the partial outputs are all-gathered and combined.
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from sparse_attention_16_b200.workloads import SOFTMAX_SCALE, make_workload, small_case, to_numpy

        from sparse_attention_16_b200 import context_parallel as cp

        k = 256
        wl = make_workload(small_case("cp", (5000,), layers=(64,), seed=4), "cpu")
        lay = wl.layers[0]
        lo, hi = cp.shard_range(5000, rank, world)
        qp = int(cp.local_q_pos(wl.q_pos, lo, hi)[0])      # the query sits at 4999: the shard's last position
        assert qp == hi - lo - 1
        exchange = cp.dist_exchange()
        keys = to_numpy(wl.k_idx[lo:hi])
        s = oracle.index_scores(to_numpy(wl.q_idx), to_numpy(wl.w), keys, np.array([0]), np.array([0]),
                                np.array([qp]), hi - lo)
        sel, cnt = oracle.topk_select(s, np.array([qp]), k)
        pos = np.full(k, -1, np.int64)
        sc = np.full(k, -np.inf)
        pos[:cnt[0]] = sel[0, :cnt[0]] + lo
        sc[:cnt[0]] = s[0, sel[0, :cnt[0]]]
        all_pos = exchange(torch.from_numpy(pos))
        all_sc = exchange(torch.from_numpy(sc))
        assert tuple(all_pos.shape) == (world, k)
        chosen = oracle.topk_merge(all_sc.reshape(-1).numpy(), all_pos.reshape(-1).numpy(), k)
        mine = chosen[(chosen >= lo) & (chosen < hi)] - lo
        idx = np.full((1, 2048), -1, np.int32)
        idx[0, :mine.size] = mine
        o, lse = oracle.sparse_mla(to_numpy(lay.q_nope), to_numpy(lay.q_pe), to_numpy(lay.qmul), SOFTMAX_SCALE,
                                   to_numpy(lay.cache[lo:hi]), 64, np.array([0]), np.array([0]), idx,
                                   np.array([mine.size]))
        all_o = exchange(torch.from_numpy(o[0]))
        all_l = exchange(torch.from_numpy(lse[0]))
        oc, lc = oracle.lse_combine(all_o.numpy(), all_l.numpy())
        out[rank] = {"chosen": chosen.tolist(), "o": oc, "lse": lc}
    finally:
        dist.destroy_process_group()


def test_context_parallel_exchange_world_size_2():
    import oracle
    from sparse_attention_16_b200.workloads import SOFTMAX_SCALE, make_workload, small_case, to_numpy

    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_cp_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    wl = make_workload(small_case("cp", (5000,), layers=(64,), seed=4), "cpu")
    lay = wl.layers[0]
    s = oracle.index_scores(to_numpy(wl.q_idx), to_numpy(wl.w), to_numpy(wl.k_idx), np.array([0]), np.array([0]),
                            np.array([4999]), 5000)
    idx, cnt = oracle.topk_select(s, np.array([4999]), 256)
    o, lse = oracle.sparse_mla(to_numpy(lay.q_nope), to_numpy(lay.q_pe), to_numpy(lay.qmul), SOFTMAX_SCALE,
                               to_numpy(lay.cache), 64, np.array([0]), np.array([0]), idx, cnt)
    for r in range(world):
        assert out[r]["chosen"] == idx[0, :cnt[0]].tolist()
        np.testing.assert_allclose(out[r]["o"], o[0], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(out[r]["lse"], lse[0], rtol=1e-12)


def test_context_parallel_shards_cover_the_sequence_in_order():
    from sparse_attention_16_b200 import context_parallel as cp

    for length in (1, 127, 128, 5000, 1 << 20):
        for world in (1, 2, 3, 8):
            parts = [cp.shard_range(length, r, world) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == length
            for (a, b), (c, d) in zip(parts, parts[1:]):
                assert b == c and a <= b
            assert all(lo % 128 == 0 for lo, _ in parts)
    q_pos = torch.tensor([0, 99, 100, 250, 5000], dtype=torch.int32)
    assert cp.local_q_pos(q_pos, 100, 200).tolist() == [-1, -1, 0, 99, 99]


def test_shards_cover_and_balance():
    for n in (1, 5, 64, 65):
        for world in (1, 2, 3, 8):
            parts = [replicas.shard_sequences(n, r, world) for r in range(world)]
            flat = [i for p in parts for i in p]
            assert flat == list(range(n))
            assert max(len(p) for p in parts) - min(len(p) for p in parts) <= 1


def test_job_throughput_counts_all_ranks():
    assert replicas.job_throughput(64, 4, 10, 2.0) == 64 * 4 * 10 / 2.0
    assert replicas.max_over_ranks(0.25) == 0.25      # no process group: own time
