"""Multi-rank bookkeeping on CPU with the gloo backend (world size 2): sequence
sharding, the max-over-ranks time, the job-wide throughput, and that running the
path rank by rank on disjoint sequences reproduces the single-process result
(checked with the CPU oracle, so no GPU is needed)."""

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
    mgr = mp.Manager()
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
