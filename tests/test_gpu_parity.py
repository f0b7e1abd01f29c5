"""GPU parity: every C-ABI call against the fp64 oracle on seeded inputs.

Sizes span several tiles and ragged tails while the oracle still finishes in
seconds; the full-size configurations are checked on sampled queries in
test_gpu_fullsize.py.
"""

import dataclasses
import math

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_16_b200 import ops
from sparse_attention_16_b200.workloads import (CONFIGS, SOFTMAX_SCALE, make_workload, small_case,
                                                to_numpy)
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


# ------------------------------------------------------------------ indexer

INDEX_CASES = [
    small_case("ragged_decode", (4096, 4096, 1500, 37, 129, 128, 1), seed=11),
    small_case("one_long", (20000,), seed=12),
    small_case("many_short", tuple(range(1, 400, 23)), seed=13),
]


@pytest.mark.parametrize("case", INDEX_CASES, ids=lambda c: c.name)
def test_indexer_matches_oracle_decode(case):
    wl = make_workload(case, DEV)
    s = pu.gpu_scores(wl)
    ts = list(range(wl.T))
    ref = pu.oracle_scores(wl, ts, case.ld)
    pu.assert_scores_close(to_numpy(s), ref, to_numpy(wl.q_pos))


@pytest.mark.parametrize("new", [45, 64, 8, 3])
def test_indexer_matches_oracle_prefill_groups(new):
    case = small_case(f"prefill_{new}", kind="prefill", cached=700, new=new, seed=14)
    wl = make_workload(case, DEV)
    for qg in (8, 1):
        s = pu.gpu_scores(wl, q_group=qg)
        ref = pu.oracle_scores(wl, list(range(wl.T)), case.ld)
        pu.assert_scores_close(to_numpy(s), ref, to_numpy(wl.q_pos))


def test_indexer_groups_of_four_queries_of_one_sequence():
    # Several queries of a sequence decoded together (its last 4 positions):
    # scored in groups of 4 per key tile, against the oracle; and the same
    # queries scored one by one.
    case = small_case("mq4", (5000, 3000, 2100, 700, 131), per_seq=4, seed=28)
    wl = make_workload(case, DEV)
    ref = pu.oracle_scores(wl, list(range(wl.T)), case.ld)
    for qg in (4, 1):
        s = pu.gpu_scores(wl, q_group=qg)
        pu.assert_scores_close(to_numpy(s), ref, to_numpy(wl.q_pos))


def test_query_group_mixing_sequences_is_flagged():
    case = small_case("mq_bad", (3000, 3000), per_seq=2, seed=29)   # groups of 4 would span two sequences
    wl = make_workload(case, DEV)
    s = torch.empty((wl.T, case.ld), dtype=torch.float32, device=DEV)
    ops.index_scores(wl.q_idx, wl.w, wl.k_idx, wl.seq_row_start, wl.q_seq, wl.q_pos, s, q_group=4)
    with pytest.raises(ops.DSAError) as e:
        ops.check_errors()
    assert "0x4" in str(e.value)


def test_indexer_integer_inputs_are_bit_exact():
    # Small-integer q, k and dyadic w make every product and partial sum exact in fp32.
    case = small_case("int_exact", (3000, 700, 130), seed=15)
    wl = make_workload(case, DEV)
    g = torch.Generator(device=DEV).manual_seed(5)
    wl.q_idx = torch.randint(-3, 4, wl.q_idx.shape, generator=g, device=DEV).to(torch.bfloat16)
    wl.k_idx = torch.randint(-3, 4, wl.k_idx.shape, generator=g, device=DEV).to(torch.bfloat16)
    wl.w = torch.randint(-8, 9, wl.w.shape, generator=g, device=DEV).float() / 4.0
    s = to_numpy(pu.gpu_scores(wl))
    ref = pu.oracle_scores(wl, list(range(wl.T)), case.ld)
    qp = to_numpy(wl.q_pos)
    for t in range(wl.T):
        n = qp[t] + 1
        np.testing.assert_array_equal(s[t, :n].astype(np.float64), ref[t, :n])


# ------------------------------------------------------------------ top-k

@pytest.mark.parametrize("k", [2048, 1, 7, 4096])
def test_topk_bit_exact_on_gpu_scores(k):
    case = small_case("topk_src", (4096, 9000, 1500, 37, 2049, 2048), seed=16)
    wl = make_workload(case, DEV)
    s = pu.gpu_scores(wl)
    idx, cnt = pu.gpu_topk(s, wl.q_pos, k)
    pu.assert_topk_exact(to_numpy(idx), to_numpy(cnt), to_numpy(s).astype(np.float64),
                         to_numpy(wl.q_pos), k)


@pytest.mark.parametrize("T,ld", [(1, 100_000), (1, 500_000), (200, 40_000), (100, 5_000), (3, 131_072),
                                  (2, 1_000_000)])
def test_topk_cluster_sizes_and_ties(T, ld):
    # Integer-valued scores: heavy ties everywhere, including at the threshold.
    g = torch.Generator(device=DEV).manual_seed(T * 7 + ld)
    scores = torch.randint(-40, 41, (T, ld), generator=g, device=DEV).float()
    scores[:, ::5] = -0.0
    q_pos = torch.randint(ld // 2, ld, (T,), generator=g, device=DEV, dtype=torch.int32)
    q_pos[0] = ld - 1
    idx, cnt = pu.gpu_topk(scores, q_pos, 2048)
    pu.assert_topk_exact(to_numpy(idx), to_numpy(cnt), to_numpy(scores).astype(np.float64),
                         to_numpy(q_pos), 2048)


@pytest.mark.parametrize("T,ld", [(200, 40_000), (2, 1_000_000), (64, 32_768)])
def test_topk_continuous_scores_all_stash_modes(T, ld):
    # Slices of up to 32K keys per CTA stage whole keys, 32K-64K stage their top
    # 16 bits; continuous scores keep the candidate set small (no overflow path).
    g = torch.Generator(device=DEV).manual_seed(T + ld)
    scores = torch.randn((T, ld), generator=g, device=DEV)
    q_pos = torch.randint(ld // 2, ld, (T,), generator=g, device=DEV, dtype=torch.int32)
    q_pos[0] = ld - 1
    idx, cnt = pu.gpu_topk(scores, q_pos, 2048)
    pu.assert_topk_exact(to_numpy(idx), to_numpy(cnt), to_numpy(scores).astype(np.float64),
                         to_numpy(q_pos), 2048)


def test_topk_special_values_and_short_rows():
    ld = 6000
    s = torch.randn((6, ld), device=DEV)
    s[0, :] = 1.0                        # all equal: lowest positions win
    s[1, 100:3000] = float("nan")        # NaN ranks as -inf
    s[2, :] = -0.0
    s[2, ::2] = 0.0                      # signed zeros are equal
    s[3, 500:700] = float("inf")
    q_pos = torch.tensor([5999, 5999, 5999, 5999, 100, -1], dtype=torch.int32, device=DEV)
    idx, cnt = pu.gpu_topk(s, q_pos, 2048)
    pu.assert_topk_exact(to_numpy(idx), to_numpy(cnt), to_numpy(s).astype(np.float64),
                         to_numpy(q_pos), 2048)
    assert to_numpy(cnt).tolist()[-2:] == [101, 0]


# ------------------------------------------------------------------ top-k from the indexer's histogram

def _key_bins(scores_row):
    """Top 11 bits of the order-preserving key of fp32 scores (NaN as -inf, -0 as +0),
    written out from the IEEE-754 bit layout."""
    u = np.asarray(scores_row, dtype=np.float32).view(np.uint32).copy()
    u[(u & 0x7FFFFFFF) > 0x7F800000] = 0xFF800000
    u[u == 0x80000000] = 0
    key = np.where(u & 0x80000000, ~u, u | 0x80000000).astype(np.uint32)
    return key >> 21


def _hist_of(scores, q_pos):
    s = to_numpy(scores)
    qp = to_numpy(q_pos)
    h = np.zeros((s.shape[0], 2048), np.int64)
    for t in range(s.shape[0]):
        n = int(qp[t]) + 1
        if n > 0:
            h[t] = np.bincount(_key_bins(s[t, :n]), minlength=2048)
    return h


# Rows of at most 40,960 scores are selected from one CTA's shared memory, longer ones
# by slices on every SM; the first and last cases take the slices, the others the rows.
HIST_CASES = [
    small_case("hist_ragged", (4096, 40000, 1500, 37, 9000, 2049, 2048, 130000), seed=51),
    small_case("hist_many", (32768,) * 70, seed=52),
    small_case("hist_ragged_rows", (4096, 40960, 1500, 37, 9000, 2049, 2048, 31), seed=53),
    small_case("hist_one_past_rows", (40961, 2050), seed=54),
]


@pytest.mark.parametrize("case", HIST_CASES, ids=lambda c: c.name)
def test_indexer_histogram_counts_its_scores(case):
    wl = make_workload(dataclasses.replace(case, layers=()), DEV)
    scores = torch.empty((wl.T, case.ld), dtype=torch.float32, device=DEV)
    hist = torch.full((wl.T, 2048), 12345, dtype=torch.int32, device=DEV)   # overwritten by the call
    ops.index_scores(wl.q_idx, wl.w, wl.k_idx, wl.seq_row_start, wl.q_seq, wl.q_pos, scores, hist=hist)
    np.testing.assert_array_equal(to_numpy(hist).astype(np.int64), _hist_of(scores, wl.q_pos))


@pytest.mark.parametrize("case", HIST_CASES, ids=lambda c: c.name)
def test_topk_from_the_histogram_is_bit_exact(case):
    wl = make_workload(dataclasses.replace(case, layers=()), DEV)
    scores = torch.empty((wl.T, case.ld), dtype=torch.float32, device=DEV)
    hist = torch.empty((wl.T, 2048), dtype=torch.int32, device=DEV)
    ops.index_scores(wl.q_idx, wl.w, wl.k_idx, wl.seq_row_start, wl.q_seq, wl.q_pos, scores, hist=hist)
    for k in (2048, 7, 4096):
        idx = torch.empty((wl.T, k), dtype=torch.int32, device=DEV)
        cnt = torch.empty((wl.T,), dtype=torch.int32, device=DEV)
        ops.topk(scores, wl.q_pos, k, idx, cnt, hist=hist)
        pu.assert_topk_exact(to_numpy(idx), to_numpy(cnt), to_numpy(scores).astype(np.float64),
                             to_numpy(wl.q_pos), k)
    assert ops.check_errors() == 0


def test_topk_from_the_histogram_one_million_positions():
    case = dataclasses.replace(CONFIGS["decode_b4_1m_4layers"], layers=())
    wl = make_workload(case, DEV)
    scores = torch.empty((wl.T, case.ld), dtype=torch.float32, device=DEV)
    hist = torch.empty((wl.T, 2048), dtype=torch.int32, device=DEV)
    ops.index_scores(wl.q_idx, wl.w, wl.k_idx, wl.seq_row_start, wl.q_seq, wl.q_pos, scores, hist=hist)
    idx, cnt = pu.gpu_topk(scores, wl.q_pos, 2048)
    idx2 = torch.empty_like(idx)
    cnt2 = torch.empty_like(cnt)
    ops.topk(scores, wl.q_pos, 2048, idx2, cnt2, hist=hist)
    assert torch.equal(idx, idx2) and torch.equal(cnt, cnt2)     # both paths agree bit for bit
    s0 = to_numpy(scores[:2]).astype(np.float64)
    pu.assert_topk_exact(to_numpy(idx2[:2]), to_numpy(cnt2[:2]), s0, to_numpy(wl.q_pos[:2]), 2048)


@pytest.mark.parametrize("ld", [300_000, 40_960])
def test_topk_histogram_path_ties_and_foreign_histograms(ld):
    # (a) Integer scores: heavy ties, bins far over the candidate caps -> the
    #     kernels fall back to the whole row; (b) a histogram of other scores, and
    #     one with its bins shifted, must not change the result.  ld 40,960: the
    #     shared-memory row path; 300,000: the slice path.
    g = torch.Generator(device=DEV).manual_seed(77)
    T = 6
    scores = torch.randint(-3, 4, (T, ld), generator=g, device=DEV).float()
    scores[1] = torch.randn((ld,), generator=g, device=DEV)
    scores[2, :] = 1.0
    q_pos = torch.tensor([ld - 1, ld - 1, min(99_999, ld // 2), 5000, 2047, ld - 1], dtype=torch.int32,
                         device=DEV)
    true_hist = torch.as_tensor(_hist_of(scores, q_pos), dtype=torch.int32, device=DEV)
    other = torch.as_tensor(_hist_of(torch.randn((T, ld), generator=g, device=DEV), q_pos), dtype=torch.int32,
                            device=DEV)
    shifted = torch.roll(true_hist, 3, dims=1)
    for h in (true_hist, other, shifted):
        idx = torch.empty((T, 2048), dtype=torch.int32, device=DEV)
        cnt = torch.empty((T,), dtype=torch.int32, device=DEV)
        ops.topk(scores, q_pos, 2048, idx, cnt, hist=h)
        pu.assert_topk_exact(to_numpy(idx), to_numpy(cnt), to_numpy(scores).astype(np.float64), to_numpy(q_pos), 2048)
    assert ops.check_errors() == 0


@pytest.mark.parametrize("ld", [6_000, 300_000])
def test_topk_histogram_path_special_values(ld):
    # The histogram paths decide "at or above the k-th bin" by a float
    # comparison against the bin's first value; rows whose k-th bin holds NaN
    # (ranked as -inf), +-inf, signed zeros or values on a bin boundary.
    # ld 6,000: the shared-memory row kernel; 300,000: the slice filter + select.
    g = torch.Generator(device=DEV).manual_seed(ld + 5)
    T = 7
    s = torch.randn((T, ld), generator=g, device=DEV)
    s[0, 100:ld - 500] = float("nan")              # k-th among the few finite ones, then NaN = -inf
    s[1, :] = float("-inf")
    s[1, ::997] = 3.0                              # k-th bin is that of -inf (every key qualifies)
    s[2, :] = float("nan")                         # all NaN: ties at -inf, lowest positions win
    s[3, :] = -0.0
    s[3, ::3] = 0.0                                # signed zeros, all equal
    s[3, ::701] = -1.0
    s[4, 1000:1000 + 3000] = float("inf")          # more +inf than k
    s[5, :] = 1.25                                 # first value of its bin
    s[5, ::2] = 1.0                                # first value of the bin below
    s[5, ::7] = 1.2499999                          # last value of the bin below 1.25
    s[6, :] = -1.0                                 # negative: first value of its bin from the top
    s[6, ::5] = -0.9999999
    q_pos = torch.full((T,), ld - 1, dtype=torch.int32, device=DEV)
    hist = torch.as_tensor(_hist_of(s, q_pos), dtype=torch.int32, device=DEV)
    for k in (2048, 7):
        idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
        cnt = torch.empty((T,), dtype=torch.int32, device=DEV)
        ops.topk(s, q_pos, k, idx, cnt, hist=hist)
        pu.assert_topk_exact(to_numpy(idx), to_numpy(cnt), to_numpy(s).astype(np.float64), to_numpy(q_pos), k)
    assert ops.check_errors() == 0


def test_topk_row_path_list_segment_overflow():
    # The shared-memory row path lists the keys of the k-th bin in per-warp
    # segments (320 entries each).  Here the 1,280 keys of that bin all sit at
    # the positions one warp reads (p mod 1024 in one 32-wide band), more than
    # its segment holds although the whole bin would fit the list: the kernel
    # must take its pass over the whole row, and stay exact.
    g = torch.Generator(device=DEV).manual_seed(78)
    T, ld = 3, 40_960
    pos = torch.arange(ld, device=DEV)
    scores = -torch.rand((T, ld), generator=g, device=DEV)
    for t, lo in enumerate((0, 992, 480)):
        band = ((pos % 1024) >= lo) & ((pos % 1024) < lo + 32)
        scores[t, band] = 1.0 + 0.001 * torch.rand((int(band.sum()),), generator=g, device=DEV)
        top = pos[~band & (pos % 7 == 0)][:1500]
        scores[t, top] = 100.0 + torch.rand((1500,), generator=g, device=DEV)
    q_pos = torch.full((T,), ld - 1, dtype=torch.int32, device=DEV)
    hist = torch.as_tensor(_hist_of(scores, q_pos), dtype=torch.int32, device=DEV)
    idx = torch.empty((T, 2048), dtype=torch.int32, device=DEV)
    cnt = torch.empty((T,), dtype=torch.int32, device=DEV)
    ops.topk(scores, q_pos, 2048, idx, cnt, hist=hist)
    pu.assert_topk_exact(to_numpy(idx), to_numpy(cnt), to_numpy(scores).astype(np.float64), to_numpy(q_pos), 2048)
    assert ops.check_errors() == 0


# ------------------------------------------------------------------ attention

def _random_selection(wl, counts, sort=True, holes=False, seed=0):
    rng = np.random.default_rng(seed)
    q_pos = to_numpy(wl.q_pos)
    k = 2048
    idx = np.full((wl.T, k), -1, np.int32)
    for t, c in enumerate(counts):
        n = int(q_pos[t]) + 1
        c = min(c, n)
        sel = rng.choice(n, c, replace=False)
        if sort:
            sel = np.sort(sel)
        idx[t, :c] = sel
        if holes and c > 10:
            idx[t, 3] = -1      # skipped entries inside the counted prefix
    cnt = np.array([min(c, int(q_pos[t]) + 1) for t, c in enumerate(counts)], np.int32)
    return idx, cnt


@pytest.mark.parametrize("d_rope", [64, 0])
@pytest.mark.parametrize("sort", [True, False])
def test_attention_matches_oracle_split_path(d_rope, sort):
    # 5 queries: the kernel splits each selection across several CTAs and merges.
    case = small_case("attn_split", (4096, 3000, 2100, 600, 50), layers=(d_rope,), seed=17)
    wl = make_workload(case, DEV)
    idx, cnt = _random_selection(wl, [2048, 1500, 2048, 129, 37], sort=sort, holes=not sort, seed=3)
    lay = wl.layers[0]
    o, lse = pu.gpu_attend(wl, lay, torch.as_tensor(idx, device=DEV), torch.as_tensor(cnt, device=DEV))
    ref_o, ref_l = pu.oracle_attend(wl, lay, list(range(wl.T)), idx, cnt)
    pu.assert_attention_close(to_numpy(o), to_numpy(lse), ref_o, ref_l)


@pytest.mark.parametrize("d_rope", [64, 0])
def test_attention_matches_oracle_single_split_path(d_rope):
    # Enough queries that each one is handled by one CTA (bf16 written directly).
    lengths = tuple(int(x) for x in np.random.default_rng(4).integers(1, 3000, size=160))
    case = small_case("attn_many", lengths, layers=(d_rope,), seed=18, mla_q_std=1.0)
    wl = make_workload(case, DEV)
    counts = [2048 if i % 3 else min(2048, int(lengths[i])) for i in range(len(lengths))]
    idx, cnt = _random_selection(wl, counts, seed=5)
    lay = wl.layers[0]
    o, lse = pu.gpu_attend(wl, lay, torch.as_tensor(idx, device=DEV), torch.as_tensor(cnt, device=DEV))
    ts = list(range(0, wl.T, 7))
    ref_o, ref_l = pu.oracle_attend(wl, lay, ts, idx, cnt)
    pu.assert_attention_close(to_numpy(o)[ts], to_numpy(lse)[ts], ref_o, ref_l)


def _merge_widths():
    """(T, n_layers) of the smallest batch for which this GPU's plan merges a
    (layer, query)'s splits in a cluster of each width (2-8 blocks)."""
    found = {}
    for n_layers in (1, 2, 4):
        for T in range(1, 149):
            p = ops.plan_attend(T, n_layers, 2048)
            if p.merge and p.n_split not in found:
                found[p.n_split] = (T, n_layers)
    return found


def test_attention_cluster_merge_every_width_the_gpu_runs():
    # The splits of a (layer, query) merge their partials in distributed shared
    # memory when every cluster of that width can be resident at once.  The
    # batch sizes come from the library's own plan for this GPU, so every width
    # the GPU can run is exercised.  Short selections leave trailing CTAs empty.
    found = _merge_widths()
    assert len(found) >= 3, found
    for width, (T, n_layers) in sorted(found.items()):
        rng = np.random.default_rng(T * 10 + n_layers)
        lengths = tuple(int(x) for x in rng.integers(2100, 6000, size=T))
        rope = [64, 0, 64, 64][:n_layers]
        case = small_case(f"merge{width}", lengths, layers=tuple(rope), seed=40 + width, mla_q_std=1.0)
        wl = make_workload(case, DEV)
        counts = [2048 if i % 4 else int(rng.integers(1, 700)) for i in range(T)]
        idx, cnt = _random_selection(wl, counts, sort=(T % 2 == 0), holes=True, seed=T)
        plan = ops.plan_attend(T, n_layers, 2048)
        assert plan.merge and plan.n_split == width
        outs, lses = _attend_layers(wl, idx, cnt)
        ts = sorted(set(range(0, T, max(1, T // 4))) | {T - 1})
        for lay, o, l in zip(wl.layers, outs, lses):
            ref_o, ref_l = pu.oracle_attend(wl, lay, ts, idx, cnt)
            pu.assert_attention_close(to_numpy(o)[ts], to_numpy(l)[ts], ref_o, ref_l)


def _attend_layers(wl, idx, cnt, q_pos=None):
    T = wl.T
    outs = [torch.empty((T, 64, 512), dtype=torch.bfloat16, device=DEV) for _ in wl.layers]
    lses = [torch.empty((T, 64), dtype=torch.float32, device=DEV) for _ in wl.layers]
    layers = [dict(q_nope=L.q_nope, q_pe=L.q_pe, qmul=L.qmul, cache=L.cache, d_rope=L.d_rope, out=o, lse=l)
              for L, o, l in zip(wl.layers, outs, lses)]
    ops.sparse_mla_attend_layers(layers, wl.layers[0].cache.shape[0], wl.seq_row_start, wl.q_seq,
                                 torch.as_tensor(idx, device=DEV), torch.as_tensor(cnt, device=DEV), q_pos=q_pos)
    torch.cuda.synchronize()
    return outs, lses


def test_attend_layers_mixed_rope_and_nope_share_one_selection():
    # Four layers (three RoPE, one NoPE, as the 1M-context decode configuration)
    # in one launch over one selection: each layer against the oracle.
    case = small_case("layers4", (5000, 3000, 2100, 900), layers=(64, 64, 64, 0), seed=26)
    wl = make_workload(case, DEV)
    idx, cnt = _random_selection(wl, [2048, 2048, 2048, 900], seed=9, sort=False, holes=True)
    outs, lses = _attend_layers(wl, idx, cnt, q_pos=wl.q_pos)
    for lay, o, l in zip(wl.layers, outs, lses):
        ref_o, ref_l = pu.oracle_attend(wl, lay, list(range(wl.T)), idx, cnt)
        pu.assert_attention_close(to_numpy(o), to_numpy(l), ref_o, ref_l)
    assert ops.check_errors() == 0


def test_attention_empty_selection_gives_zero_and_minus_inf():
    case = small_case("attn_empty", (300, 300), seed=19)
    wl = make_workload(case, DEV)
    idx = torch.full((2, 2048), -1, dtype=torch.int32, device=DEV)
    cnt = torch.zeros(2, dtype=torch.int32, device=DEV)
    o, lse = pu.gpu_attend(wl, wl.layers[0], idx, cnt)
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


def test_attention_softmax_rows_sum_to_one():
    # sum_i exp(z_i - lse_gpu) = 1 with z recomputed by the oracle's definition.
    case = small_case("attn_norm", (2500, 900), seed=20)
    wl = make_workload(case, DEV)
    idx, cnt = _random_selection(wl, [2048, 700], seed=6)
    lay = wl.layers[0]
    _, lse = pu.gpu_attend(wl, lay, torch.as_tensor(idx, device=DEV), torch.as_tensor(cnt, device=DEV))
    lse = to_numpy(lse).astype(np.float64)
    starts, q_seq, _ = pu.host_meta(wl)
    cache = to_numpy(lay.cache).astype(np.float64)
    for t in range(wl.T):
        rows = cache[starts[q_seq[t]] + idx[t, :cnt[t]]]
        z = (to_numpy(lay.q_nope[t]).astype(np.float64) @ rows[:, :512].T
             + to_numpy(lay.q_pe[t]).astype(np.float64) @ rows[:, 512:576].T)
        z *= SOFTMAX_SCALE * to_numpy(lay.qmul[t]).astype(np.float64)[:, None]
        s = np.exp(z - lse[t][:, None]).sum(1)
        np.testing.assert_allclose(s, 1.0, atol=2e-3)


# ------------------------------------------------------------------ fused forward

def test_forward_tiny_decode_config_end_to_end():
    case = CONFIGS["tiny_decode"]
    wl = make_workload(case, DEV)
    T, ld = wl.T, case.ld
    lay = wl.layers[0]
    out = torch.empty((T, 64, 512), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((T, 64), dtype=torch.float32, device=DEV)
    idx = torch.empty((T, 2048), dtype=torch.int32, device=DEV)
    cnt = torch.empty((T,), dtype=torch.int32, device=DEV)
    ops.sparse_mla_forward(wl.q_idx, wl.w, wl.k_idx, wl.seq_row_start, wl.q_seq, wl.q_pos,
                           [dict(q_nope=lay.q_nope, q_pe=lay.q_pe, qmul=lay.qmul, cache=lay.cache,
                                 d_rope=64, out=out, lse=lse)], ld, idx_out=idx, count_out=cnt)
    torch.cuda.synchronize()
    assert to_numpy(cnt).tolist() == [2048, 2048, 1500, 37]
    ref_scores = pu.oracle_scores(wl, list(range(T)), ld)
    idx_h, cnt_h = to_numpy(idx), to_numpy(cnt)
    for t in range(T):
        n = int(to_numpy(wl.q_pos)[t]) + 1
        pu.assert_selection_overlap(idx_h[t, :cnt_h[t]], ref_scores[t, :n], 2048)
    # attention parity on the GPU's own selection
    ref_o, ref_l = pu.oracle_attend(wl, lay, list(range(T)), idx_h, cnt_h)
    pu.assert_attention_close(to_numpy(out), to_numpy(lse), ref_o, ref_l)
    # and the fused call equals the three separate calls bit for bit
    s = pu.gpu_scores(wl)
    idx2, cnt2 = pu.gpu_topk(s, wl.q_pos, 2048)
    o2, l2 = pu.gpu_attend(wl, lay, idx2, cnt2)
    assert torch.equal(idx2, idx) and torch.equal(o2, out) and torch.equal(l2, lse)


def test_forward_one_selection_feeds_rope_and_nope_layers_with_chunking():
    case = small_case("fwd_prefill", kind="prefill", cached=3000, new=40, layers=(64, 0), seed=21,
                      mla_q_std=1.0)
    wl = make_workload(case, DEV)
    T, ld = wl.T, case.ld
    outs = [torch.empty((T, 64, 512), dtype=torch.bfloat16, device=DEV) for _ in wl.layers]
    lses = [torch.empty((T, 64), dtype=torch.float32, device=DEV) for _ in wl.layers]
    layers = [dict(q_nope=L.q_nope, q_pe=L.q_pe, qmul=L.qmul, cache=L.cache, d_rope=L.d_rope, out=o,
                   lse=l) for L, o, l in zip(wl.layers, outs, lses)]
    idx = torch.empty((T, 2048), dtype=torch.int32, device=DEV)
    cnt = torch.empty((T,), dtype=torch.int32, device=DEV)
    # a workspace for 16 queries forces several chunks; a canary after it must survive
    ws_bytes = ops.forward_workspace_bytes(16, ld, 2048, 8, 2)
    plan = ops.plan_forward(T, ld, 2048, 8, 2, 1, 1, ws_bytes)
    assert plan.n_chunks > 1
    buf = torch.full((ws_bytes + (2 << 20),), 0xA5, dtype=torch.uint8, device=DEV)
    ops.sparse_mla_forward(wl.q_idx, wl.w, wl.k_idx, wl.seq_row_start, wl.q_seq, wl.q_pos, layers, ld,
                           q_group=8, idx_out=idx, count_out=cnt, ws=buf[:ws_bytes])
    torch.cuda.synchronize()
    assert bool((buf[ws_bytes:] == 0xA5).all()), "the fused call wrote past its workspace"
    idx_h, cnt_h = to_numpy(idx), to_numpy(cnt)
    s_ref = pu.oracle_scores(wl, list(range(T)), ld)
    for t in range(T):
        n = int(to_numpy(wl.q_pos)[t]) + 1
        pu.assert_selection_overlap(idx_h[t, :cnt_h[t]], s_ref[t, :n], 2048)
    for L, o, l in zip(wl.layers, outs, lses):
        ref_o, ref_l = pu.oracle_attend(wl, L, list(range(T)), idx_h, cnt_h)
        pu.assert_attention_close(to_numpy(o), to_numpy(l), ref_o, ref_l)


def test_forward_tail_chunk_stays_inside_the_workspace():
    # 151 decode queries at context 4,096 with a workspace sized for 148: the
    # last chunk is planned differently from the full ones (a small batch is
    # split wider).  A 2 MB canary after the workspace must survive, and the
    # results must match the oracle.
    case = small_case("tail151", (4096,) * 151, seed=25)
    wl = make_workload(case, DEV)
    T, ld = wl.T, case.ld
    lay = wl.layers[0]
    out = torch.empty((T, 64, 512), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((T, 64), dtype=torch.float32, device=DEV)
    ws_bytes = ops.forward_workspace_bytes(148, ld, 2048, 1, 1)
    plan = ops.plan_forward(T, ld, 2048, 1, 1, 0, 0, ws_bytes)
    assert plan.n_chunks > 1 and plan.end <= ws_bytes
    buf = torch.full((ws_bytes + (2 << 20),), 0x5A, dtype=torch.uint8, device=DEV)
    idx = torch.empty((T, 2048), dtype=torch.int32, device=DEV)
    cnt = torch.empty((T,), dtype=torch.int32, device=DEV)
    ops.sparse_mla_forward(wl.q_idx, wl.w, wl.k_idx, wl.seq_row_start, wl.q_seq, wl.q_pos,
                           [dict(q_nope=lay.q_nope, q_pe=lay.q_pe, qmul=lay.qmul, cache=lay.cache, d_rope=64,
                                 out=out, lse=lse)], ld, ws=buf[:ws_bytes])
    torch.cuda.synchronize()
    assert bool((buf[ws_bytes:] == 0x5A).all()), "the fused call wrote past its workspace"
    assert ops.check_errors() == 0
    # the same selection through the separate calls, for the sampled queries' parity
    s = pu.gpu_scores(wl)
    idx2, cnt2 = pu.gpu_topk(s, wl.q_pos, 2048)
    ts = [0, 37, 75, 112, 147, 148, 150]
    idx_h, cnt_h = to_numpy(idx2), to_numpy(cnt2)
    ref_s = pu.oracle_scores(wl, ts, ld)
    for i, t in enumerate(ts):
        pu.assert_selection_overlap(idx_h[t, :cnt_h[t]], ref_s[i, :4096], 2048)
    ref_o, ref_l = pu.oracle_attend(wl, lay, ts, idx_h, cnt_h)
    pu.assert_attention_close(to_numpy(out)[ts], to_numpy(lse)[ts], ref_o, ref_l)


def test_forward_four_layers_small_decode():
    # The 1M-context configuration's shape of work (4 queries, one selection ->
    # 3 RoPE + 1 NoPE layers) at small contexts, through the fused call.
    case = small_case("fwd4", (9000, 5000, 2049, 700), layers=(64, 64, 64, 0), seed=27)
    wl = make_workload(case, DEV)
    T, ld = wl.T, case.ld
    outs = [torch.empty((T, 64, 512), dtype=torch.bfloat16, device=DEV) for _ in wl.layers]
    lses = [torch.empty((T, 64), dtype=torch.float32, device=DEV) for _ in wl.layers]
    layers = [dict(q_nope=L.q_nope, q_pe=L.q_pe, qmul=L.qmul, cache=L.cache, d_rope=L.d_rope, out=o,
                   lse=l) for L, o, l in zip(wl.layers, outs, lses)]
    idx = torch.empty((T, 2048), dtype=torch.int32, device=DEV)
    cnt = torch.empty((T,), dtype=torch.int32, device=DEV)
    ops.sparse_mla_forward(wl.q_idx, wl.w, wl.k_idx, wl.seq_row_start, wl.q_seq, wl.q_pos, layers, ld,
                           idx_out=idx, count_out=cnt)
    assert ops.check_errors() == 0
    idx_h, cnt_h = to_numpy(idx), to_numpy(cnt)
    assert cnt_h.tolist() == [2048, 2048, 2048, 700]
    s_ref = pu.oracle_scores(wl, list(range(T)), ld)
    for t in range(T):
        n = int(to_numpy(wl.q_pos)[t]) + 1
        pu.assert_selection_overlap(idx_h[t, :cnt_h[t]], s_ref[t, :n], 2048)
    for L, o, l in zip(wl.layers, outs, lses):
        ref_o, ref_l = pu.oracle_attend(wl, L, list(range(T)), idx_h, cnt_h)
        pu.assert_attention_close(to_numpy(o), to_numpy(l), ref_o, ref_l)


def test_forward_four_queries_per_sequence():
    # One token plus three drafted tokens per sequence verified in one pass:
    # the fused call with q_group 4, against the oracle.
    case = small_case("fwd_mq", (6000, 2500, 2051), per_seq=4, layers=(64,), seed=30)
    wl = make_workload(case, DEV)
    T, ld = wl.T, case.ld
    lay = wl.layers[0]
    out = torch.empty((T, 64, 512), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((T, 64), dtype=torch.float32, device=DEV)
    idx = torch.empty((T, 2048), dtype=torch.int32, device=DEV)
    cnt = torch.empty((T,), dtype=torch.int32, device=DEV)
    ops.sparse_mla_forward(wl.q_idx, wl.w, wl.k_idx, wl.seq_row_start, wl.q_seq, wl.q_pos,
                           [dict(q_nope=lay.q_nope, q_pe=lay.q_pe, qmul=lay.qmul, cache=lay.cache, d_rope=64,
                                 out=out, lse=lse)], ld, q_group=4, idx_out=idx, count_out=cnt)
    assert ops.check_errors() == 0
    idx_h, cnt_h = to_numpy(idx), to_numpy(cnt)
    q_pos = to_numpy(wl.q_pos)
    assert cnt_h.tolist() == [min(2048, int(p) + 1) for p in q_pos]
    s_ref = pu.oracle_scores(wl, list(range(T)), ld)
    for t in range(T):
        pu.assert_selection_overlap(idx_h[t, :cnt_h[t]], s_ref[t, :int(q_pos[t]) + 1], 2048)
    ref_o, ref_l = pu.oracle_attend(wl, lay, list(range(T)), idx_h, cnt_h)
    pu.assert_attention_close(to_numpy(out), to_numpy(lse), ref_o, ref_l)


# ------------------------------------------------------------------ device-side checks

def test_bad_indices_are_flagged_not_faulted():
    case = small_case("bad_idx", (500, 500), seed=22)
    wl = make_workload(case, DEV)
    idx, cnt = _random_selection(wl, [300, 300], seed=7)
    idx[0, 5] = 10_000_000          # far outside the cache
    idx[1, 7] = -5                  # negative, not the -1 padding value
    out = torch.empty((2, 64, 512), dtype=torch.bfloat16, device=DEV)
    ops.sparse_mla_attend(wl.layers[0].q_nope, wl.layers[0].q_pe, wl.layers[0].qmul, wl.layers[0].cache,
                          64, wl.seq_row_start, wl.q_seq, torch.as_tensor(idx, device=DEV),
                          torch.as_tensor(cnt, device=DEV), out)
    with pytest.raises(ops.DSAError) as e:
        ops.check_errors()
    assert "0x1" in str(e.value)
    assert ops.check_errors() == 0   # cleared; the context is still usable
    assert torch.isfinite(out.float()).all()


def test_positions_past_q_pos_are_flagged_and_skipped():
    # A selected position past the query's own position (here: inside the cache,
    # in the next sequence's rows) is skipped and flagged when q_pos is given.
    case = small_case("qpos", (3000, 2500, 1000), seed=24)
    wl = make_workload(case, DEV)
    idx, cnt = _random_selection(wl, [500, 400, 300], seed=8)
    bad = idx.copy()
    bad[0, 10] = 3005          # sequence 1's rows
    bad[1, 20] = 2600          # sequence 2's rows
    lay = wl.layers[0]
    out = torch.empty((3, 64, 512), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((3, 64), dtype=torch.float32, device=DEV)
    ops.sparse_mla_attend(lay.q_nope, lay.q_pe, lay.qmul, lay.cache, 64, wl.seq_row_start, wl.q_seq,
                          torch.as_tensor(bad, device=DEV), torch.as_tensor(cnt, device=DEV), out, lse,
                          q_pos=wl.q_pos)
    with pytest.raises(ops.DSAError) as e:
        ops.check_errors()
    assert "0x1" in str(e.value)
    skipped = bad.copy()
    skipped[0, 10] = -1
    skipped[1, 20] = -1
    ref_o, ref_l = pu.oracle_attend(wl, lay, [0, 1, 2], skipped, cnt)
    pu.assert_attention_close(to_numpy(out), to_numpy(lse), ref_o, ref_l)
    assert ops.check_errors() == 0


def test_bad_sequence_ids_are_flagged():
    case = small_case("bad_seq", (500, 500), seed=23)
    wl = make_workload(case, DEV)
    wl.q_seq[1] = 7                 # only 2 sequences exist
    s = torch.empty((2, wl.case.ld), dtype=torch.float32, device=DEV)
    ops.index_scores(wl.q_idx, wl.w, wl.k_idx, wl.seq_row_start, wl.q_seq, wl.q_pos, s)
    with pytest.raises(ops.DSAError):
        ops.check_errors()
    assert torch.isneginf(s[1]).all()
