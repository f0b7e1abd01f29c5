"""Pins for the CPU oracle: checks against what the pages and the mathematics fix,
never against a retyped copy of the oracle's own formulas.

Each test names the property it relies on.  A plausible mistake in the oracle
(dropped ReLU, wrong sign, transposed operand, wrong tie rule, missing scale or
multiplier, off-by-one in the causal range, wrong sequence offset) fails at
least one of them.
"""

import json
import math
import os

import numpy as np
import pytest

from oracle import (dense_causal_mla, e4m3_decode, explicit_mla, forward, index_scores,
                    index_scores_fp8, latent_fp8_decode, lse_combine, sparse_mla, sparse_mla_fp8,
                    topk_merge, topk_select)

RNG = np.random.default_rng(1234)


def _bf16ish(x):
    """Round float64 values to bf16-representable float32 (truncate-to-nearest via float32 bits)."""
    f = np.asarray(x, dtype=np.float32)
    b = f.view(np.uint32).astype(np.uint64)
    b = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16
    return b.astype(np.uint32).view(np.float32)


def _toy(golden_dir):
    with open(os.path.join(golden_dir, "toy_examples.json")) as f:
        return json.load(f)


# --------------------------------------------------------------------------- indexer

def test_indexer_hand_worked_example(golden_dir):
    g = _toy(golden_dir)["indexer"]
    s = index_scores(np.array(g["q_idx"], float), np.array(g["w"]), np.array(g["k_idx"], float),
                     np.array(g["seq_row_start"]), np.array(g["q_seq"]), np.array(g["q_pos"]),
                     g["ld"])
    want = np.array([[float(v) for v in row] for row in g["scores"]])
    assert np.array_equal(s, want)


def _rand_index_case(T=3, lens=(40, 75, 9), H=32, D=128):
    rows = sum(lens)
    starts = np.cumsum([0] + list(lens[:-1]))
    q = _bf16ish(RNG.standard_normal((T, H, D)))
    w = (RNG.standard_normal((T, H)) / math.sqrt(H)).astype(np.float32).astype(np.float64)
    k = _bf16ish(RNG.standard_normal((rows, D)))
    q_seq = np.arange(T) % len(lens)
    q_pos = np.array([lens[b] - 1 for b in q_seq])
    return q, w, k, starts, q_seq, q_pos, max(lens)


def test_indexer_single_head_unit_query_closed_form():
    # w = a * e_j and q[t, j] = beta * e_d  =>  I[t, s] = a * beta * max(0, k[s, d]).
    q, w, k, starts, q_seq, q_pos, ld = _rand_index_case()
    j, d, a, beta = 5, 17, -1.75, 2.5
    w[:] = 0.0
    w[:, j] = a
    q[:, j, :] = 0.0
    q[:, j, d] = beta
    s = index_scores(q, w, k, starts, q_seq, q_pos, ld)
    for t in range(len(q_seq)):
        n = q_pos[t] + 1
        rows = k[starts[q_seq[t]]:starts[q_seq[t]] + n, d].astype(np.float64)
        np.testing.assert_allclose(s[t, :n], a * beta * np.maximum(rows, 0.0), rtol=0, atol=0)


def test_indexer_odd_part_identity():
    # relu(x) - relu(-x) = x, so I(k) - I(-k) = (sum_j w_j q_j) . k: linear in k,
    # with the head weights applied once and the ReLU present.
    q, w, k, starts, q_seq, q_pos, ld = _rand_index_case()
    sp = index_scores(q, w, k, starts, q_seq, q_pos, ld)
    sm = index_scores(q, w, -k, starts, q_seq, q_pos, ld)
    for t in range(len(q_seq)):
        n = q_pos[t] + 1
        d = (w[t].astype(np.float64)[:, None] * q[t].astype(np.float64)).sum(0)
        rows = k[starts[q_seq[t]]:starts[q_seq[t]] + n].astype(np.float64)
        np.testing.assert_allclose(sp[t, :n] - sm[t, :n], rows @ d, rtol=1e-10, atol=1e-9)
        # and both parts are genuinely non-linear: I(k) + I(-k) = sum_j w_j |q_j . k|
        assert not np.allclose(sp[t, :n] + sm[t, :n], 0.0)


def test_indexer_homogeneity_and_sign_of_w():
    q, w, k, starts, q_seq, q_pos, ld = _rand_index_case()
    base = index_scores(q, w, k, starts, q_seq, q_pos, ld)
    fin = np.isfinite(base)
    # positive scaling of q or k passes through the ReLU; w enters linearly.
    np.testing.assert_allclose(index_scores(2 * q, w, k, starts, q_seq, q_pos, ld)[fin],
                               2 * base[fin], rtol=1e-12)
    np.testing.assert_allclose(index_scores(q, w, 0.5 * k, starts, q_seq, q_pos, ld)[fin],
                               0.5 * base[fin], rtol=1e-12)
    np.testing.assert_allclose(index_scores(q, -3 * w, k, starts, q_seq, q_pos, ld)[fin],
                               -3 * base[fin], rtol=1e-12)
    # with every weight positive, every score is non-negative (ReLU before weighting)
    assert (index_scores(q, np.abs(w), k, starts, q_seq, q_pos, ld)[fin] >= 0).all()


def test_indexer_causal_range_and_sequence_offsets():
    q, w, k, starts, q_seq, q_pos, ld = _rand_index_case(T=3, lens=(40, 75, 9))
    s = index_scores(q, w, k, starts, q_seq, q_pos, ld)
    for t in range(3):
        n = q_pos[t] + 1
        assert np.isfinite(s[t, :n]).all()            # own position included
        assert np.isneginf(s[t, n:]).all()            # later positions masked
    # changing another sequence's keys, or keys beyond q_pos, changes nothing
    k2 = k.copy()
    k2[starts[1]:starts[1] + 75] = 0.0
    s2 = index_scores(q, w, k2, starts, q_seq, q_pos, ld)
    np.testing.assert_allclose(s2[[0, 2]], s[[0, 2]], rtol=1e-12, atol=1e-12)
    assert np.all(s2[1, :75] == 0.0)
    # moving the query earlier only truncates its row
    q_pos3 = q_pos.copy()
    q_pos3[1] = 30
    s3 = index_scores(q, w, k, starts, q_seq, q_pos3, ld)
    np.testing.assert_allclose(s3[1, :31], s[1, :31], rtol=1e-12, atol=1e-12)
    assert np.isneginf(s3[1, 31:]).all()


# --------------------------------------------------------------------------- FP8 (E4M3) index keys

def test_e4m3_decode_matches_library_conversion_for_every_code():
    # torch's float8_e4m3fn is the same OCP E4M3 format; all 256 codes agree (NaN where it has NaN).
    torch = pytest.importorskip("torch")
    c = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(c.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = e4m3_decode(c)
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    assert np.array_equal(mine[~np.isnan(mine)], ref[~np.isnan(ref)])


def test_e4m3_decode_landmark_values():
    # The format's definition: 1.0 = 0.0111.000, largest finite 448 = 0.1111.110, smallest normal
    # 2^-6 = 0.0001.000, smallest subnormal 2^-9 = 0.0000.001, sign bit, NaN = S.1111.111.
    v = e4m3_decode(np.array([0x38, 0x7E, 0x08, 0x01, 0xB8, 0x00, 0x40, 0x44, 0x7F, 0xFF], np.uint8))
    assert v[:8].tolist() == [1.0, 448.0, 2.0 ** -6, 2.0 ** -9, -1.0, 0.0, 2.0, 3.0]
    assert np.isnan(v[8]) and np.isnan(v[9])


def test_indexer_fp8_hand_worked_example():
    # Two heads x 2 dims, integer codes: q0 = (1, 2), q1 = (-1, 1); keys (1, 1) and (2, 0); w = (1, 0.5).
    #   s=0: head0 1+2 = 3, head1 -1+1 = 0  -> I = 1*3 + 0.5*0 = 3, times k_scale 2 -> 6
    #   s=1: head0 2+0 = 2, head1 -2+0 = -2 -> I = 1*2 + 0.5*ReLU(-2) = 2 (not ReLU(2 - 1) = 1)
    one, two, mone, zero = 0x38, 0x40, 0xB8, 0x00
    q8 = np.array([[[one, two], [mone, one]]], np.uint8)
    k8 = np.array([[one, one], [two, zero]], np.uint8)
    I = index_scores_fp8(q8, np.ones((1, 2)), np.array([[1.0, 0.5]]), k8, np.array([2.0, 1.0]),
                         np.array([0]), np.array([0]), np.array([1]), 4)
    assert I[0, :2].tolist() == [6.0, 2.0]
    assert np.all(np.isneginf(I[0, 2:]))


def test_indexer_fp8_scale_homogeneity_and_offsets():
    # Each key scale multiplies its own column; each query's scales multiply its row (ReLU of a
    # positively scaled argument); a zero scale zeroes the scores; sequences read their own rows.
    rng = np.random.default_rng(8)
    T, H, d, rows = 3, 4, 16, 90
    q8 = rng.integers(0, 256, (T, H, d)).astype(np.uint8)
    k8 = rng.integers(0, 256, (rows, d)).astype(np.uint8)
    q8[(q8 & 0x7F) == 0x7F] = 0x38     # no NaN codes
    k8[(k8 & 0x7F) == 0x7F] = 0x38
    qs = rng.uniform(0.01, 0.1, (T, H))
    ks = rng.uniform(0.01, 0.1, rows)
    w = rng.normal(size=(T, H))
    starts, q_seq, q_pos = np.array([0, 40]), np.array([0, 1, 1]), np.array([39, 49, 20])
    base = index_scores_fp8(q8, qs, w, k8, ks, starts, q_seq, q_pos, 64)
    ks2 = ks.copy()
    ks2[40 + 7] *= 4.0                   # row 7 of sequence 1
    b2 = index_scores_fp8(q8, qs, w, k8, ks2, starts, q_seq, q_pos, 64)
    np.testing.assert_allclose(b2[1:, 7], 4.0 * base[1:, 7], rtol=1e-12)
    np.testing.assert_array_equal(np.delete(b2[1:], 7, axis=1), np.delete(base[1:], 7, axis=1))
    np.testing.assert_array_equal(b2[0], base[0])   # sequence 0 never reads row 47's scale at s = 7
    qs3 = qs.copy()
    qs3[2] *= 3.0
    b3 = index_scores_fp8(q8, qs3, w, k8, ks, starts, q_seq, q_pos, 64)
    np.testing.assert_allclose(b3[2, :21], 3.0 * base[2, :21], rtol=1e-12)
    b0 = index_scores_fp8(q8, np.zeros_like(qs), w, k8, ks, starts, q_seq, q_pos, 64)
    assert np.all(b0[0, :40] == 0.0) and np.all(np.isneginf(b0[0, 40:]))
    assert np.all(np.isneginf(base[2, 21:]))


# --------------------------------------------------------------------------- top-k

def test_topk_hand_worked_example(golden_dir):
    g = _toy(golden_dir)["indexer"]
    scores = np.array([[float(v) for v in row] for row in g["scores"]])
    for key, kk in (("k1", 1), ("k2", 2), ("k4", 4)):
        idx, cnt = topk_select(scores, np.array(g["q_pos"]), kk)
        assert idx.tolist() == g["topk"][key]["idx"]
        assert cnt.tolist() == g["topk"][key]["count"]


def _select_by_repeated_argmax(row, k):
    """Brute force: repeatedly take the best remaining score, lower position first on ties."""
    vals = [(-math.inf if math.isnan(v) else v) for v in row]
    left = list(range(len(vals)))
    chosen = []
    for _ in range(min(k, len(vals))):
        best = left[0]
        for i in left[1:]:
            if vals[i] > vals[best]:
                best = i
        chosen.append(best)
        left.remove(best)
    return sorted(chosen)


@pytest.mark.parametrize("trial", range(40))
def test_topk_brute_force_tiny_with_ties(trial):
    rng = np.random.default_rng(100 + trial)
    T, ld = 3, int(rng.integers(1, 24))
    k = int(rng.integers(1, 12))
    scores = rng.integers(-3, 4, size=(T, ld)).astype(np.float64)   # many ties
    if trial % 5 == 0:
        scores[:, ::3] = -0.0
    q_pos = rng.integers(0, ld, size=T)
    idx, cnt = topk_select(scores, q_pos, k)
    for t in range(T):
        want = _select_by_repeated_argmax(list(scores[t, :q_pos[t] + 1]), k)
        assert cnt[t] == len(want)
        assert idx[t, :cnt[t]].tolist() == want
        assert (idx[t, cnt[t]:] == -1).all()


def test_topk_signed_zero_and_nan():
    scores = np.array([[0.0, -0.0, np.nan, 0.0, -1.0, np.nan]])
    idx, cnt = topk_select(scores, np.array([5]), 3)
    assert idx.tolist() == [[0, 1, 3]]      # -0 == +0, ties to lower positions
    idx, cnt = topk_select(scores, np.array([5]), 5)
    assert idx.tolist() == [[0, 1, 2, 3, 4]]  # NaN ranks as -inf, below -1.0, lower NaN first


def test_topk_closed_forms():
    n, k = 300, 37
    q_pos = np.array([n - 1])
    idx, _ = topk_select(np.full((1, n), 2.5), q_pos, k)
    assert idx[0].tolist() == list(range(k))                 # all equal -> lowest positions
    idx, _ = topk_select(-np.arange(n, dtype=float)[None], q_pos, k)
    assert idx[0].tolist() == list(range(k))                 # decreasing
    idx, _ = topk_select(np.arange(n, dtype=float)[None], q_pos, k)
    assert idx[0].tolist() == list(range(n - k, n))          # increasing
    idx, cnt = topk_select(np.arange(n, dtype=float)[None], q_pos, 2048)
    assert cnt[0] == n and idx[0, :n].tolist() == list(range(n)) and (idx[0, n:] == -1).all()


def test_topk_invariants_random():
    rng = np.random.default_rng(7)
    T, ld, k = 4, 5000, 2048
    scores = rng.standard_normal((T, ld)).astype(np.float32).astype(np.float64)
    scores[:, 100:140] = scores[0, 3]   # a block of exact ties
    q_pos = np.array([4999, 3000, 2047, 10])
    idx, cnt = topk_select(scores, q_pos, k)
    for t in range(T):
        n = q_pos[t] + 1
        sel = idx[t, :cnt[t]]
        assert cnt[t] == min(k, n)
        assert np.all(np.diff(sel) > 0)
        rest = np.setdiff1d(np.arange(n), sel)
        if rest.size:
            lo = scores[t, sel].min()
            assert lo >= scores[t, rest].max()
            tied_out = rest[scores[t, rest] == lo]
            tied_in = sel[scores[t, sel] == lo]
            if tied_out.size:
                assert tied_in.max() < tied_out.min()


# --------------------------------------------------------------------------- attention

# --------------------------------------------------------------------------- context-parallel pieces

@pytest.mark.parametrize("trial", range(12))
def test_topk_merge_of_shard_selections_equals_whole_row(trial):
    # Every element of the global top-k is in its own shard's top-k (the tie rule is the
    # same global-position order inside a shard), so merging the shards' lists is exact.
    rng = np.random.default_rng(100 + trial)
    n = int(rng.integers(5, 400))
    k = int(rng.integers(1, 60))
    row = rng.integers(-4, 5, n).astype(float) if trial % 2 else rng.normal(size=n)
    row[rng.random(n) < 0.1] = -0.0
    whole, cnt = topk_select(row[None, :], np.array([n - 1]), k)
    G = int(rng.integers(2, 6))
    edges = np.linspace(0, n, G + 1).astype(int)
    cs, cp = [], []
    for a, b in zip(edges[:-1], edges[1:]):
        if b <= a:
            continue
        sel, c = topk_select(row[None, a:b], np.array([b - a - 1]), k)
        pos = sel[0, :c[0]].astype(np.int64) + a
        cs.append(row[pos])
        cp.append(pos)
    cs.append(np.array([np.inf, 3.0]))     # empty slots (position -1) never take part, whatever their score
    cp.append(np.array([-1, -1]))
    merged = topk_merge(np.concatenate(cs), np.concatenate(cp), k)
    assert merged.tolist() == whole[0, :cnt[0]].tolist()


def test_lse_combine_of_parts_equals_whole_selection():
    qn, qp, m, cache, starts, q_seq, q_pos = _rand_attn_case(T=1, lens=(300,))
    scale = 0.2
    for n_parts in (2, 3, 5):
        sel = np.sort(np.random.default_rng(n_parts).choice(300, 97, replace=False))
        idx = np.full((1, 2048), -1, np.int32)
        idx[0, :97] = sel
        o_all, l_all = sparse_mla(qn, qp, m, scale, cache, 64, starts, q_seq, idx, np.array([97]))
        parts = np.array_split(np.random.default_rng(7).permutation(sel), n_parts)
        parts.append(np.array([], dtype=np.int64))          # an empty part contributes nothing
        o_p, l_p = [], []
        for part in parts:
            ip = np.full((1, 2048), -1, np.int32)
            ip[0, :part.size] = part
            o, l = sparse_mla(qn, qp, m, scale, cache, 64, starts, q_seq, ip, np.array([part.size]))
            o_p.append(o[0])
            l_p.append(l[0])
        o, l = lse_combine(np.stack(o_p), np.stack(l_p))
        np.testing.assert_allclose(o, o_all[0], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(l, l_all[0], rtol=1e-12)
    o0, l0 = lse_combine(np.zeros((2, 64, 512)), np.full((2, 64), -np.inf))
    assert np.all(o0 == 0) and np.all(np.isneginf(l0))


def test_attention_hand_worked_example(golden_dir):
    g = _toy(golden_dir)["attention"]
    cache = np.array(g["cache"], float)
    for c in g["cases"]:
        o, lse = sparse_mla(np.array([[c["q_nope"]]]), np.array([[c["q_pe"]]]), np.ones((1, 1)),
                            g["scale"], cache, g["d_rope"], np.array([0]), np.array([0]),
                            np.array([[0, 1]]), np.array([2]))
        np.testing.assert_allclose(o[0, 0], c["o"], rtol=1e-12)
        np.testing.assert_allclose(lse[0, 0], c["lse"], rtol=1e-12)


def _rand_attn_case(T=2, lens=(33, 50), H=64, d_c=512, d_r=64, std=1.0 / math.sqrt(192)):
    rows = sum(lens)
    starts = np.cumsum([0] + list(lens[:-1]))
    cache = _bf16ish(RNG.standard_normal((rows, d_c + d_r)))
    qn = _bf16ish(RNG.standard_normal((T, H, d_c)) * std)
    qp = _bf16ish(RNG.standard_normal((T, H, d_r)) * std) if d_r else None
    m = (RNG.random((T, H)) + 0.5).astype(np.float32)
    q_seq = np.arange(T) % len(lens)
    q_pos = np.array([lens[b] - 1 for b in q_seq])
    return qn, qp, m, cache, starts, q_seq, q_pos


@pytest.mark.parametrize("d_r", [64, 0])
def test_sparse_equals_dense_when_everything_is_selected(d_r):
    qn, qp, m, cache, starts, q_seq, q_pos = _rand_attn_case(d_r=d_r, std=1.0)
    scale = 1.0 / math.sqrt(192)
    n_max = q_pos.max() + 1
    idx = np.full((len(q_seq), 2048), -1, np.int32)
    cnt = np.zeros(len(q_seq), np.int32)
    for t in range(len(q_seq)):
        n = q_pos[t] + 1
        idx[t, :n] = RNG.permutation(n)          # any order of the full set
        cnt[t] = n
    o_s, l_s = sparse_mla(qn, qp, m, scale, cache, d_r, starts, q_seq, idx, cnt)
    o_d, l_d = dense_causal_mla(qn, qp, m, scale, cache, d_r, starts, q_seq, q_pos)
    assert n_max <= 2048
    np.testing.assert_allclose(o_s, o_d, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(l_s, l_d, rtol=1e-12)


def test_absorbed_equals_explicit_per_head_mla():
    # q_nope_h = W_UK_h^T q_h  and  out_h = W_UV_h o_h  (absorption of the up-projections).
    H, d_c, d_r, d_h = 64, 512, 64, 128
    qn_unused, qp, m, cache, starts, q_seq, q_pos = _rand_attn_case(T=2, H=H, d_c=d_c, d_r=d_r)
    W_UK = RNG.standard_normal((H, d_h, d_c)) / math.sqrt(d_c)
    W_UV = RNG.standard_normal((H, d_h, d_c)) / math.sqrt(d_c)
    q_head = RNG.standard_normal((2, H, d_h))
    q_nope = np.einsum("hdc,thd->thc", W_UK, q_head)
    idx = np.full((2, 2048), -1, np.int32)
    cnt = np.array([20, 41], np.int32)
    idx[0, :20] = np.sort(RNG.choice(33, 20, replace=False))
    idx[1, :41] = np.sort(RNG.choice(50, 41, replace=False))
    scale = 1.0 / math.sqrt(192)
    o_abs, _ = sparse_mla(q_nope, qp, m, scale, cache, d_r, starts, q_seq, idx, cnt)
    out = explicit_mla(q_head, qp, W_UK, W_UV, m, scale, cache, d_r, starts, q_seq, idx, cnt)
    np.testing.assert_allclose(np.einsum("hdc,thc->thd", W_UV, o_abs), out, rtol=1e-9, atol=1e-12)


def test_single_row_and_uniform_closed_forms():
    qn, qp, m, cache, starts, q_seq, q_pos = _rand_attn_case(T=1, lens=(60,))
    scale = 0.3
    idx = np.full((1, 2048), -1, np.int32)
    idx[0, 0] = 17
    o, lse = sparse_mla(qn, qp, m, scale, cache, 64, starts, q_seq, idx, np.array([1]))
    np.testing.assert_allclose(o[0], np.broadcast_to(cache[17, :512], (64, 512)), rtol=1e-15)
    z = ((qn[0].astype(float) @ cache[17, :512]) + qp[0].astype(float) @ cache[17, 512:]) * scale * m[0]
    np.testing.assert_allclose(lse[0], z, rtol=1e-12)
    # zero multiplier: uniform weights -> mean of the selected rows, lse = ln n
    sel = np.array([3, 9, 10, 44, 59])
    idx[0, :5] = sel
    o, lse = sparse_mla(qn, qp, np.zeros_like(m), scale, cache, 64, starts, q_seq, idx, np.array([5]))
    # (atol: a column whose mean is ~0 differs by float64 rounding of the two summation orders, ~1e-17)
    np.testing.assert_allclose(o[0], np.broadcast_to(cache[sel, :512].astype(np.float64).mean(0), (64, 512)),
                               rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(lse[0], math.log(5), rtol=1e-12)


def test_softmax_normalises_and_rows_weighted():
    # For a tiny head the logits are computed by loops here; the oracle's lse must
    # normalise them and o must be the corresponding weighted sum of rows.
    H, d_c, d_r = 2, 3, 2
    cache = np.array([[1, -2, 0.5, 1, 0], [0, 1, 2, -1, 3], [2, 2, -1, 0.5, 0.5]], float)
    qn = np.array([[[0.3, -0.1, 0.7], [1.0, 0.0, -0.5]]])
    qp = np.array([[[0.2, 0.1], [-0.3, 0.4]]])
    m = np.array([[1.5, 0.5]])
    idx = np.array([[0, 2, 1]])
    o, lse = sparse_mla(qn, qp, m, 0.9, cache, d_r, np.array([0]), np.array([0]), idx, np.array([3]))
    for h in range(H):
        z = []
        for s in (0, 2, 1):
            acc = 0.0
            for d in range(d_c):
                acc += qn[0, h, d] * cache[s, d]
            for r in range(d_r):
                acc += qp[0, h, r] * cache[s, d_c + r]
            z.append(acc * 0.9 * m[0, h])
        p = [math.exp(v - lse[0, h]) for v in z]
        assert abs(sum(p) - 1.0) < 1e-12
        want = [sum(p[i] * cache[s, d] for i, s in enumerate((0, 2, 1))) for d in range(d_c)]
        np.testing.assert_allclose(o[0, h], want, rtol=1e-12)


def test_permutation_and_padding_invariance():
    qn, qp, m, cache, starts, q_seq, q_pos = _rand_attn_case(T=1, lens=(80,))
    sel = np.sort(RNG.choice(80, 30, replace=False))
    idx = np.full((1, 2048), -1, np.int32)
    idx[0, :30] = sel
    o1, l1 = sparse_mla(qn, qp, m, 0.1, cache, 64, starts, q_seq, idx, np.array([30]))
    idx[0, :30] = sel[::-1]
    o2, l2 = sparse_mla(qn, qp, m, 0.1, cache, 64, starts, q_seq, idx, np.array([30]))
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(l1, l2, rtol=1e-12)


def test_nope_layer_equals_rope_layer_with_zero_rotary_query():
    qn, qp, m, cache, starts, q_seq, q_pos = _rand_attn_case(T=1, lens=(40,))
    idx = np.full((1, 2048), -1, np.int32)
    idx[0, :25] = np.arange(25)
    o_r, l_r = sparse_mla(qn, np.zeros_like(qp), m, 0.2, cache, 64, starts, q_seq, idx, np.array([25]))
    o_n, l_n = sparse_mla(qn, None, m, 0.2, np.ascontiguousarray(cache[:, :512]), 0, starts, q_seq,
                          idx, np.array([25]))
    np.testing.assert_allclose(o_r, o_n, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(l_r, l_n, rtol=1e-12)


def test_empty_selection():
    qn, qp, m, cache, starts, q_seq, q_pos = _rand_attn_case(T=1, lens=(10,))
    idx = np.full((1, 2048), -1, np.int32)
    o, lse = sparse_mla(qn, qp, m, 0.2, cache, 64, starts, q_seq, idx, np.array([0]))
    assert np.all(o == 0) and np.all(np.isneginf(lse))


# --------------------------------------------------------------------------- FP8 latent cache

def _fp8_rows(codes, scales, row_bytes, pad=0):
    """Byte rows of the FP8 latent layout: codes, then little-endian fp32 scales, then padding."""
    codes = np.asarray(codes, dtype=np.uint8)
    scales = np.asarray(scales, dtype="<f4")
    n, nc = codes.shape
    out = np.full((n, row_bytes), pad, dtype=np.uint8)
    out[:, :nc] = codes
    out[:, nc:nc + 4 * scales.shape[1]] = scales.view(np.uint8).reshape(n, -1)
    return out


def test_latent_fp8_hand_worked_rows(golden_dir):
    g = _toy(golden_dir)["latent_fp8"]
    d_c, d_r = g["d_c"], g["d_rope"]
    codes, scales = [], []
    for r in g["rows"]:
        c = np.full(d_c + d_r, r["fill_code"], dtype=np.uint8)
        for col, code in r["codes_at"].items():
            c[int(col)] = code
        codes.append(c)
        scales.append(r["scales"])
    rows = _fp8_rows(np.stack(codes), np.array(scales), g["row_bytes"], pad=g["pad_byte"])
    got = latent_fp8_decode(rows, d_c, d_r)
    assert got.shape == (len(g["rows"]), d_c + d_r)
    for i, e in enumerate(g["expected"]):
        want = np.concatenate([np.full(128, e["fill_by_block"][0]), np.full(d_c - 128, e["fill_by_block"][1]),
                               np.full(d_r, e["fill_by_block"][2])])
        for col, v in e["at"].items():
            want[int(col)] = v
        np.testing.assert_array_equal(got[i], want)


def _rand_fp8_attn_case(T=2, lens=(40, 70), d_r=64):
    qn, qp, m, _, starts, q_seq, q_pos = _rand_attn_case(T=T, lens=lens, d_r=d_r, std=0.3)
    rows = sum(lens)
    codes = RNG.integers(0, 256, size=(rows, 512 + d_r)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x38                  # no NaN codes
    n_blk = 4 + (1 if d_r else 0)
    scales = np.exp2(RNG.integers(-3, 2, size=(rows, n_blk))) * (1.0 + RNG.random((rows, n_blk)))
    scales = (scales / 64.0).astype(np.float32)           # values up to ~448 * 4 / 64
    row_bytes = (512 + d_r + 4 * n_blk + 15) // 16 * 16
    idx = np.full((T, 64), -1, np.int32)
    cnt = np.zeros(T, np.int32)
    for t in range(T):
        n = min(64, q_pos[t] + 1)
        idx[t, :n] = np.sort(RNG.choice(q_pos[t] + 1, size=n, replace=False))
        cnt[t] = n
    return qn, qp, m, codes, scales, row_bytes, starts, q_seq, idx, cnt


@pytest.mark.parametrize("d_r", [64, 0])
def test_sparse_mla_fp8_with_unit_scales_is_attention_on_the_code_values(d_r):
    # all scales 1: the decoded cache is the E4M3 values themselves (e4m3_decode is pinned on
    # every code), so the FP8 attention is sparse_mla on those values.
    qn, qp, m, codes, scales, rb, starts, q_seq, idx, cnt = _rand_fp8_attn_case(d_r=d_r)
    rows8 = _fp8_rows(codes, np.ones_like(scales), rb, pad=0x7F)
    o8, l8 = sparse_mla_fp8(qn, qp, m, 0.1, rows8, d_r, starts, q_seq, idx, cnt)
    o, l = sparse_mla(qn, qp, m, 0.1, e4m3_decode(codes), d_r, starts, q_seq, idx, cnt)
    np.testing.assert_allclose(o8, o, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(l8, l, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("blk", [0, 1, 2, 3])
def test_sparse_mla_fp8_block_scale_trades_against_that_block_of_the_query(blk):
    # Doubling the scale of latent block b in every row while halving columns
    # [128 b, 128 b + 128) of every query leaves every logit unchanged, so the
    # weights and lse are unchanged and exactly that block of the output doubles.
    qn, qp, m, codes, scales, rb, starts, q_seq, idx, cnt = _rand_fp8_attn_case()
    o, l = sparse_mla_fp8(qn, qp, m, 0.1, _fp8_rows(codes, scales, rb), 64, starts, q_seq, idx, cnt)
    s2 = scales.copy()
    s2[:, blk] *= 2
    qn2 = qn.astype(np.float64).copy()
    qn2[:, :, 128 * blk:128 * blk + 128] /= 2
    o2, l2 = sparse_mla_fp8(qn2, qp, m, 0.1, _fp8_rows(codes, s2, rb), 64, starts, q_seq, idx, cnt)
    np.testing.assert_allclose(l2, l, rtol=1e-12, atol=1e-12)
    want = o.copy()
    want[:, :, 128 * blk:128 * blk + 128] *= 2
    np.testing.assert_allclose(o2, want, rtol=1e-11, atol=1e-14)


def test_sparse_mla_fp8_rotary_scale_trades_against_q_pe_and_zero_equals_no_rotary_query():
    qn, qp, m, codes, scales, rb, starts, q_seq, idx, cnt = _rand_fp8_attn_case()
    o, l = sparse_mla_fp8(qn, qp, m, 0.1, _fp8_rows(codes, scales, rb), 64, starts, q_seq, idx, cnt)
    s2 = scales.copy()
    s2[:, 4] *= 4
    o2, l2 = sparse_mla_fp8(qn, qp.astype(np.float64) / 4, m, 0.1, _fp8_rows(codes, s2, rb), 64, starts, q_seq,
                            idx, cnt)
    np.testing.assert_allclose(o2, o, rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(l2, l, rtol=1e-12, atol=1e-12)
    # the rotary part really takes part ...
    s3 = scales.copy()
    s3[:, 4] = 0.0
    o3, l3 = sparse_mla_fp8(qn, qp, m, 0.1, _fp8_rows(codes, s3, rb), 64, starts, q_seq, idx, cnt)
    assert np.abs(l3 - l).max() > 1e-3
    # ... and a zero rotary scale is a zero rotary query
    o4, l4 = sparse_mla_fp8(qn, np.zeros_like(qp), m, 0.1, _fp8_rows(codes, scales, rb), 64, starts, q_seq,
                            idx, cnt)
    np.testing.assert_allclose(o3, o4, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(l3, l4, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------- composition

def _forward_toy(golden_dir):
    g = _toy(golden_dir)
    ix, fw = g["indexer"], g["forward"]
    layers = []
    for lay in fw["layers"]:
        layers.append(dict(q_nope=np.array(lay["q_nope"], float)[:, None, :],
                           q_pe=None if lay["q_pe"] is None else np.array(lay["q_pe"], float)[:, None, :],
                           qmul=np.ones((2, 1)), cache=np.array(lay["cache"], float), d_rope=lay["d_rope"]))
    args = (np.array(ix["q_idx"], float), np.array(ix["w"]), np.array(ix["k_idx"], float),
            np.array(ix["seq_row_start"]), np.array(ix["q_seq"]), np.array(fw["q_pos"]))
    return fw, args, layers


def test_forward_hand_worked_example(golden_dir):
    # Hand-worked selection and per-layer outputs (one RoPE and one NoPE layer
    # sharing one selection) for k = 1, 2 and 4 (more than the candidates).
    fw, args, layers = _forward_toy(golden_dir)
    want_scores = np.array([[float(v) for v in row] for row in fw["scores"]])
    np.testing.assert_array_equal(index_scores(*args, 3), want_scores)
    for key, kk in (("k1", 1), ("k2", 2), ("k4", 4)):
        c = fw["cases"][key]
        idx, cnt, outs = forward(*args, layers, 1.0, k=kk)
        assert idx.tolist() == c["idx"], key
        assert cnt.tolist() == c["count"], key
        assert len(outs) == len(layers)
        for (o, lse), o_want, l_want in zip(outs, c["o"], c["lse"]):
            np.testing.assert_allclose(o, np.array(o_want), rtol=1e-12, atol=1e-15)
            np.testing.assert_allclose(lse, np.array(l_want), rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("trial", range(6))
def test_forward_selection_is_the_top_k_of_the_indexer_scores(trial):
    # The shared selection is the top-k of the indexer's own scores, over the
    # causal range of each query, with the given k (random sizes, some queries
    # with fewer than k candidates, several queries per sequence).
    rng = np.random.default_rng(500 + trial)
    lens = tuple(int(x) for x in rng.integers(5, 90, size=3))
    q, w, k, starts, q_seq, q_pos, ld = _rand_index_case(T=3, lens=lens)
    q_pos = np.array([int(rng.integers(0, lens[b])) for b in q_seq])
    qn, qp, m, cache, _, _, _ = _rand_attn_case(T=3, lens=lens)
    layers = [dict(q_nope=qn, q_pe=qp, qmul=m, cache=cache, d_rope=64)]
    kk = int(rng.integers(1, 70))
    idx, cnt, outs = forward(q, w, k, starts, q_seq, q_pos, layers, 0.1, k=kk)
    for t in range(3):
        n = q_pos[t] + 1
        b = q_seq[t]
        # brute force on this query alone: scores of its candidates, best kk by repeated argmax
        row = index_scores(q[t:t + 1], w[t:t + 1], k[starts[b]:starts[b] + n], np.array([0]), np.array([0]),
                           np.array([n - 1]), n)[0]
        want = _select_by_repeated_argmax(list(row), kk)
        assert cnt[t] == len(want) == min(kk, n)
        assert idx[t, :cnt[t]].tolist() == want
        assert (idx[t, cnt[t]:] == -1).all()
    o_ref, l_ref = sparse_mla(qn, qp, m, 0.1, cache, 64, starts, q_seq, idx, cnt)
    np.testing.assert_array_equal(outs[0][0], o_ref)
    np.testing.assert_array_equal(outs[0][1], l_ref)


def test_forward_shares_one_selection_across_layers():
    q, w, k, starts, q_seq, q_pos, ld = _rand_index_case(T=2, lens=(300, 120))
    qn, qp, m, cache, _, _, _ = _rand_attn_case(T=2, lens=(300, 120))
    layers = [dict(q_nope=qn, q_pe=qp, qmul=m, cache=cache, d_rope=64),
              dict(q_nope=qn, q_pe=None, qmul=m, cache=np.ascontiguousarray(cache[:, :512]),
                   d_rope=0)]
    idx, cnt, outs = forward(q, w, k, starts, q_seq, q_pos, layers, 0.1, k=64)
    assert cnt.tolist() == [64, 64]
    for lay, (o, lse) in zip(layers, outs):
        o2, _ = sparse_mla(lay["q_nope"], lay["q_pe"], lay["qmul"], 0.1, lay["cache"],
                           lay["d_rope"], starts, q_seq, idx, cnt)
        np.testing.assert_array_equal(o, o2)
