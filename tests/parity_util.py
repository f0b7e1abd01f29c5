"""Helpers for GPU-vs-oracle parity tests: run the C-ABI path on a workload and
compare against the fp64 oracle with the tolerances the benchmark spec fixes:

  indexer   |I_gpu - I_ref| <= 1e-3 * max(|I_ref|, rms of that query's row)
  top-k     bit-exact when both select from the same (GPU) score array
  selection end to end: set overlap >= 99.9%, misses only where neighbouring
            scores differ by < 1e-3 relative
  attention max |o_gpu - o_ref| <= 2e-2 (plus an internal bar: <= 1e-2 of max|o_ref| per query)
"""

from __future__ import annotations

import numpy as np
import torch

import oracle
from sparse_attention_16_b200 import ops
from sparse_attention_16_b200.workloads import SOFTMAX_SCALE, quantize_e4m3_rows, to_numpy

SCORE_RTOL = 1e-3
ATTN_ATOL = 2e-2
ATTN_REL = 1e-2     # internal bar: max error <= 1% of the query's largest |o|
LSE_ATOL = 2e-3


def gpu_scores(wl, ld=None, q_group=1):
    ld = ld or wl.case.ld
    scores = torch.empty((wl.T, ld), dtype=torch.float32, device=wl.q_idx.device)
    ops.index_scores(wl.q_idx, wl.w, wl.k_idx, wl.seq_row_start, wl.q_seq, wl.q_pos, scores,
                     q_group=q_group)
    return scores


def gpu_topk(scores, q_pos, k):
    T = scores.shape[0]
    idx = torch.empty((T, k), dtype=torch.int32, device=scores.device)
    cnt = torch.empty((T,), dtype=torch.int32, device=scores.device)
    ops.topk(scores, q_pos, k, idx, cnt)
    return idx, cnt


def gpu_attend(wl, layer, idx, cnt, with_lse=True):
    T = wl.T
    out = torch.empty((T, 64, 512), dtype=torch.bfloat16, device=idx.device)
    lse = torch.empty((T, 64), dtype=torch.float32, device=idx.device) if with_lse else None
    ops.sparse_mla_attend(layer.q_nope, layer.q_pe, layer.qmul, layer.cache, layer.d_rope,
                          wl.seq_row_start, wl.q_seq, idx, cnt, out, lse)
    return out, lse


def host_meta(wl):
    return (to_numpy(wl.seq_row_start), to_numpy(wl.q_seq), to_numpy(wl.q_pos))


def oracle_scores(wl, ts, ld):
    """Oracle score rows for the queries in ``ts`` (fetches only their key rows)."""
    starts, q_seq, q_pos = host_meta(wl)
    rows = []
    for t in ts:
        b = int(q_seq[t])
        n = int(q_pos[t]) + 1
        k = to_numpy(wl.k_idx[int(starts[b]):int(starts[b]) + n])
        rows.append(oracle.index_scores(to_numpy(wl.q_idx[t:t + 1]), to_numpy(wl.w[t:t + 1]), k,
                                        np.array([0]), np.array([0]), np.array([q_pos[t]]), ld)[0])
    return np.stack(rows)


def fp8_inputs(wl):
    """E4M3 codes and per-row scales of the workload's indexer queries and keys."""
    q8, qs = quantize_e4m3_rows(wl.q_idx)
    k8, ks = quantize_e4m3_rows(wl.k_idx)
    return q8, qs, k8, ks


def gpu_scores_fp8(wl, q8, qs, k8, ks, ld=None, q_group=1):
    ld = ld or wl.case.ld
    scores = torch.empty((wl.T, ld), dtype=torch.float32, device=wl.q_idx.device)
    ops.index_scores_fp8(q8, qs, wl.w, k8, ks, wl.seq_row_start, wl.q_seq, wl.q_pos, scores,
                         q_group=q_group)
    return scores


def oracle_scores_fp8(wl, q8, qs, k8, ks, ts, ld):
    """Oracle FP8-key score rows for the queries in ``ts`` (fetches only their key rows)."""
    starts, q_seq, q_pos = host_meta(wl)
    rows = []
    for t in ts:
        b = int(q_seq[t])
        n = int(q_pos[t]) + 1
        lo = int(starts[b])
        rows.append(oracle.index_scores_fp8(to_numpy(q8[t:t + 1]), to_numpy(qs[t:t + 1]), to_numpy(wl.w[t:t + 1]),
                                            to_numpy(k8[lo:lo + n]), to_numpy(ks[lo:lo + n]), np.array([0]),
                                            np.array([0]), np.array([q_pos[t]]), ld)[0])
    return np.stack(rows)


def assert_scores_close(gpu_rows, ref_rows, q_pos_rows):
    for g, r, qp in zip(gpu_rows, ref_rows, q_pos_rows):
        n = int(qp) + 1
        assert np.all(np.isneginf(g[n:])), "positions after q_pos must be -inf"
        rr = r[:n]
        rms = float(np.sqrt(np.mean(rr * rr))) if n else 0.0
        tol = SCORE_RTOL * np.maximum(np.abs(rr), rms)
        err = np.abs(g[:n].astype(np.float64) - rr)
        bad = err > tol
        assert not bad.any(), f"{bad.sum()} scores out of tolerance, worst {err.max():.3e}"


def assert_topk_exact(gpu_idx, gpu_cnt, scores_host, q_pos_host, k):
    ref_idx, ref_cnt = oracle.topk_select(scores_host, q_pos_host, k)
    np.testing.assert_array_equal(gpu_cnt, ref_cnt)
    np.testing.assert_array_equal(gpu_idx, ref_idx)


def assert_selection_overlap(gpu_sel, ref_scores_row, k, min_overlap=0.999):
    """End-to-end check: the GPU's selection (from its own fp32 scores) against the
    oracle's fp64 ranking; misses only at near-ties (< 1e-3 relative)."""
    n = ref_scores_row.shape[0]
    keff = min(k, n)
    order = np.lexsort((np.arange(n), -ref_scores_row))
    ref_set = set(order[:keff].tolist())
    got = set(int(x) for x in gpu_sel if x >= 0)
    assert len(got) == keff
    missed = ref_set - got
    assert len(got & ref_set) >= min_overlap * keff, f"overlap {len(got & ref_set)}/{keff}"
    if missed:
        thr = ref_scores_row[order[keff - 1]]
        scale = max(abs(thr), 1e-30)
        for m in missed:
            assert abs(ref_scores_row[m] - thr) <= 1e-3 * scale, "a miss that is not a near-tie"
        for e in got - ref_set:
            assert abs(ref_scores_row[e] - thr) <= 1e-3 * scale, "an extra that is not a near-tie"


def oracle_attend(wl, layer, ts, idx_host, cnt_host):
    """Oracle attention for queries ``ts`` using the given selection (host arrays)."""
    starts, q_seq, _ = host_meta(wl)
    outs, lses = [], []
    for t in ts:
        b = int(q_seq[t])
        sel = idx_host[t, :cnt_host[t]]
        sel = sel[sel >= 0]
        uniq = np.unique(sel)
        base = int(starts[b])
        rows_dev = torch.as_tensor(base + uniq, device=layer.cache.device, dtype=torch.int64)
        sub = to_numpy(layer.cache.index_select(0, rows_dev)) if len(uniq) else np.zeros(
            (0, layer.cache.shape[1]), np.float32)
        # remap the selection onto the compact sub-cache
        pos = np.searchsorted(uniq, sel)
        idx1 = np.full((1, max(1, len(pos))), -1, np.int32)
        idx1[0, :len(pos)] = pos
        qp = to_numpy(layer.q_pe[t:t + 1]) if layer.q_pe is not None else None
        o, l = oracle.sparse_mla(to_numpy(layer.q_nope[t:t + 1]), qp, to_numpy(layer.qmul[t:t + 1]),
                                 SOFTMAX_SCALE, sub, layer.d_rope, np.array([0]), np.array([0]),
                                 idx1, np.array([len(pos)]))
        outs.append(o[0])
        lses.append(l[0])
    return np.stack(outs), np.stack(lses)


def assert_attention_close(gpu_o, gpu_lse, ref_o, ref_lse):
    g = gpu_o.astype(np.float64)
    err = np.abs(g - ref_o)
    assert err.max() <= ATTN_ATOL, f"max abs err {err.max():.3e}"
    for t in range(ref_o.shape[0]):
        mx = float(np.abs(ref_o[t]).max())
        if mx > 0:
            assert err[t].max() <= ATTN_REL * mx + 1e-6, f"query {t}: max err {err[t].max():.3e} vs max|o| {mx:.3e}"
    if gpu_lse is not None:
        both_inf = np.isneginf(gpu_lse) & np.isneginf(ref_lse)
        d = np.abs(np.where(both_inf, 0.0, gpu_lse.astype(np.float64) - ref_lse))
        assert d.max() <= LSE_ATOL, f"lse err {d.max():.3e}"
