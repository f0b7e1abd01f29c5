"""Attention over latent caches kept in FP8 (E4M3 codes with one fp32 scale per
128 latent values and one for the rotary key; the report's serving section,
native FP8 KV cache), through the C ABI, against the oracle's sparse_mla_fp8 on
the same bytes.

The kernel widens each selected row to bf16 on chip (one rounding of
scale * value, relative error <= 2^-9), then computes as on a bf16 cache, so the
attention tolerances of the bf16 path apply.  Covered: RoPE and NoPE layers,
ragged selections with -1 holes and unsorted entries, the single-CTA, cluster-merge
and combine split plans, four layers in one launch, and the fused call.
"""

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_16_b200 import ops
from sparse_attention_16_b200.workloads import (CONFIGS, SOFTMAX_SCALE, latent_fp8_row_bytes, make_workload,
                                                quantize_latent_fp8, small_case, to_numpy)
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


def _fp8_caches(wl):
    caches = [quantize_latent_fp8(L.cache, L.d_rope) for L in wl.layers]
    for L, c in zip(wl.layers, caches):
        assert c.shape[1] == latent_fp8_row_bytes(L.d_rope)
    return caches


def _selection(wl, counts, seed, sort=True, holes=False):
    rng = np.random.default_rng(seed)
    q_pos = to_numpy(wl.q_pos)
    idx = np.full((wl.T, 2048), -1, np.int32)
    cnt = np.zeros(wl.T, np.int32)
    for t, c in enumerate(counts):
        n = int(q_pos[t]) + 1
        c = min(c, n)
        sel = rng.choice(n, c, replace=False)
        idx[t, :c] = np.sort(sel) if sort else sel
        if holes and c > 10:
            idx[t, 3] = -1
        cnt[t] = c
    return idx, cnt


def _oracle_fp8(wl, layer, cache8, ts, idx_host, cnt_host):
    """Oracle attention over the FP8 rows each query selected (only those rows leave the GPU)."""
    starts, q_seq, _ = pu.host_meta(wl)
    outs, lses = [], []
    for t in ts:
        sel = idx_host[t, :cnt_host[t]]
        sel = sel[sel >= 0]
        uniq = np.unique(sel)
        rows = torch.as_tensor(int(starts[q_seq[t]]) + uniq, device=DEV, dtype=torch.int64)
        sub = cache8.index_select(0, rows).cpu().numpy() if len(uniq) else np.zeros((0, cache8.shape[1]), np.uint8)
        pos = np.searchsorted(uniq, sel)
        idx1 = np.full((1, max(1, len(pos))), -1, np.int32)
        idx1[0, :len(pos)] = pos
        qp = to_numpy(layer.q_pe[t:t + 1]) if layer.q_pe is not None else None
        o, l = oracle.sparse_mla_fp8(to_numpy(layer.q_nope[t:t + 1]), qp, to_numpy(layer.qmul[t:t + 1]),
                                     SOFTMAX_SCALE, sub, layer.d_rope, np.array([0]), np.array([0]), idx1,
                                     np.array([len(pos)]))
        outs.append(o[0])
        lses.append(l[0])
    return np.stack(outs), np.stack(lses)


def _attend(wl, caches, idx, cnt, q_pos=None):
    T = wl.T
    outs = [torch.empty((T, 64, 512), dtype=torch.bfloat16, device=DEV) for _ in wl.layers]
    lses = [torch.empty((T, 64), dtype=torch.float32, device=DEV) for _ in wl.layers]
    layers = [dict(q_nope=L.q_nope, q_pe=L.q_pe, qmul=L.qmul, cache=c, d_rope=L.d_rope, out=o, lse=l)
              for L, c, o, l in zip(wl.layers, caches, outs, lses)]
    ops.sparse_mla_attend_layers(layers, caches[0].shape[0], wl.seq_row_start, wl.q_seq,
                                 torch.as_tensor(idx, device=DEV), torch.as_tensor(cnt, device=DEV), q_pos=q_pos)
    torch.cuda.synchronize()
    return outs, lses


@pytest.mark.parametrize("d_rope", [64, 0])
@pytest.mark.parametrize("sort", [True, False])
def test_fp8_cache_attention_matches_oracle(d_rope, sort):
    # 5 queries: each selection is split over several CTAs (combine path).
    case = small_case("fp8c_split", (4096, 3000, 2100, 600, 50), layers=(d_rope,), seed=41)
    wl = make_workload(case, DEV)
    caches = _fp8_caches(wl)
    idx, cnt = _selection(wl, [2048, 1500, 2048, 129, 37], seed=5, sort=sort, holes=not sort)
    plan = ops.plan_attend(wl.T, 1, 2048, ops.device_props())
    assert plan.n_split > 1
    outs, lses = _attend(wl, caches, idx, cnt, q_pos=wl.q_pos)
    ref_o, ref_l = _oracle_fp8(wl, wl.layers[0], caches[0], range(wl.T), idx, cnt)
    pu.assert_attention_close(to_numpy(outs[0]), to_numpy(lses[0]), ref_o, ref_l)
    assert ops.check_errors() == 0


def test_fp8_cache_four_layers_in_one_launch():
    # Three RoPE layers and one NoPE layer over one selection, four queries: the
    # 1M-context decode's launch shape (16 units split into partials + combine).
    case = small_case("fp8c_layers", (6000, 3000, 2100, 900), layers=(64, 64, 64, 0), seed=42)
    wl = make_workload(case, DEV)
    caches = _fp8_caches(wl)
    idx, cnt = _selection(wl, [2048, 2048, 2048, 900], seed=6, sort=False, holes=True)
    outs, lses = _attend(wl, caches, idx, cnt, q_pos=wl.q_pos)
    for lay, c, o, l in zip(wl.layers, caches, outs, lses):
        ref_o, ref_l = _oracle_fp8(wl, lay, c, range(wl.T), idx, cnt)
        pu.assert_attention_close(to_numpy(o), to_numpy(l), ref_o, ref_l)
    assert ops.check_errors() == 0


def test_fp8_cache_cluster_merge_and_single_split():
    # 64 queries: two CTAs per query merging in a cluster; 160 queries: one CTA
    # per query (every 64-row tile of a 2,048-row selection in one CTA).
    props = ops.device_props()
    for T, seed in ((64, 43), (160, 44)):
        plan = ops.plan_attend(T, 1, 2048, props)
        lengths = tuple(3000 + 37 * i for i in range(T))
        wl = make_workload(small_case(f"fp8c_{T}", lengths, layers=(64,), seed=seed), DEV)
        caches = _fp8_caches(wl)
        idx, cnt = _selection(wl, [2048 - 13 * (i % 5) for i in range(T)], seed=seed)
        outs, lses = _attend(wl, caches, idx, cnt, q_pos=wl.q_pos)
        ts = sorted({0, 1, T // 2, T - 1})
        ref_o, ref_l = _oracle_fp8(wl, wl.layers[0], caches[0], ts, idx, cnt)
        pu.assert_attention_close(to_numpy(outs[0])[ts], to_numpy(lses[0])[ts], ref_o, ref_l)
        if T == 64:
            assert plan.merge == 1 or plan.n_split == 1
    assert ops.check_errors() == 0


def test_fp8_cache_matches_bf16_path_on_exact_values():
    # Unit scales and codes whose values are bf16 numbers: the widened tile is
    # exactly the bf16 cache holding those values, so the FP8 path must give the
    # bf16 path's bits.
    case = small_case("fp8c_exact", (2500, 1300, 700), layers=(64,), seed=45)
    wl = make_workload(case, DEV)
    L = wl.layers[0]
    rows = L.cache.shape[0]
    g = torch.Generator(device="cpu").manual_seed(45)
    codes = torch.randint(0, 256, (rows, 576), generator=g, dtype=torch.int32).to(torch.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x38
    vals = codes.view(torch.float8_e4m3fn).float()
    c8 = torch.zeros((rows, latent_fp8_row_bytes(64)), dtype=torch.uint8)
    c8[:, :576] = codes
    c8[:, 576:596] = torch.ones((rows, 5), dtype=torch.float32).view(torch.uint8)
    c8 = c8.to(DEV)
    cache_bf16 = vals.to(torch.bfloat16).to(DEV)
    assert torch.equal(cache_bf16.float().cpu(), vals)
    idx, cnt = _selection(wl, [2048, 1000, 640], seed=7)
    o8, l8 = _attend(wl, [c8], idx, cnt)
    ob = torch.empty_like(o8[0])
    lb = torch.empty_like(l8[0])
    ops.sparse_mla_attend_layers([dict(q_nope=L.q_nope, q_pe=L.q_pe, qmul=L.qmul, cache=cache_bf16, d_rope=64,
                                       out=ob, lse=lb)], rows, wl.seq_row_start, wl.q_seq,
                                 torch.as_tensor(idx, device=DEV), torch.as_tensor(cnt, device=DEV))
    torch.cuda.synchronize()
    assert torch.equal(o8[0], ob)
    assert torch.equal(l8[0], lb)


def test_fp8_cache_in_the_fused_call():
    # dsa_sparse_mla_forward with FP8 latent caches: the selection is the bf16
    # index path's (bit-exact top-k of the GPU scores) and every layer matches
    # the oracle's FP8 attention over it.
    case = small_case("fp8c_fwd", (5000, 2500, 800, 37), layers=(64, 0), seed=46)
    wl = make_workload(case, DEV)
    caches = _fp8_caches(wl)
    T, k = wl.T, 2048
    ld = int(to_numpy(wl.q_pos).max()) + 1
    ld = (ld + 3) // 4 * 4
    outs = [torch.empty((T, 64, 512), dtype=torch.bfloat16, device=DEV) for _ in wl.layers]
    lses = [torch.empty((T, 64), dtype=torch.float32, device=DEV) for _ in wl.layers]
    layers = [dict(q_nope=L.q_nope, q_pe=L.q_pe, qmul=L.qmul, cache=c, d_rope=L.d_rope, out=o, lse=l)
              for L, c, o, l in zip(wl.layers, caches, outs, lses)]
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    cnt = torch.empty((T,), dtype=torch.int32, device=DEV)
    ops.sparse_mla_forward(wl.q_idx, wl.w, wl.k_idx, wl.seq_row_start, wl.q_seq, wl.q_pos, layers, ld=ld, k=k,
                           idx_out=idx, count_out=cnt)
    torch.cuda.synchronize()
    scores = pu.gpu_scores(wl, ld)
    idx_ref, cnt_ref = pu.gpu_topk(scores, wl.q_pos, k)
    assert torch.equal(idx, idx_ref) and torch.equal(cnt, cnt_ref)
    idx_h, cnt_h = to_numpy(idx), to_numpy(cnt)
    for lay, c, o, l in zip(wl.layers, caches, outs, lses):
        ref_o, ref_l = _oracle_fp8(wl, lay, c, range(T), idx_h, cnt_h)
        pu.assert_attention_close(to_numpy(o), to_numpy(l), ref_o, ref_l)
    assert ops.check_errors() == 0
