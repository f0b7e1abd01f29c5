"""The FP8 (E4M3) index-key indexer (dsa_index_scores_fp8) against the oracle's
index_scores_fp8 on the same codes and scales, through the C ABI.

Keys and queries are encoded per row (scale = row max / 448) from the seeded
bf16 inputs; both sides receive the same bytes.  Scores must agree within the
indexer tolerance (1e-3 relative, rms floor); integer codes with power-of-two
scales make every product and sum exact, so there the match is bit for bit.
"""

import numpy as np
import pytest
import torch

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


CASES = [
    small_case("fp8_ragged", (4096, 4096, 1500, 37, 129, 128, 1), seed=21),
    small_case("fp8_one_long", (20000,), seed=22),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c.name)
def test_fp8_indexer_matches_oracle_decode(case):
    wl = make_workload(case, DEV)
    q8, qs, k8, ks = pu.fp8_inputs(wl)
    s = pu.gpu_scores_fp8(wl, q8, qs, k8, ks)
    ref = pu.oracle_scores_fp8(wl, q8, qs, k8, ks, list(range(wl.T)), case.ld)
    pu.assert_scores_close(to_numpy(s), ref, to_numpy(wl.q_pos))
    assert ops.check_errors() == 0


@pytest.mark.parametrize("new", [45, 8])
def test_fp8_indexer_matches_oracle_prefill_groups(new):
    case = small_case(f"fp8_prefill_{new}", kind="prefill", cached=700, new=new, seed=24)
    wl = make_workload(case, DEV)
    q8, qs, k8, ks = pu.fp8_inputs(wl)
    ref = pu.oracle_scores_fp8(wl, q8, qs, k8, ks, list(range(wl.T)), case.ld)
    for qg in (8, 1):
        s = pu.gpu_scores_fp8(wl, q8, qs, k8, ks, q_group=qg)
        pu.assert_scores_close(to_numpy(s), ref, to_numpy(wl.q_pos))


def test_fp8_indexer_integer_codes_are_bit_exact():
    # Codes of -3..3 with power-of-two scales and dyadic w: every product and
    # partial sum is exact in fp32, so the scores must equal the oracle's.
    case = small_case("fp8_int", (3000, 700, 130), seed=25)
    wl = make_workload(case, DEV)
    table = torch.tensor([0xC4, 0xC0, 0xB8, 0x00, 0x38, 0x40, 0x44], dtype=torch.uint8, device=DEV)  # -3..3
    g = torch.Generator(device=DEV).manual_seed(6)
    q8 = table[torch.randint(0, 7, tuple(wl.q_idx.shape), generator=g, device=DEV)].contiguous()
    k8 = table[torch.randint(0, 7, tuple(wl.k_idx.shape), generator=g, device=DEV)].contiguous()
    qs = torch.pow(2.0, torch.randint(-2, 3, (wl.T, 32), generator=g, device=DEV).float()).contiguous()
    ks = torch.pow(2.0, torch.randint(-2, 3, (wl.k_idx.shape[0],), generator=g, device=DEV).float()).contiguous()
    wl.w = (torch.randint(-8, 9, wl.w.shape, generator=g, device=DEV).float() / 4.0).contiguous()
    s = to_numpy(pu.gpu_scores_fp8(wl, q8, qs, k8, ks))
    ref = pu.oracle_scores_fp8(wl, q8, qs, k8, ks, list(range(wl.T)), case.ld)
    qp = to_numpy(wl.q_pos)
    for t in range(wl.T):
        n = qp[t] + 1
        np.testing.assert_array_equal(s[t, :n].astype(np.float64), ref[t, :n])
        assert np.all(np.isneginf(s[t, n:]))


def test_fp8_selection_overlaps_bf16_selection():
    # The FP8 keys are a coarser encoding of the same keys: the top-2048 chosen
    # from FP8 scores is close to the bf16 one (a property, not a tolerance of
    # the kernel; the kernel itself is checked above against its own oracle).
    case = small_case("fp8_vs_bf16", (32768,), seed=26)
    wl = make_workload(case, DEV)
    q8, qs, k8, ks = pu.fp8_inputs(wl)
    s8 = pu.gpu_scores_fp8(wl, q8, qs, k8, ks)
    s16 = pu.gpu_scores(wl)
    i8, _ = pu.gpu_topk(s8, wl.q_pos, 2048)
    i16, _ = pu.gpu_topk(s16, wl.q_pos, 2048)
    a, b = set(to_numpy(i8)[0].tolist()), set(to_numpy(i16)[0].tolist())
    assert len(a & b) / 2048 > 0.8


@pytest.mark.parametrize("per_seq,q_group", [(1, 1), (4, 4)])
def test_fused_forward_with_fp8_keys(per_seq, q_group):
    # The fused call on FP8 (E4M3) index keys: the selection is the top-k of the
    # FP8 indexer's own scores (bit-exact against the separate calls), overlaps
    # the oracle's fp64 FP8 ranking, and the attention matches the oracle.
    lengths = (7000, 4096, 2500, 900) if per_seq == 1 else (6000, 3000)
    case = small_case("fwd_fp8", lengths, layers=(64, 0), seed=36, per_seq=per_seq)
    wl = make_workload(case, DEV)
    T, ld = wl.T, case.ld
    q8, qs, k8, ks = pu.fp8_inputs(wl)
    outs = [torch.empty((T, 64, 512), dtype=torch.bfloat16, device=DEV) for _ in wl.layers]
    lses = [torch.empty((T, 64), dtype=torch.float32, device=DEV) for _ in wl.layers]
    layers = [dict(q_nope=L.q_nope, q_pe=L.q_pe, qmul=L.qmul, cache=L.cache, d_rope=L.d_rope, out=o, lse=l)
              for L, o, l in zip(wl.layers, outs, lses)]
    idx = torch.empty((T, 2048), dtype=torch.int32, device=DEV)
    cnt = torch.empty((T,), dtype=torch.int32, device=DEV)
    ops.sparse_mla_forward_fp8(q8, qs, wl.w, k8, ks, wl.seq_row_start, wl.q_seq, wl.q_pos, layers, ld,
                               q_group=q_group, idx_out=idx, count_out=cnt)
    assert ops.check_errors() == 0
    s = pu.gpu_scores_fp8(wl, q8, qs, k8, ks, q_group=q_group)
    idx2, cnt2 = pu.gpu_topk(s, wl.q_pos, 2048)
    assert torch.equal(idx, idx2) and torch.equal(cnt, cnt2)
    idx_h, cnt_h = to_numpy(idx), to_numpy(cnt)
    q_pos = to_numpy(wl.q_pos)
    ref_s = pu.oracle_scores_fp8(wl, q8, qs, k8, ks, list(range(T)), ld)
    for t in range(T):
        pu.assert_selection_overlap(idx_h[t, :cnt_h[t]], ref_s[t, :int(q_pos[t]) + 1], 2048)
    for L, o, l in zip(wl.layers, outs, lses):
        ref_o, ref_l = pu.oracle_attend(wl, L, list(range(T)), idx_h, cnt_h)
        pu.assert_attention_close(to_numpy(o), to_numpy(l), ref_o, ref_l)
