"""Full-size configurations, in the launch configuration bench.py times (the fused
forward call), checked on sampled queries that the oracle computes one by one:

  * score rows of the sampled queries within 1e-3 relative (separate indexer call)
  * the fused call's selection equals the oracle's top-k of the GPU score row
    (bit-exact), and overlaps the oracle's fp64 ranking >= 99.9% with misses only
    at near-ties
  * attention output of every layer within 2e-2 of the oracle on that selection
"""

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_16_b200 import ops
from sparse_attention_16_b200.workloads import CONFIGS, make_workload, to_numpy
from tests import parity_util as pu

pytestmark = pytest.mark.gpu
DEV = "cuda"

SAMPLES = {
    "decode_b64_32k": [0, 31, 63],
    "decode_b16_128k_planted": [0, 9, 15],
    "prefill_32k_plus_8k": [0, 1, 8, 4095, 8191],
    "decode_b4_1m_4layers": [0, 3],
}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    ops.load_library()
    yield


@pytest.mark.parametrize("name", list(SAMPLES))
def test_fullsize_config_sampled_parity(name):
    case = CONFIGS[name]
    wl = make_workload(case, DEV)
    T, ld = wl.T, case.ld
    q_group = 8 if case.kind == "prefill" else 1
    outs = [torch.empty((T, 64, 512), dtype=torch.bfloat16, device=DEV) for _ in wl.layers]
    lses = [torch.empty((T, 64), dtype=torch.float32, device=DEV) for _ in wl.layers]
    layers = [dict(q_nope=L.q_nope, q_pe=L.q_pe, qmul=L.qmul, cache=L.cache, d_rope=L.d_rope, out=o,
                   lse=l) for L, o, l in zip(wl.layers, outs, lses)]
    idx = torch.empty((T, 2048), dtype=torch.int32, device=DEV)
    cnt = torch.empty((T,), dtype=torch.int32, device=DEV)
    ops.sparse_mla_forward(wl.q_idx, wl.w, wl.k_idx, wl.seq_row_start, wl.q_seq, wl.q_pos, layers, ld,
                           q_group=q_group, idx_out=idx, count_out=cnt)
    assert ops.check_errors() == 0

    ts = SAMPLES[name]
    scores = pu.gpu_scores(wl, ld, q_group=q_group)
    s_rows = to_numpy(scores[ts]).astype(np.float64)
    del scores
    q_pos = to_numpy(wl.q_pos)
    ref_rows = pu.oracle_scores(wl, ts, ld)
    pu.assert_scores_close(s_rows, ref_rows, q_pos[ts])

    idx_h, cnt_h = to_numpy(idx), to_numpy(cnt)
    ref_idx, ref_cnt = oracle.topk_select(s_rows, q_pos[ts], 2048)
    np.testing.assert_array_equal(idx_h[ts], ref_idx)
    np.testing.assert_array_equal(cnt_h[ts], ref_cnt)
    for i, t in enumerate(ts):
        n = int(q_pos[t]) + 1
        pu.assert_selection_overlap(idx_h[t, :cnt_h[t]], ref_rows[i, :n], 2048)

    if wl.planted_pos is not None:
        planted = to_numpy(wl.planted_pos)
        for t in ts:   # decode: query t belongs to sequence t
            assert set(planted[t].tolist()) <= set(idx_h[t, :cnt_h[t]].tolist())

    for L, o, l in zip(wl.layers, outs, lses):
        ref_o, ref_l = pu.oracle_attend(wl, L, ts, idx_h, cnt_h)
        pu.assert_attention_close(to_numpy(o)[ts], to_numpy(l)[ts], ref_o, ref_l)


def test_fullsize_one_million_decode_with_fp8_latent_caches():
    # The 1M x 4-layer decode with every latent cache kept as FP8 rows (the
    # report's native FP8 KV cache), in the fused launch: the selection is the
    # bf16 index path's, and each layer's attention on sampled queries matches
    # the oracle's FP8 attention over the same bytes.
    from sparse_attention_16_b200.workloads import quantize_latent_fp8
    from tests.test_gpu_fp8_cache import _oracle_fp8

    case = CONFIGS["decode_b4_1m_4layers"]
    wl = make_workload(case, DEV)
    T, ld = wl.T, case.ld
    caches = []
    for L in wl.layers:
        caches.append(quantize_latent_fp8(L.cache, L.d_rope))
        L.cache = None
    torch.cuda.empty_cache()
    outs = [torch.empty((T, 64, 512), dtype=torch.bfloat16, device=DEV) for _ in wl.layers]
    lses = [torch.empty((T, 64), dtype=torch.float32, device=DEV) for _ in wl.layers]
    layers = [dict(q_nope=L.q_nope, q_pe=L.q_pe, qmul=L.qmul, cache=c, d_rope=L.d_rope, out=o, lse=l)
              for L, c, o, l in zip(wl.layers, caches, outs, lses)]
    idx = torch.empty((T, 2048), dtype=torch.int32, device=DEV)
    cnt = torch.empty((T,), dtype=torch.int32, device=DEV)
    ops.sparse_mla_forward(wl.q_idx, wl.w, wl.k_idx, wl.seq_row_start, wl.q_seq, wl.q_pos, layers, ld,
                           idx_out=idx, count_out=cnt)
    assert ops.check_errors() == 0
    ts = [0, 3]
    idx_h, cnt_h = to_numpy(idx), to_numpy(cnt)
    assert (cnt_h == 2048).all()
    for L, c, o, l in zip(wl.layers, caches, outs, lses):
        ref_o, ref_l = _oracle_fp8(wl, L, c, ts, idx_h, cnt_h)
        pu.assert_attention_close(to_numpy(o)[ts], to_numpy(l)[ts], ref_o, ref_l)
