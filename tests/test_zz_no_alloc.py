"""sparse_mla_attend_noalloc: the attention call for callers that cannot allocate
device memory (code that is only handed its input and output buffers, such as a
plugin inside another framework's memory pool, where cudaMalloc would bypass the
pool and can synchronize the device).  Its split partials live in a fixed scratch
array inside the library instead of a caller workspace.

Checked through the C ABI against sparse_mla_attend (the entry point that takes a
workspace) and against the CPU oracle, with the attention tolerances used
everywhere else, on two calls in a row with different inputs, so stale scratch
contents from the first call would show up in the second.  This file is
collected last on purpose.
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


def _selection(wl, seed, k=2048):
    rng = np.random.default_rng(seed)
    q_pos = to_numpy(wl.q_pos)
    idx = np.full((wl.T, k), -1, np.int32)
    cnt = np.zeros(wl.T, np.int32)
    for t in range(wl.T):
        n = int(q_pos[t]) + 1
        c = min(k, n)
        idx[t, :c] = np.sort(rng.choice(n, c, replace=False))
        cnt[t] = c
    return torch.as_tensor(idx, device=DEV), torch.as_tensor(cnt, device=DEV)


def _both(wl, lay, idx, cnt):
    T = wl.T
    ref_o = torch.empty((T, 64, 512), dtype=torch.bfloat16, device=DEV)
    ref_l = torch.empty((T, 64), dtype=torch.float32, device=DEV)
    ops.sparse_mla_attend(lay.q_nope, lay.q_pe, lay.qmul, lay.cache, lay.d_rope, wl.seq_row_start, wl.q_seq,
                          idx, cnt, ref_o, ref_l)
    o = torch.full((T, 64, 512), float("nan"), dtype=torch.bfloat16, device=DEV)
    l = torch.full((T, 64), float("nan"), dtype=torch.float32, device=DEV)
    ops.sparse_mla_attend_noalloc(lay.q_nope, lay.q_pe, lay.qmul, lay.cache, lay.d_rope, wl.seq_row_start,
                                  wl.q_seq, idx, cnt, o, l)
    torch.cuda.synchronize()
    return o, l, ref_o, ref_l


def _scratch_batch():
    """A batch size and selection width whose split partials go through the
    scratch on this GPU (split across blocks that do not merge on chip, within
    the scratch limit)."""
    for k in (2048, 4096, 8192):
        for T in range(8, 0, -1):
            p = ops.plan_attend(T, 1, k)
            if p.workspace_bytes > 0 and T * p.n_split <= 128:
                return T, k
    pytest.fail("no batch of 1-8 queries uses the scratch on this GPU")


@pytest.mark.parametrize("d_rope", [64, 0])
def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row(d_rope):
    T, k = _scratch_batch()
    wl1 = make_workload(small_case("na1", (9000, 3000, 2500, 600, 4097, 90, 5000, 2100)[:T], layers=(d_rope,),
                                   seed=31), DEV)
    wl2 = make_workload(small_case("na2", (5000, 2048, 100, 8000, 3333, 777, 2200, 4100)[:T], layers=(d_rope,),
                                   seed=32, mla_q_std=1.0), DEV)
    for wl, seed in ((wl1, 1), (wl2, 2)):
        idx, cnt = _selection(wl, seed, k)
        o, l, ref_o, ref_l = _both(wl, wl.layers[0], idx, cnt)
        g, r = to_numpy(o).astype(np.float64), to_numpy(ref_o).astype(np.float64)
        assert np.abs(g - r).max() <= pu.ATTN_ATOL
        for t in range(wl.T):
            assert np.abs(g[t] - r[t]).max() <= pu.ATTN_REL * np.abs(r[t]).max() + 1e-6
        assert np.abs(to_numpy(l).astype(np.float64) - to_numpy(ref_l)).max() <= pu.LSE_ATOL
        # and against the oracle on the same selection
        ts = list(range(wl.T))
        o_ref, l_ref = pu.oracle_attend(wl, wl.layers[0], ts, to_numpy(idx), to_numpy(cnt))
        pu.assert_attention_close(to_numpy(o), to_numpy(l), o_ref, l_ref)
    assert ops.check_errors() == 0


def test_noalloc_rejects_more_partials_than_its_scratch_holds():
    # A batch (and selection width k) whose split plan needs more partials than
    # the fixed scratch holds, found from the library's plan for this GPU.
    case = next(((T, k) for k in (2048, 4096, 16384) for T in range(1, 149)
                 if ops.plan_attend(T, 1, k).workspace_bytes > 0 and T * ops.plan_attend(T, 1, k).n_split > 128),
                None)
    assert case is not None, "no batch exceeds the scratch on this GPU"
    T, k = case
    # Real buffers of the right sizes: the call must refuse before launching,
    # and nothing could read out of bounds even if it did not.
    wl = make_workload(small_case("na_rej", (2100,) * T, layers=(64,), seed=33), DEV)
    lay = wl.layers[0]
    idx = torch.zeros((T, k), dtype=torch.int32, device=DEV)
    cnt = torch.ones((T,), dtype=torch.int32, device=DEV)
    out = torch.empty((T, 64, 512), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ops.DSAError) as err:
        ops.sparse_mla_attend_noalloc(lay.q_nope, lay.q_pe, lay.qmul, lay.cache, lay.d_rope, wl.seq_row_start,
                                      wl.q_seq, idx, cnt, out)
    assert err.value.status == 6   # DSA_ERR_WORKSPACE
    assert "128" in str(err.value)
    torch.cuda.synchronize()
    assert ops.check_errors() == 0
