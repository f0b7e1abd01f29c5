"""Failure detection on the GPU without a fault: a bounded pipeline wait that
runs out.  The attention kernel's testing hook makes every block skip the
gather of one tile, so the wait for it runs out after a short limit; the kernel
must unwind (copies drained, MMAs completed, tensor memory freed), report
DSA_ERR_TIMEOUT through dsa_check_errors, and leave the context usable: the
next call, with the hook off, must match the oracle."""

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
    ops.set_fault_test(0, -1)


def _selection(wl, seed):
    rng = np.random.default_rng(seed)
    q_pos = to_numpy(wl.q_pos)
    idx = np.full((wl.T, 2048), -1, np.int32)
    for t in range(wl.T):
        idx[t] = np.sort(rng.choice(int(q_pos[t]) + 1, 2048, replace=False))
    return torch.as_tensor(idx, device=DEV), torch.full((wl.T,), 2048, dtype=torch.int32, device=DEV)


def test_stalled_tile_times_out_then_the_next_call_is_clean():
    # 150 queries: every block holds at least two tiles, so tile 1 exists everywhere.
    T = 150
    case = small_case("stall", (2100,) * T, seed=61)
    wl = make_workload(case, DEV)
    idx, cnt = _selection(wl, 3)
    assert ops.plan_attend(T, 1, 2048).rows_per_split >= 128
    lay = wl.layers[0]
    out = torch.empty((T, 64, 512), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((T, 64), dtype=torch.float32, device=DEV)
    assert ops.check_errors() == 0
    ops.set_fault_test(20_000_000, 1)      # 20 ms limit; tile 1 is never gathered
    try:
        ops.sparse_mla_attend(lay.q_nope, lay.q_pe, lay.qmul, lay.cache, 64, wl.seq_row_start, wl.q_seq, idx,
                              cnt, out, lse)
        with pytest.raises(ops.DSAError) as err:
            ops.check_errors()
        assert err.value.status == 5        # DSA_ERR_TIMEOUT
        assert "0x8" in str(err.value)
    finally:
        ops.set_fault_test(0, -1)
    # the context is still usable and the next call is right
    ops.sparse_mla_attend(lay.q_nope, lay.q_pe, lay.qmul, lay.cache, 64, wl.seq_row_start, wl.q_seq, idx, cnt,
                          out, lse)
    assert ops.check_errors() == 0
    ts = [0, 77, 149]
    ref_o, ref_l = pu.oracle_attend(wl, lay, ts, to_numpy(idx), to_numpy(cnt))
    pu.assert_attention_close(to_numpy(out)[ts], to_numpy(lse)[ts], ref_o, ref_l)
