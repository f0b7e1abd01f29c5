"""The C-ABI library loads on a machine without a GPU, exports every symbol
include/dsa.h declares, and rejects bad arguments on the host before launching
anything."""

import ctypes
import os
import re

import pytest

from sparse_attention_16_b200 import build, ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ops.load_library()


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "dsa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return set(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M))


def test_header_declares_the_four_hot_path_calls():
    names = _declared_functions()
    for n in ("dsa_index_scores", "dsa_topk", "sparse_mla_attend", "dsa_sparse_mla_forward"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    names = _declared_functions()
    assert names, "no declarations parsed"
    for n in names:
        assert hasattr(lib, n), n
    assert names == set(ops.SIGNATURES)


def test_version(lib):
    assert lib.dsa_version() == 100


NULL = None


def test_index_scores_rejects_bad_arguments(lib):
    fake = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    args = [fake, fake, fake, 100, fake, 1, fake, fake, 4, 1, fake, 128, NULL]
    bad = {
        8: -1,     # T < 0
        9: 3,      # q_group not in {1, 8}
        11: 130,   # ld % 4 != 0
        3: 0,      # n_rows < 1
        5: 0,      # B < 1
    }
    for pos, val in bad.items():
        a = list(args)
        a[pos] = val
        assert lib.dsa_index_scores(*a) == 1, pos
        assert lib.dsa_last_error()
    a = list(args)
    a[0] = NULL
    assert lib.dsa_index_scores(*a) == 1
    a = list(args)
    a[0] = ctypes.c_void_p(258)  # misaligned
    assert lib.dsa_index_scores(*a) == 1


def test_topk_rejects_bad_arguments(lib):
    fake = ctypes.c_void_p(256)
    ok = [fake, 1024, fake, 3, 2048, fake, fake, NULL, 0, NULL]
    for pos, val in [(4, 0), (4, 16385), (1, 1022), (3, -5)]:
        a = list(ok)
        a[pos] = val
        assert lib.dsa_topk(*a) == 1, (pos, val)
    assert lib.dsa_topk(fake, 1024, fake, 0, 2048, fake, fake, NULL, 0, NULL) == 0  # T == 0: no-op


def test_attend_rejects_bad_arguments(lib):
    fake = ctypes.c_void_p(256)
    ok = [fake, fake, fake, 0.07, fake, 1000, 576, 64, fake, 1, fake, fake, fake, 4, 2048, fake, NULL,
          NULL, 0, NULL]
    cases = {7: 32, 6: 500, 14: 0}
    for pos, val in cases.items():
        a = list(ok)
        a[pos] = val
        assert lib.sparse_mla_attend(*a) == 1, (pos, val)
    a = list(ok)
    a[1] = NULL          # q_pe missing on a RoPE layer
    assert lib.sparse_mla_attend(*a) == 1
    a = list(ok)
    a[7] = 0             # NoPE layer but q_pe given
    a[6] = 512
    assert lib.sparse_mla_attend(*a) == 1


def test_forward_rejects_missing_workspace(lib):
    fake = ctypes.c_void_p(256)
    layers = (ops.LayerArgs * 1)(ops.LayerArgs(256, 256, 256, 256, 576, 64, 256, None))
    st = lib.dsa_sparse_mla_forward(fake, fake, fake, 1000, fake, 1, fake, fake, 4, 1, 1024, 1, layers,
                                    0.07, 2048, NULL, NULL, NULL, 0, NULL)
    assert st == 1


def test_workspace_sizes_are_host_only(lib):
    assert lib.dsa_topk_workspace_size(64, 32768, 2048) == 0
    assert lib.sparse_mla_workspace_size(0, 2048) == 0
    # 4 queries are split 16+ ways (more than one cluster merges): partial
    # numerators go through the workspace.  2-8 way splits merge inside a
    # cluster when the GPU allows it, so their size depends on the device.
    assert lib.sparse_mla_workspace_size(4, 2048) >= 4 * 16 * 64 * 512 * 4
    assert lib.dsa_forward_workspace_size(64, 32768, 2048, 1) >= 64 * 32768 * 4
