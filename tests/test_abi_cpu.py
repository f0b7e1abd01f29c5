"""The C-ABI library loads on a machine without a GPU, exports every symbol
include/dsa.h declares, and rejects bad arguments on the host before launching
anything."""

import ctypes
import os
import re

import numpy as np
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
    assert lib.dsa_version() == 201


NULL = None


def test_index_scores_rejects_bad_arguments(lib):
    fake = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    args = [fake, fake, fake, 100, fake, 1, fake, fake, 4, 1, fake, 128, NULL, NULL]
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
    a = list(args)
    a[9], a[12] = 8, fake        # a histogram needs q_group 1
    assert lib.dsa_index_scores(*a) == 1


def test_topk_rejects_bad_arguments(lib):
    fake = ctypes.c_void_p(256)
    ok = [fake, 1024, fake, 3, 2048, fake, fake, NULL, NULL, 0, NULL]
    for pos, val in [(4, 0), (4, 16385), (1, 1022), (3, -5), (7, ctypes.c_void_p(260))]:
        a = list(ok)
        a[pos] = val
        assert lib.dsa_topk(*a) == 1, (pos, val)
    assert lib.dsa_topk(fake, 1024, fake, 0, 2048, fake, fake, NULL, NULL, 0, NULL) == 0  # T == 0: no-op


def test_attend_rejects_bad_arguments(lib):
    fake = ctypes.c_void_p(256)
    # q_nope q_pe qmul scale cache n_rows ld_c d_rope seq_row_start B q_seq q_pos idx count T k out lse ws ws_bytes stream
    ok = [fake, fake, fake, 0.07, fake, 1000, 576, 64, fake, 1, fake, NULL, fake, fake, 4, 2048, fake, NULL,
          NULL, 0, NULL]
    cases = {7: 32, 6: 500, 15: 0, 14: -1, 9: 0}
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
    a = list(ok)
    a[11] = ctypes.c_void_p(258)   # misaligned q_pos
    assert lib.sparse_mla_attend(*a) == 1
    a = list(ok)
    a[14] = 0            # T == 0: no-op, nothing launched
    assert lib.sparse_mla_attend(*a) == 0


def test_attend_layers_rejects_bad_arguments(lib):
    fake = ctypes.c_void_p(256)
    good = ops.LayerArgs(256, 256, 256, 256, 576, 64, 256, None)
    bad = ops.LayerArgs(256, None, 256, 256, 576, 64, 256, None)    # RoPE layer without q_pe
    for layers, want in (((good, bad), 1), ((good, good), 0)):
        arr = (ops.LayerArgs * 2)(*layers)
        # T = 0 so that a valid call launches nothing
        st = lib.sparse_mla_attend_layers(2, arr, 0.07, 1000, fake, 1, fake, NULL, fake, fake, 0, 2048, NULL, 0,
                                          NULL)
        assert st == want
    assert lib.sparse_mla_attend_layers(2, None, 0.07, 1000, fake, 1, fake, NULL, fake, fake, 4, 2048, NULL, 0,
                                        NULL) == 1


def test_fp8_cache_rows_are_validated(lib):
    # FP8 latent rows: ld_c in bytes, a multiple of 16, at least codes + scales
    # (608 RoPE, 528 NoPE); every layer of a call uses one cache format.
    fake = ctypes.c_void_p(256)

    def layer(q_pe, ld_c, d_rope, fp8):
        return ops.LayerArgs(256, q_pe, 256, 256, ld_c, d_rope, 256, None, 0, fp8)

    cases = (
        ((layer(256, 608, 64, 1),), 0),
        ((layer(None, 528, 0, 1),), 0),
        ((layer(256, 592, 64, 1),), 1),        # scales do not fit
        ((layer(256, 600, 64, 1),), 1),        # not a multiple of 16
        ((layer(None, 512, 0, 1),), 1),
        ((layer(256, 608, 64, 2),), 1),        # unknown format
        ((layer(256, 608, 64, 1), layer(256, 576, 64, 0)), 1),   # mixed formats
        ((layer(256, 576, 64, 0), layer(None, 512, 0, 0)), 0),
    )
    for layers, want in cases:
        arr = (ops.LayerArgs * len(layers))(*layers)
        st = lib.sparse_mla_attend_layers(len(layers), arr, 0.07, 1000, fake, 1, fake, NULL, fake, fake, 0, 2048,
                                          NULL, 0, NULL)
        assert st == want, (layers, want)


def test_forward_rejects_missing_workspace(lib):
    fake = ctypes.c_void_p(256)
    layers = (ops.LayerArgs * 1)(ops.LayerArgs(256, 256, 256, 256, 576, 64, 256, None))
    st = lib.dsa_sparse_mla_forward(fake, fake, fake, 1000, fake, 1, fake, fake, 4, 1, 1024, 1, layers,
                                    0.07, 2048, NULL, NULL, NULL, 0, NULL)
    assert st == 1


def test_fault_test_hook_is_host_only(lib):
    assert lib.dsa_set_fault_test(20_000_000, 1) == 0
    assert lib.dsa_set_fault_test(0, -1) == 0


# ------------------------------------------------------------------ launch planning (explicit device properties)

PER_PARTIAL = 64 * (512 + 4) * 4          # one (query, split) partial: 64 heads x (512 + 4) fp32

# SM count and resident clusters of 2..8 attention blocks: none merge; a B200-like
# residency (clusters must fit a GPC); everything resident; a smaller GPU.
PROPS = {
    "no_merge": (148, {}),
    "b200_like": (148, {2: 74, 3: 48, 4: 32, 5: 24, 6: 16, 7: 16, 8: 16}),
    "all_resident": (148, {c: 148 // c for c in range(2, 9)}),
    "small_gpu": (60, {2: 30, 3: 18, 4: 12, 5: 6, 6: 6, 7: 6, 8: 6}),
}


def _props(name):
    sms, mc = PROPS[name]
    return ops.make_props(sms, mc)


@pytest.mark.parametrize("name", sorted(PROPS))
def test_attend_plan_covers_every_row_and_fits_its_workspace(lib, name):
    props = _props(name)
    sms, mc = PROPS[name]
    for k in (1, 37, 64, 700, 2048, 4096):
        for T in list(range(1, 40)) + [64, 100, 147, 148, 149, 300, 1000]:
            for n_layers in (1, 2, 4, 8):
                p = ops.plan_attend(T, n_layers, k, props)
                units = T * n_layers
                assert 1 <= p.n_split <= 32 and p.rows_per_split % 64 == 0
                assert p.n_split * p.rows_per_split >= k > (p.n_split - 1) * p.rows_per_split
                if p.merge:
                    assert 2 <= p.n_split <= 8 and units <= mc.get(p.n_split, 0)
                    assert p.workspace_bytes == 0
                elif p.n_split > 1:
                    assert p.workspace_bytes >= units * p.n_split * PER_PARTIAL
                else:
                    assert p.workspace_bytes == 0


def _check_forward_layout(lib, T, ld, k, q_group, n_layers, has_idx, has_cnt, ws, props):
    try:
        f = ops.plan_forward(T, ld, k, q_group, n_layers, has_idx, has_cnt, ws, props)
    except ops.DSAError as e:
        assert e.status == 6
        return None
    assert 1 <= f.chunk <= T and f.end <= ws
    assert f.chunk == T or f.chunk % q_group == 0
    assert f.n_chunks == -(-T // f.chunk) and f.last_chunk == T - (f.n_chunks - 1) * f.chunk > 0
    # every chunk size the call runs, with every layer group it launches: the
    # attention plan's partials fit the region reserved for them
    groups = {min(n_layers, 8)} | ({n_layers % 8} if n_layers > 8 and n_layers % 8 else set())
    for n in {f.chunk, f.last_chunk}:
        for g in groups:
            if g:
                need = ops.plan_attend(n, g, k, props, allow_partials=bool(f.attend_partials)).workspace_bytes
                assert need <= f.attend_bytes, (T, ws, n, g, need, f.attend_bytes)
    # regions in order, disjoint, inside the workspace
    regions = []
    if not has_idx:
        regions.append((f.idx_offset, f.chunk * k * 4))
    if not has_cnt:
        regions.append((f.count_offset, f.chunk * 4))
    regions.append((f.attend_offset, f.attend_bytes))
    if q_group == 1:
        regions += [(f.hist_offset, f.chunk * 2048 * 4), (f.topk_offset, f.topk_bytes)]
        if ld <= 40960:
            assert f.topk_bytes == 0                       # rows selected from shared memory
        else:
            assert f.topk_bytes >= 2 * f.chunk * 10240 * 4     # at least one candidate list per query
    else:
        assert f.hist_offset == f.topk_offset == 2 ** 64 - 1
    regions.append((f.scores_offset, f.chunk * ld * 4))
    end = 0
    for off, size in regions:
        assert off >= end and off % 256 == 0
        end = off + size
    assert end <= f.end <= ws
    return f


@pytest.mark.parametrize("name", sorted(PROPS))
def test_forward_chunks_stay_inside_the_workspace(lib, name):
    # Sweep batch sizes and workspaces, including workspaces sized for another
    # batch (the tail chunk is then planned differently from the full chunks).
    props = _props(name)
    k = 2048
    rng = np.random.default_rng(5)
    Ts = sorted(set(list(range(1, 200)) + [int(x) for x in rng.integers(200, 2049, size=40)] + [2048]))
    for T in Ts:
        for ld, q_group, n_layers in ((4096, 1, 1), (32768, 1, 4), (41_000, 8, 2)):
            full = ops.plan_forward(T, ld, k, q_group, n_layers, 0, 0, 1 << 60, props).end
            sizes = {full, full - 1, full // 2, full // 3, full // 7 + 12345}
            for other in (1, 8, 16, 75, 148, 150):
                try:
                    sizes.add(ops.plan_forward(other, ld, k, q_group, n_layers, 0, 0, 1 << 60, props).end)
                except ops.DSAError:
                    pass
            for ws in sorted(sizes):
                for has_idx, has_cnt in ((0, 0), (1, 1)):
                    _check_forward_layout(lib, T, ld, k, q_group, n_layers, has_idx, has_cnt, ws, props)


def test_forward_tail_chunk_regression(lib):
    # 151 decode queries at context 4,096 with a workspace sized for 148: the
    # old layout reserved partials for the full chunks only, and a 1-query tail
    # split 32 ways wrote ~1.2 MB past the end of the workspace.
    props = _props("b200_like")
    ws = ops.plan_forward(148, 4096, 2048, 1, 1, 0, 0, 1 << 60, props).end
    f = _check_forward_layout(lib, 151, 4096, 2048, 1, 1, 0, 0, ws, props)
    assert f is not None and f.end <= ws
    assert f.n_chunks > 1


def test_workspace_sizes_need_a_device_or_explicit_props(lib):
    # Without a GPU the size queries of the current device answer 0 (no device
    # to plan for); the planning queries with explicit properties still work.
    assert lib.dsa_topk_workspace_size(64, 32768, 2048) == 0
    assert lib.sparse_mla_workspace_size(0, 2048) == 0
    p = ops.plan_attend(4, 1, 2048, _props("no_merge"))
    assert p.n_split == 32 and not p.merge and p.workspace_bytes >= 4 * 32 * PER_PARTIAL
    f = ops.plan_forward(64, 32768, 2048, 1, 1, 0, 0, 1 << 40, _props("b200_like"))
    assert f.chunk == 64 and f.n_chunks == 1 and f.end >= 64 * 32768 * 4


def test_tight_workspace_falls_back_to_plans_without_partials(lib):
    # A workspace sized for 16 prefill queries (two layers) must still run 40:
    # chunks of 8 would need split partials that do not fit, so the layout
    # restricts the attention to plans without partials.
    for name in ("b200_like", "no_merge", "small_gpu"):
        props = _props(name)
        ws = ops.plan_forward(16, 3040, 2048, 8, 2, 1, 1, 1 << 60, props).end
        f = _check_forward_layout(lib, 40, 3040, 2048, 8, 2, 1, 1, ws, props)
        assert f is not None, name
        if not f.attend_partials:
            assert f.attend_bytes == 0
            for n in {f.chunk, f.last_chunk}:
                p = ops.plan_attend(n, 2, 2048, props, allow_partials=False)
                assert p.workspace_bytes == 0 and (p.n_split == 1 or p.merge)
