"""The cost model and byte accounting against the numbers the pages print."""

import json
import os

import pytest

from sparse_attention_16_b200 import accounting as acc


def _golden(golden_dir):
    with open(os.path.join(golden_dir, "cost_model.json")) as f:
        return {e["name"]: e for e in json.load(f)["entries"]}


def _computed():
    m = acc.ModelSchedule()
    owner = m.kv_owner
    reusing = [l for l in range(72) if owner[l] != l]
    return {
        "values_per_position_rope_layer": m.row_values(0),
        "cached_values_per_position": m.cached_values_per_position(),
        "reusing_layers_would_add": sum(m.row_values(l) for l in reusing),
        "full_kv_values_per_position": m.full_kv_values_per_position(),
        "full_kv_over_latent": m.full_kv_values_per_position() / m.cached_values_per_position(),
        "latent_cache_gb_at_2p20_bf16": m.latent_cache_bytes(1 << 20) / 1e9,
        "fp8_index_keys_gb_at_2p20": m.index_key_bytes(1 << 20) / 1e9,
        "macs_per_attended_position": m.macs_per_attended_position(),
        "macs_per_scored_position": m.macs_per_scored_position(),
        "indexer_crossover_tokens": m.indexer_crossover(),
        "dense_over_sparse_at_8k": m.dense_over_sparse(8 * 1024),
        "dense_over_sparse_at_128k": m.dense_over_sparse(128 * 1024),
        "dense_over_sparse_at_1m": m.dense_over_sparse(1 << 20),
        "indexer_extra_below_2k_percent": 100 * m.macs_per_scored_position() / m.macs_per_attended_position(),
        "reuse_removes_indexer_work_percent": 100 * m.reuse_saving(),
        "indexer_share_at_1m_percent": 100 * m.indexer_share(1 << 20),
        "prefill_scoring_macs_1m": m.prefill_scoring_macs(1 << 20),
        "layers_running_indexer": sum(m.runs_idx),
    }


def test_cost_model_reproduces_printed_numbers(golden_dir):
    g = _golden(golden_dir)
    c = _computed()
    assert set(g) == set(c)
    for name, e in g.items():
        assert abs(c[name] - e["value"]) <= e["tol"], (name, c[name], e["value"], e["cite"])


def test_schedule_structure():
    m = acc.ModelSchedule()
    rope = m.rope
    assert sum(rope) == 54 and rope.count(False) == 18          # 3:1 RoPE:NoPE
    owner = m.kv_owner
    assert all(not rope[l] for l in range(72) if owner[l] != l)  # sharers are NoPE
    assert not rope[35] and sum(1 for l in range(72) if owner[l] != l) == 9
    r = m.runs_idx
    assert sum(r) == 44 and r[:17] == [True] * 17 and r[-3:] == [False, False, True]


def test_row_sizes():
    assert acc.D_LATENT + acc.D_ROPE == 576
    m = acc.ModelSchedule()
    assert m.row_values(3) == 512 and m.row_values(4) == 576


def test_decode_bytes_of_the_batch64_config():
    # 64 sequences x 32,768 positions, one RoPE layer, top 2,048.
    T, L = 64, 32768
    idx_b = acc.indexer_bytes(T * L, T, 0)
    att_b = acc.attend_bytes(T * 2048, T, 64)
    assert idx_b == T * (L * 256 + 8192 + 128)
    per_q = (idx_b + att_b) / T
    assert per_q == pytest.approx(32768 * 256 + 8320 + 2359296 + 73728 + 256 + 65536 + 256 + 8196)
    assert (idx_b + att_b) / 1e6 == pytest.approx(698, abs=1)


def test_fp8_indexer_bytes_per_key_and_query():
    # E4M3 keys: 128 B of codes + a 4 B fp32 scale per scored key; per query 32 x 128 B of codes,
    # 32 fp32 scales and 32 fp32 weights; the score row as before.
    T, L = 64, 32768
    b = acc.indexer_bytes(T * L, T, T * L, fp8=True)
    assert b == T * L * (128 + 4) + T * (4096 + 128 + 128) + T * L * 4
    # about half of the bf16 stream for the same work
    assert b / acc.indexer_bytes(T * L, T, T * L) == pytest.approx(136 / 260, rel=1e-3)


def test_flop_counts():
    assert acc.attend_flops(1, 64) == 2 * 64 * 1088
    assert acc.attend_flops(1, 0) == 2 * 64 * 1024
    assert acc.indexer_flops(1) == 8192
