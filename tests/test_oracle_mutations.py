"""Plant plausible mistakes in a copy of the CPU oracle and check that the pins
in test_oracle_pins.py catch every one.  Runs on the CPU only: the mistakes
live in a throw-away module built from the oracle's source text."""

import importlib.util
import inspect
import os
import types

import pytest

import oracle.dsa_oracle as real
import tests.test_oracle_pins as pins

SRC = inspect.getsource(real)

MUTATIONS = {
    "indexer_drops_relu": ("np.maximum(dots, 0.0) @ wt[t]", "dots @ wt[t]"),
    "indexer_relu_after_weighting": ("np.maximum(dots, 0.0) @ wt[t]", "np.maximum(dots @ wt[t], 0.0)"),
    "indexer_ignores_weights": ("np.maximum(dots, 0.0) @ wt[t]", "np.maximum(dots, 0.0).sum(1)"),
    "indexer_excludes_own_position": (
        "        n = int(q_pos[t]) + 1\n        if n <= 0:\n            continue\n        base = int(seq_row_start[int(q_seq[t])])\n        k_rows",
        "        n = int(q_pos[t])\n        if n <= 0:\n            continue\n        base = int(seq_row_start[int(q_seq[t])])\n        k_rows"),
    "indexer_ignores_sequence_offset": (
        "        k_rows = _f64(keys[base:base + n])", "        k_rows = _f64(keys[0:n])"),
    "topk_ties_to_higher_position": ("np.lexsort((pos, -cand))", "np.lexsort((-pos, -cand))"),
    "topk_ascending_scores": ("np.lexsort((pos, -cand))", "np.lexsort((pos, cand))"),
    "topk_unsorted_output": ("chosen = np.sort(order[:keff])", "chosen = order[:keff]"),
    "topk_count_not_clamped": ("count[t] = keff", "count[t] = int(k)"),
    "attn_drops_multiplier": ("z = z * scale * mult[:, None]", "z = z * scale"),
    "attn_drops_scale": ("z = z * scale * mult[:, None]", "z = z * mult[:, None]"),
    "attn_drops_rotary_term": ("z = z + qp @ rows[:, d_c:d_c + qp.shape[1]].T", "z = z"),
    "attn_rotary_reads_latent": ("z = z + qp @ rows[:, d_c:d_c + qp.shape[1]].T",
                                 "z = z + qp @ rows[:, :qp.shape[1]].T"),
    "attn_lse_without_max": ("lse = zmax[:, 0] + np.log(", "lse = np.log("),
    "attn_values_shifted_window": ("return p @ rows[:, :d_c], lse", "return p @ rows[:, -d_c:], lse"),
    "e4m3_exponent_bias_8": ("np.exp2((e - 7).astype(np.float64))", "np.exp2((e - 8).astype(np.float64))"),
    "e4m3_no_subnormals": ("np.where(e == 0, (m / 8.0) * 2.0 ** -6,", "np.where(e == 0, 0.0 * m,"),
    "fp8_indexer_ignores_key_scale": (
        "k_rows = e4m3_decode(k8[base:base + n]) * _f64(k_scale[base:base + n])[:, None]",
        "k_rows = e4m3_decode(k8[base:base + n])"),
    "fp8_indexer_key_scale_of_wrong_row": (
        "k_rows = e4m3_decode(k8[base:base + n]) * _f64(k_scale[base:base + n])[:, None]",
        "k_rows = e4m3_decode(k8[base:base + n]) * _f64(k_scale[:n])[:, None]"),
    "merge_ties_to_higher_position": ("order = np.lexsort((ps, -sc))", "order = np.lexsort((-ps, -sc))"),
    "merge_keeps_empty_slots": ("    keep = ps >= 0\n", "    keep = ps >= -1\n"),
    "combine_plain_average": ('o = np.einsum("rh,rhd->hd", w, o_p) / np.where(tot > 0, tot, 1.0)[:, None]',
                              'o = o_p.mean(axis=0)'),
    "combine_lse_without_shift": ("lse = np.where(tot > 0, safe + np.log(", "lse = np.where(tot > 0, 0.0 + np.log("),
    "forward_ignores_k": ("idx, count = topk_select(scores, q_pos, k)",
                          "idx, count = topk_select(scores, q_pos, 2048)"),
    "forward_ld_one_short": ("ld = int(np.max(q_pos)) + 1", "ld = int(np.max(q_pos))"),
    "forward_selects_past_q_pos": ("idx, count = topk_select(scores, q_pos, k)",
                                   "idx, count = topk_select(scores, np.full(len(q_pos), ld - 1), k)"),
    "forward_every_layer_reads_first_cache": ('lay["cache"], lay["d_rope"], seq_row_start',
                                              'layers[0]["cache"], lay["d_rope"], seq_row_start'),
    "forward_drops_last_layer": ("    for lay in layers:\n", "    for lay in layers[:-1]:\n"),
    "fp8_latent_blocks_of_64": ("np.concatenate([np.arange(d_c) // LATENT_BLOCK,",
                                "np.concatenate([np.arange(d_c) // 64 % 4,"),
    "fp8_latent_rotary_takes_last_latent_scale": ("np.full(d_rope, d_c // LATENT_BLOCK, dtype=np.int64)",
                                                  "np.full(d_rope, d_c // LATENT_BLOCK - 1, dtype=np.int64)"),
    "fp8_latent_scales_ignored": ("    return values * scales[:, block_of_col]", "    return values"),
    "fp8_latent_scales_read_after_latent": ("r[:, n_codes:n_codes + 4 * n_blk]", "r[:, d_c:d_c + 4 * n_blk]"),
    "fp8_latent_reads_first_rows": ("rows = latent_fp8_decode(cache_np[base + sel], d_c, int(d_rope))",
                                    "rows = latent_fp8_decode(cache_np[sel], d_c, int(d_rope))"),
    "fp8_indexer_relu_after_weighting": ("out[t, :n] = np.maximum(k_rows @ q.T, 0.0) @ wt[t]",
                                         "out[t, :n] = np.maximum(k_rows @ q.T @ wt[t], 0.0)"),
}


def _mutant(name):
    old, new = MUTATIONS[name]
    assert SRC.count(old) >= 1, name
    mod = types.ModuleType("oracle_mutant_" + name)
    exec(compile(SRC.replace(old, new, 1), mod.__name__, "exec"), mod.__dict__)
    return mod


def _run_pins(mod, golden_dir, monkeypatch):
    for fn in ("index_scores", "topk_select", "sparse_mla", "dense_causal_mla", "explicit_mla",
               "forward", "e4m3_decode", "index_scores_fp8", "topk_merge", "lse_combine",
               "latent_fp8_decode", "sparse_mla_fp8"):
        monkeypatch.setattr(pins, fn, getattr(mod, fn))
    failures = 0
    for tname, test in inspect.getmembers(pins, inspect.isfunction):
        if not tname.startswith("test_"):
            continue
        params = inspect.signature(test).parameters
        variants = [{}]
        if "trial" in params:
            variants = [{"trial": i} for i in range(40)]
        if "d_r" in params:
            variants = [{"d_r": 64}, {"d_r": 0}]
        if "blk" in params:
            variants = [{"blk": b} for b in range(4)]
        for kw in variants:
            if "golden_dir" in params:
                kw = dict(kw, golden_dir=golden_dir)
            try:
                test(**kw)
            except Exception:
                failures += 1
    return failures


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, golden_dir, monkeypatch):
    assert _run_pins(_mutant(name), golden_dir, monkeypatch) > 0, name


def test_unmutated_oracle_passes_every_pin(golden_dir, monkeypatch):
    mod = types.ModuleType("oracle_copy")
    exec(compile(SRC, mod.__name__, "exec"), mod.__dict__)
    assert _run_pins(mod, golden_dir, monkeypatch) == 0
