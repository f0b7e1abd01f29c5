"""Algorithmic bytes and flops of the hot path, and the model-level cost model.

Two layers of accounting live here:

* ``ModelSchedule`` restates, from the rules the Mistral Large 4 concept page
  (liminalml.com/concepts/mistral-large-4) gives in its bullet list and its
  "Cache" / "Sparse attention" / "When does sparse attention pay?" paragraphs,
  which of the 72 layers use rotary keys, which own a latent cache and which run
  their indexer.  From it follow the per-position cache size and the
  multiply-add counts the page prints (35,712 values per position, 74.9 GB at
  2^20 positions, 4.94e6 / 1.80e5 multiply-adds per attended / scored
  position, a crossover near 56K tokens, 3.5x / 19x / 26x savings, 39% of the
  indexer work removed by selection reuse).  tests/test_accounting.py checks
  these against the printed values (tests/golden/cost_model.json).

* ``decode_bytes`` / ``prefill_indexer_flops`` / ... give the compulsory HBM
  traffic and the flops of one call of each kernel, which bench.py divides by
  the measured kernel time to get the roofline fraction.

Nothing here touches a GPU.
"""

from __future__ import annotations

from dataclasses import dataclass

# Dimensions of one attention layer (concept page, "What to keep" / "Where to look";
# xfinit.ro blog "Mistral Large 4: Architecture, ...", section "Architecture").
N_HEADS = 64          # attention heads
D_LATENT = 512        # latent c_s
D_ROPE = 64           # rotary key kR_s (RoPE layers only)
N_IDX_HEADS = 32      # indexer heads
D_IDX = 128           # indexer head dim
TOPK = 2048           # positions kept per query
BF16 = 2
F32 = 4
I32 = 4


@dataclass(frozen=True)
class ModelSchedule:
    """Per-layer flags of the 72-layer decoder.

    rope[l]      layer l rotates its keys; every fourth layer (l = 3, 7, ...) is NoPE.
    kv_owner[l]  layer whose latent layer l reads: from layer 39 on, every fourth
                 layer (the NoPE ones) reads layer 35's latent.
    runs_idx[l]  layer l runs its own indexer; the others reuse the selection of
                 the most recent layer that ran one.  The first 17 layers run; then
                 13 groups of four follow the pattern reuse, reuse, run, run; the
                 last three layers are reuse, reuse, run.
    """

    n_layers: int = 72

    @property
    def rope(self):
        return [(l % 4) != 3 for l in range(self.n_layers)]

    @property
    def kv_owner(self):
        return [35 if (l >= 39 and l % 4 == 3) else l for l in range(self.n_layers)]

    @property
    def runs_idx(self):
        flags = [True] * 17
        for _ in range(13):
            flags += [False, False, True, True]
        flags += [False, False, True]
        assert len(flags) == self.n_layers
        return flags

    # ---- cache ----------------------------------------------------------------
    def row_values(self, layer: int) -> int:
        """Values cached per position by one layer: 512 + 64 on RoPE layers."""
        return D_LATENT + (D_ROPE if self.rope[layer] else 0)

    def cached_values_per_position(self) -> int:
        owner = self.kv_owner
        return sum(self.row_values(l) for l in range(self.n_layers) if owner[l] == l)

    def full_kv_values_per_position(self, d_head_k: int = 128, d_head_v: int = 128) -> int:
        return self.n_layers * N_HEADS * (d_head_k + d_head_v)

    def latent_cache_bytes(self, positions: int, bytes_per_value: int = BF16) -> int:
        return self.cached_values_per_position() * bytes_per_value * positions

    def index_key_bytes(self, positions: int, bytes_per_value: int = 1) -> int:
        """One 128-value key per position per indexer-running layer (FP8 = 1 B)."""
        return sum(self.runs_idx) * D_IDX * bytes_per_value * positions

    # ---- work -----------------------------------------------------------------
    def macs_per_attended_position(self) -> int:
        """64 heads x (512 score + 64 rotary score + 512 value) per layer."""
        return sum(N_HEADS * (D_LATENT + (D_ROPE if r else 0) + D_LATENT) for r in self.rope)

    def macs_per_scored_position(self) -> int:
        return sum(self.runs_idx) * N_IDX_HEADS * D_IDX

    def macs_per_token(self, context: int, sparse: bool = True) -> int:
        a = self.macs_per_attended_position()
        if not sparse:
            return a * context
        return a * min(context, TOPK) + self.macs_per_scored_position() * context

    def indexer_crossover(self) -> float:
        """Context length beyond which scoring costs more than attending."""
        return self.macs_per_attended_position() * TOPK / self.macs_per_scored_position()

    def dense_over_sparse(self, context: int) -> float:
        return self.macs_per_token(context, sparse=False) / self.macs_per_token(context)

    def indexer_share(self, context: int) -> float:
        s = self.macs_per_scored_position() * context
        return s / self.macs_per_token(context)

    def reuse_saving(self) -> float:
        r = self.runs_idx
        return (len(r) - sum(r)) / len(r)

    def prefill_scoring_macs(self, positions: int) -> float:
        return self.macs_per_scored_position() * positions * positions / 2


# ---- per-call algorithmic traffic (compulsory bytes, read once / written once) ----

def indexer_bytes(n_scored_total: int, n_queries: int, n_cols_written: int, fp8: bool = False) -> int:
    """Index keys read once, q and w per query, and the fp32 score row written.

    n_scored_total: key rows read (sum over queries of q_pos + 1 for decode).
    n_cols_written: score entries written (T x ld).
    fp8: E4M3 keys and queries (1 B per value) plus one fp32 scale per key row
         and per query head.
    """
    if fp8:
        q_w = n_queries * (N_IDX_HEADS * D_IDX * 1 + 2 * N_IDX_HEADS * F32)
        return n_scored_total * (D_IDX * 1 + F32) + q_w + n_cols_written * F32
    q_w = n_queries * (N_IDX_HEADS * D_IDX * BF16 + N_IDX_HEADS * F32)
    return n_scored_total * D_IDX * BF16 + q_w + n_cols_written * F32


def topk_bytes(n_candidates_total: int, n_queries: int, k: int = TOPK) -> int:
    """Scores read once, idx and count written."""
    return n_candidates_total * F32 + n_queries * (k * I32 + I32)


def attend_bytes(n_rows_total: int, n_queries: int, d_rope: int, with_lse: bool = True,
                 row_bytes: int | None = None) -> int:
    """Selected cache rows gathered once, query/multiplier read, output written.
    ``row_bytes``: bytes per cache row when it is not bf16 (FP8 latent rows)."""
    row = (D_LATENT + d_rope) * BF16 if row_bytes is None else row_bytes
    q = N_HEADS * (D_LATENT + d_rope) * BF16 + N_HEADS * F32
    out = N_HEADS * D_LATENT * BF16 + (N_HEADS * F32 if with_lse else 0)
    idx = TOPK * I32 + I32
    return n_rows_total * row + n_queries * (q + out + idx)


def attend_flops(n_rows_total: int, d_rope: int) -> int:
    """2 flops per multiply-add: 64 heads x (512 + d_rope) for the logits and 64 x 512 for o."""
    return 2 * n_rows_total * N_HEADS * (D_LATENT + d_rope + D_LATENT)


def indexer_flops(n_pairs: int) -> int:
    """2 x 32 heads x 128 dims per scored (query, position) pair."""
    return 2 * n_pairs * N_IDX_HEADS * D_IDX
