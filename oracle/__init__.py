"""CPU oracle for the DeepSeek-Sparse-Attention hot path (TEST INFRASTRUCTURE ONLY).

This package is a plain, slow, fp64 restatement of what the hot path computes:
the lightning indexer, the per-query top-k selection and absorbed MLA attention
over the selected rows, plus two independent cross-checks (dense causal MLA and
explicit per-head MLA).  It exists to prove the CUDA library right.

Only the test suite, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
reference arm of ``bench.py`` may import it.  The CUDA library under
``sparse_attention_16_b200`` never imports it, shares no code with it, and
fails loudly instead of falling back to it.

Parity status per function (what pins it, see tests/test_oracle_pins.py):
  index_scores      pinned: closed forms (one-hot head / unit query), the odd-part
                    identity relu(x) - relu(-x) = x, positive homogeneity,
                    hand-worked integer example, causal/sequence-offset checks.
  topk_select       pinned: brute force by repeated argmax on tiny inputs with
                    forced ties, order/padding invariants, closed forms for
                    monotone and all-equal rows.
  sparse_mla        pinned: equals dense_causal_mla when every candidate is
                    selected; equals explicit_mla (random W_UK / W_UV); single
                    row and zero-multiplier closed forms; permutation invariance.
  dense_causal_mla  pinned through the same equalities (independent code path).
  explicit_mla      pinned through the same equality (independent code path).
  forward           pinned: hand-worked two-layer example (RoPE + NoPE layer sharing one
                    selection, k = 1, 2 and more than the candidates); its selection equals a
                    brute-force top-k (repeated argmax) of each query's own scores over its
                    causal range; five planted mistakes (k ignored, ld one short, selection past
                    q_pos, every layer reading the first cache, last layer dropped) are caught.
  e4m3_decode       pinned: every one of the 256 codes against torch's float8_e4m3fn
                    conversion, and the format's landmark values (1, 448, 2^-6, 2^-9).
  topk_merge        pinned: the merge of per-shard top-k lists equals topk_select on the
                    whole row (tied and random rows, several shard counts).
  lse_combine       pinned: combining sparse_mla over disjoint parts of a selection equals
                    sparse_mla over the whole selection; empty parts contribute nothing.
  index_scores_fp8  pinned: hand-worked example with integer codes, positive
                    homogeneity in each key scale and in each query's scales, zero
                    scale gives zero scores, causal/offset checks.
  latent_fp8_decode pinned: hand-worked row (landmark codes, subnormal, per-block
                    scales, the rotary block's own scale, padding ignored).
  sparse_mla_fp8    pinned: with unit scales it is sparse_mla on the codes' values;
                    doubling one block's scale while halving that block of the query
                    doubles exactly that block of the output and leaves lse alone;
                    the rotary scale trades against q_pe; a zero rotary scale equals
                    a zero rotary query.
"""

from .dsa_oracle import (  # noqa: F401
    index_scores,
    e4m3_decode,
    index_scores_fp8,
    topk_select,
    topk_merge,
    lse_combine,
    sparse_mla,
    dense_causal_mla,
    explicit_mla,
    forward,
    latent_fp8_decode,
    sparse_mla_fp8,
)
