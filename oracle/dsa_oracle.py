"""Plain fp64 CPU oracle for the DSA indexer, top-k selection and absorbed sparse MLA.

TEST INFRASTRUCTURE ONLY: imported by tests/, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference arm of bench.py, never by the CUDA library.

Sources (the web pages about Mistral Large 4 this library follows):
  [CP]  "Mistral Large 4" concept page, liminalml.com/concepts/mistral-large-4:
        paragraphs "What to keep" (MLA latent + rotary key), "Where to look"
        (32-head indexer, best 2,048 positions, 64 attention heads), "Cache"
        (576 values per position per layer), "Sparse attention" (scores every
        earlier position, keeps the top 2,048, softmax over those alone;
        32 x 128 multiply-adds per scored position, 64 x (512 + 64 + 512) per
        attended one), "Query scaling" (per-head, position-dependent query
        multiplier).  The page's display equations were lost in extraction, so
        the formulas are the plain reading of that prose:
            I[t,s] = sum_j w[t,j] * max(0, q[t,j] . k[s])            (indexer)
            z[h,i] = (q_nope[t,h] . c_s + q_pe[t,h] . kR_s) * scale * m[t,h]
            p      = softmax over the selected s only;  o[t,h] = sum_i p_i c_s
  [TR]  "Mistral Large 4" reading of the technical report,
        avisoori1x.github.io/mistral_large_4, DSA paragraph: the indexer picks
        the top 2,048 keys per query, chosen per query.

Readings where the pages are silent:
  * the query's own position is a candidate: candidates are 0..q_pos[t];
  * ties go to the lower position; -0.0 equals +0.0; NaN scores rank as -inf;
  * the selection is returned sorted by ascending position, padded with -1;
  * the multiplier m[t,h] multiplies the whole logit, after ``scale``;
  * count = 0 gives o = 0 and lse = -inf.

Everything is computed in float64 from the exact values of the (bf16) inputs.
numpy's matmul and lexsort are the only library primitives used.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "index_scores",
    "topk_select",
    "sparse_mla",
    "dense_causal_mla",
    "explicit_mla",
    "forward",
    "latent_fp8_decode",
    "sparse_mla_fp8",
]


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def index_scores(q_idx, w, k_idx, seq_row_start, q_seq, q_pos, ld):
    """Lightning-indexer scores, [CP] "Where to look" and "Sparse attention".

    q_idx [T, H_I, d_I], w [T, H_I], k_idx [rows, d_I]; seq_row_start [B] is the
    first k_idx row of each sequence; query t belongs to sequence q_seq[t] and
    sits at position q_pos[t].  For every earlier position s (0 <= s <= q_pos[t])
        I[t, s] = sum_j w[t, j] * max(0, sum_d q_idx[t, j, d] * k[row(s), d])
    with row(s) = seq_row_start[q_seq[t]] + s.  Columns q_pos[t] < s < ld hold
    -inf.  Returns float64 [T, ld].
    """
    q = _f64(q_idx)
    wt = _f64(w)
    keys = np.asarray(k_idx)
    T = q.shape[0]
    out = np.full((T, int(ld)), -np.inf, dtype=np.float64)
    for t in range(T):
        n = int(q_pos[t]) + 1
        if n <= 0:
            continue
        base = int(seq_row_start[int(q_seq[t])])
        k_rows = _f64(keys[base:base + n])           # [n, d_I]
        dots = k_rows @ q[t].T                       # [n, H_I]: q_j . k_s
        out[t, :n] = np.maximum(dots, 0.0) @ wt[t]   # sum_j w_j ReLU(.)
    return out


def e4m3_decode(codes):
    """Value of FP8 E4M3 codes (the OCP 8-bit floating-point format, E4M3 variant),
    written out from the format's definition:
      bit 7 sign; bits 6..3 exponent e (bias 7); bits 2..0 mantissa m;
      e == 0: subnormal, value (m / 8) * 2^-6;  e > 0: (1 + m / 8) * 2^(e - 7);
      S.1111.111 is NaN; there are no infinities (largest finite: 448).
    Returns float64 of the same shape."""
    c = np.asarray(codes).astype(np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2((e - 7).astype(np.float64)))
    return np.where((c & 0x7F) == 0x7F, np.nan, sign * mag)


def index_scores_fp8(q8, q_scale, w, k8, k_scale, seq_row_start, q_seq, q_pos, ld):
    """Lightning-indexer scores on FP8 (E4M3) keys and queries with per-row scales.

    The concept page stores the indexer keys in FP8 in production ("1M-token
    serving scenario": 128 B per position per indexer layer) and does not give
    a scale convention.  The reading taken: key row s is
        k[s, :] = k_scale[s] * e4m3(k8[row(s), :])
    and query head j of query t is
        q[t, j, :] = q_scale[t, j] * e4m3(q8[t, j, :]),
    with positive fp32 scales; the scores are then the indexer's definition
        I[t, s] = sum_j w[t, j] * max(0, q[t, j, :] . k[s, :])
    on those values (columns q_pos[t] < s < ld hold -inf).  Returns float64 [T, ld].
    """
    wt = _f64(w)
    T = wt.shape[0]
    out = np.full((T, int(ld)), -np.inf, dtype=np.float64)
    for t in range(T):
        n = int(q_pos[t]) + 1
        if n <= 0:
            continue
        base = int(seq_row_start[int(q_seq[t])])
        q = e4m3_decode(q8[t]) * _f64(q_scale[t])[:, None]                              # [H_I, d_I]
        k_rows = e4m3_decode(k8[base:base + n]) * _f64(k_scale[base:base + n])[:, None]  # [n, d_I]
        out[t, :n] = np.maximum(k_rows @ q.T, 0.0) @ wt[t]
    return out


def topk_select(scores, q_pos, k):
    """Per-query top-k selection, [CP] "Sparse attention" and [TR] DSA paragraph.

    For query t the candidates are positions 0..q_pos[t].  They are ranked by
    score (descending) and then by position (ascending), so equal scores go to
    the lower position; -0.0 and +0.0 are equal; NaN ranks as -inf.  The best
    k_eff = min(k, q_pos[t] + 1) positions are kept and returned sorted by
    ascending position, padded with -1.  Returns (idx int32 [T, k],
    count int32 [T]).
    """
    s_all = np.asarray(scores)
    T = s_all.shape[0]
    idx = np.full((T, int(k)), -1, dtype=np.int32)
    count = np.zeros(T, dtype=np.int32)
    for t in range(T):
        n = int(q_pos[t]) + 1
        if n <= 0:
            continue
        cand = s_all[t, :n].astype(np.float64) + 0.0      # -0.0 + 0.0 == +0.0
        cand = np.where(np.isnan(cand), -np.inf, cand)
        pos = np.arange(n)
        order = np.lexsort((pos, -cand))                  # score desc, pos asc
        keff = min(int(k), n)
        chosen = np.sort(order[:keff])
        idx[t, :keff] = chosen
        count[t] = keff
    return idx, count


def topk_merge(cand_scores, cand_pos, k):
    """Global top-k of one query from the union of per-shard candidate lists.

    Context-parallel decode ([TR] serving section, Figure 16: each rank selects
    among its own positions, the candidates are exchanged, then merged):
    cand_scores [n] and cand_pos [n] hold every shard's candidates with their
    global positions (-1 marks an empty slot).  The rule is topk_select's:
    score descending, then position ascending; -0.0 == +0.0; NaN ranks as -inf.
    Returns the k_eff = min(k, valid candidates) best positions, ascending.
    """
    sc = np.asarray(cand_scores, dtype=np.float64) + 0.0
    ps = np.asarray(cand_pos, dtype=np.int64)
    keep = ps >= 0
    sc, ps = sc[keep], ps[keep]
    sc = np.where(np.isnan(sc), -np.inf, sc)
    order = np.lexsort((ps, -sc))
    return np.sort(ps[order[:min(int(k), ps.size)]])


def lse_combine(o_parts, lse_parts):
    """Attention over a selection split into disjoint parts, merged exactly.

    For one query, parts r = 0..R-1 each give o_r = sum_{i in r} exp(z_i - lse_r) c_i
    and lse_r = log sum_{i in r} exp(z_i) (-inf and o_r = 0 for an empty part).
    Over the whole selection, lse = log sum_r exp(lse_r) and
    o = sum_r exp(lse_r - lse) o_r: the context-parallel "output combine"
    ([TR] serving section, Figure 16).  o_parts [R, H, d], lse_parts [R, H].
    Returns (o [H, d], lse [H]); a head with every part empty gives 0 and -inf.
    """
    o_p = np.asarray(o_parts, dtype=np.float64)
    l_p = np.asarray(lse_parts, dtype=np.float64)
    top = np.max(l_p, axis=0)                                  # [H]
    safe = np.where(np.isneginf(top), 0.0, top)
    w = np.where(np.isneginf(l_p), 0.0, np.exp(l_p - safe))   # [R, H]
    tot = w.sum(axis=0)
    lse = np.where(tot > 0, safe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    o = np.einsum("rh,rhd->hd", w, o_p) / np.where(tot > 0, tot, 1.0)[:, None]
    return o, lse


def _attend_rows(qn, qp, mult, scale, rows, d_c):
    """Softmax attention of one query (all heads) over the given cache rows.

    qn [H, d_c], qp [H, d_r] or None, mult [H], rows [n, d_c + d_r] (float64).
    Returns (o [H, d_c], lse [H]).
    """
    H = qn.shape[0]
    if rows.shape[0] == 0:
        return np.zeros((H, d_c)), np.full(H, -np.inf)
    z = qn @ rows[:, :d_c].T                                  # q_nope . c_s
    if qp is not None and qp.shape[1] > 0:
        z = z + qp @ rows[:, d_c:d_c + qp.shape[1]].T         # + q_pe . kR_s
    z = z * scale * mult[:, None]                             # * scale * m[t,h]
    zmax = z.max(axis=1, keepdims=True)
    lse = zmax[:, 0] + np.log(np.exp(z - zmax).sum(axis=1))
    p = np.exp(z - lse[:, None])
    return p @ rows[:, :d_c], lse


def sparse_mla(q_nope, q_pe, qmul, scale, cache, d_rope, seq_row_start, q_seq,
               idx, count):
    """Absorbed MLA over the selected rows only, [CP] "What to keep",
    "Sparse attention" and "Query scaling".

    q_nope [T, H, d_c] (already absorbed through W_UK), q_pe [T, H, d_r] or
    None when d_rope == 0 (NoPE layer), qmul [T, H], cache [rows, >= d_c+d_r]
    holding [c_s | kR_s] per position.  For every head
        z_i = (q_nope . c_{s_i} + q_pe . kR_{s_i}) * scale * qmul[t, h]
        lse = log sum_i exp(z_i),  o = sum_i exp(z_i - lse) c_{s_i}
    over the first count[t] entries of idx[t] (entries equal to -1 are
    skipped).  Returns (o float64 [T, H, d_c], lse float64 [T, H]).
    """
    qn_all = _f64(q_nope)
    T, H, d_c = qn_all.shape
    qp_all = _f64(q_pe) if (q_pe is not None and d_rope > 0) else None
    mult_all = _f64(qmul)
    cache_np = np.asarray(cache)
    o = np.zeros((T, H, d_c))
    lse = np.full((T, H), -np.inf)
    for t in range(T):
        sel = np.asarray(idx[t, :int(count[t])], dtype=np.int64)
        sel = sel[sel >= 0]
        base = int(seq_row_start[int(q_seq[t])])
        rows = _f64(cache_np[base + sel, :d_c + int(d_rope)])
        o[t], lse[t] = _attend_rows(qn_all[t], None if qp_all is None else qp_all[t],
                                    mult_all[t], scale, rows, d_c)
    return o, lse


LATENT_BLOCK = 128   # latent values per FP8 scale (the report's blockwise scales)


def latent_fp8_decode(rows8, d_c, d_rope):
    """Values of latent-cache rows kept in FP8 (E4M3) with blockwise scales.

    The report's serving section keeps the KV cache in FP8 natively, and its
    training section runs FP8 with blockwise scales; neither gives a layout.
    The reading taken, for one position (one row of bytes):
      bytes [0, d_c + d_rope)                E4M3 codes of [c_s | kR_s]
      bytes [d_c + d_rope, + 4 * n_blocks)   fp32 scales (little-endian): one per
                                             128 latent values (d_c / 128 of them)
                                             and, when d_rope > 0, one more for kR_s
    so that column i < d_c is scale[i // 128] * e4m3(code[i]) and column d_c + j
    is scale[d_c // 128] * e4m3(code[d_c + j]).  Bytes after the scales are
    padding.  rows8: uint8 [n, >= d_c + d_rope + 4 * n_blocks].
    Returns float64 [n, d_c + d_rope].
    """
    r = np.asarray(rows8, dtype=np.uint8)
    n_codes = d_c + d_rope
    n_blk = d_c // LATENT_BLOCK + (1 if d_rope > 0 else 0)
    values = e4m3_decode(r[:, :n_codes])
    scales = np.ascontiguousarray(r[:, n_codes:n_codes + 4 * n_blk]).view("<f4").astype(np.float64)
    block_of_col = np.concatenate([np.arange(d_c) // LATENT_BLOCK,
                                   np.full(d_rope, d_c // LATENT_BLOCK, dtype=np.int64)])
    return values * scales[:, block_of_col]


def sparse_mla_fp8(q_nope, q_pe, qmul, scale, cache8, d_rope, seq_row_start, q_seq,
                   idx, count):
    """sparse_mla over a latent cache kept in FP8 (rows as latent_fp8_decode
    reads them; the report's serving section, native FP8 KV cache): the
    attention of the decoded values, everything else as sparse_mla.
    Returns (o float64 [T, H, d_c], lse float64 [T, H]).
    """
    qn_all = _f64(q_nope)
    T, H, d_c = qn_all.shape
    qp_all = _f64(q_pe) if (q_pe is not None and d_rope > 0) else None
    mult_all = _f64(qmul)
    cache_np = np.asarray(cache8, dtype=np.uint8)
    o = np.zeros((T, H, d_c))
    lse = np.full((T, H), -np.inf)
    for t in range(T):
        sel = np.asarray(idx[t, :int(count[t])], dtype=np.int64)
        sel = sel[sel >= 0]
        base = int(seq_row_start[int(q_seq[t])])
        rows = latent_fp8_decode(cache_np[base + sel], d_c, int(d_rope))
        o[t], lse[t] = _attend_rows(qn_all[t], None if qp_all is None else qp_all[t],
                                    mult_all[t], scale, rows, d_c)
    return o, lse


def dense_causal_mla(q_nope, q_pe, qmul, scale, cache, d_rope, seq_row_start,
                     q_seq, q_pos):
    """Dense causal absorbed MLA over every position 0..q_pos[t].

    Independent of the selection path: it never looks at an index list.  With
    k >= q_pos + 1 the sparse layer must equal it (the sparse attention of [CP]
    "Sparse attention" only drops positions).
    """
    qn_all = _f64(q_nope)
    T, H, d_c = qn_all.shape
    cache_np = np.asarray(cache)
    o = np.zeros((T, H, d_c))
    lse = np.full((T, H), -np.inf)
    for t in range(T):
        base = int(seq_row_start[int(q_seq[t])])
        n = int(q_pos[t]) + 1
        z = np.zeros((H, n))
        c = _f64(cache_np[base:base + n, :d_c])
        for h in range(H):                       # head by head, no shared helper
            zh = c @ qn_all[t, h]
            if q_pe is not None and d_rope > 0:
                kr = _f64(cache_np[base:base + n, d_c:d_c + d_rope])
                zh = zh + kr @ _f64(q_pe)[t, h]
            z[h] = zh * scale * float(qmul[t, h])
        mx = z.max(axis=1)
        e = np.exp(z - mx[:, None])
        den = e.sum(axis=1)
        lse[t] = mx + np.log(den)
        o[t] = (e / den[:, None]) @ c
    return o, lse


def explicit_mla(q_head, q_pe, W_UK, W_UV, qmul, scale, cache, d_rope,
                 seq_row_start, q_seq, idx, count):
    """Explicit (non-absorbed) MLA with per-head keys and values rebuilt from the
    latent, [CP] "What to keep": each head rebuilds its own keys and values from
    the 512-value latent through a learned up-projection.

    q_head [T, H, d_h] is the per-head no-rope query, W_UK / W_UV [H, d_h, d_c].
    Per head: key_s = [W_UK_h c_s ; kR_s], value_s = W_UV_h c_s, logit
    (q_head . W_UK_h c_s + q_pe . kR_s) * scale * m.  Returns the per-head
    output [T, H, d_h] (float64).  The absorbed form must satisfy
    out_h = W_UV_h @ o_abs_h with q_nope_h = W_UK_h^T q_head_h.
    """
    qh = _f64(q_head)
    T, H, d_h = qh.shape
    wk = _f64(W_UK)
    wv = _f64(W_UV)
    cache_np = np.asarray(cache)
    d_c = wk.shape[2]
    out = np.zeros((T, H, d_h))
    for t in range(T):
        sel = np.asarray(idx[t, :int(count[t])], dtype=np.int64)
        sel = sel[sel >= 0]
        base = int(seq_row_start[int(q_seq[t])])
        c = _f64(cache_np[base + sel, :d_c])                     # [n, d_c]
        for h in range(H):
            keys = c @ wk[h].T                                   # [n, d_h]
            vals = c @ wv[h].T                                   # [n, d_h]
            z = keys @ qh[t, h]
            if q_pe is not None and d_rope > 0:
                kr = _f64(cache_np[base + sel, d_c:d_c + d_rope])
                z = z + kr @ _f64(q_pe)[t, h]
            z = z * scale * float(qmul[t, h])
            z = z - z.max()
            p = np.exp(z)
            p = p / p.sum()
            out[t, h] = p @ vals
    return out


def forward(q_idx, w, k_idx, seq_row_start, q_seq, q_pos, layers, scale,
            k=2048, ld=None):
    """One selection feeding several layers, [CP] bullet "28 layers reuse the
    selection made by the most recent layer that ran its indexer".

    ``layers`` is a list of dicts with keys q_nope, q_pe (or None), qmul, cache,
    d_rope.  Returns (idx, count, [(o, lse) per layer]).
    """
    if ld is None:
        ld = int(np.max(q_pos)) + 1
    scores = index_scores(q_idx, w, k_idx, seq_row_start, q_seq, q_pos, ld)
    idx, count = topk_select(scores, q_pos, k)
    outs = []
    for lay in layers:
        outs.append(sparse_mla(lay["q_nope"], lay.get("q_pe"), lay["qmul"], scale,
                               lay["cache"], lay["d_rope"], seq_row_start, q_seq,
                               idx, count))
    return idx, count, outs
