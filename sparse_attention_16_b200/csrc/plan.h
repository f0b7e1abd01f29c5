// plan.h - launch planning on the host: how the attention splits each
// (layer, query) across thread blocks, and how the fused call cuts its queries
// into chunks that fit the caller's workspace.  Pure functions of the problem
// size and of a few device properties (no CUDA calls), so the same code plans
// the launches and answers the planning queries of the C ABI, also on a
// machine without a GPU.
#pragma once

#include <algorithm>
#include <cstddef>
#include <cstdint>

namespace dsa {

constexpr int kPlanHeads = 64;
constexpr int kPlanLatent = 512;
constexpr int kPlanTileRows = 64;     // rows per attention tile
constexpr int kPlanMaxSplits = 32;    // blocks per (layer, query)
constexpr int kPlanMaxMerge = 8;      // largest cluster that merges on chip
constexpr int kPlanMaxLayers = 8;     // layers per attention launch
constexpr int kPlanTopkCap = 10240;   // top-k candidates per query (histogram path)
constexpr int kPlanTopkBins = 2048;   // bins of the indexer's score histogram
constexpr int kPlanTopkRowCap = 40960;   // rows up to this long are selected from shared memory (no workspace)

inline size_t plan_round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// What the planner needs to know about the device.
struct DevProps {
  int sms = 148;                 // streaming multiprocessors
  int max_clusters[9] = {};      // [c]: clusters of c attention blocks resident at once (c = 2..8)
};

struct SplitPlan {
  int n_split = 1;               // blocks per (layer, query)
  int rows_per_split = 0;        // selected rows per block, multiple of 64
  bool merge = false;            // the n_split blocks form a cluster and merge in distributed shared memory
};

// Even split of k selected rows over (about) `want` blocks, in whole tiles.
inline SplitPlan split_rows(int32_t k, int want) {
  const int max_tiles = (int)((k + kPlanTileRows - 1) / kPlanTileRows);
  want = std::max(1, std::min(want, std::min(max_tiles, kPlanMaxSplits)));
  const int tiles_per = (max_tiles + want - 1) / want;
  SplitPlan sp;
  sp.rows_per_split = tiles_per * kPlanTileRows;
  sp.n_split = (int)((k + sp.rows_per_split - 1) / sp.rows_per_split);
  return sp;
}

inline bool merge_fits(const DevProps& d, int64_t units, int n_split) {
  return n_split >= 2 && n_split <= kPlanMaxMerge && units <= d.max_clusters[n_split];
}

// Estimated time (microseconds) of a split plan: one block per SM, so the
// blocks run in waves; each block pays a fixed start (query gather, first-tile
// latency) plus its tiles; splits then merge on chip (cluster) or through the
// combine kernel (an extra launch and the partials' round trip through L2).
// The constants are per-tile and per-launch times measured on B200 at 64 heads
// (the combine path: ~5 us to write the fp32 partials, ~5-7 us for the combine
// kernel; the on-chip merge: a few us).
constexpr double kCostStartUs = 3.0;
constexpr double kCostTileUs = 2.3;
constexpr double kCostMergeUs = 10.0;
constexpr double kCostCombineUs = 10.0;

inline double plan_cost(const DevProps& d, int64_t units, int32_t k, const SplitPlan& sp) {
  const int max_tiles = (int)((k + kPlanTileRows - 1) / kPlanTileRows);
  const int tiles_per = std::min(max_tiles, sp.rows_per_split / kPlanTileRows);
  const int64_t blocks = units * sp.n_split;
  const int64_t waves = (blocks + d.sms - 1) / d.sms;
  double t = (double)waves * (kCostStartUs + tiles_per * kCostTileUs);
  if (sp.n_split > 1) t += sp.merge ? kCostMergeUs : kCostCombineUs;
  return t;
}

// Splits each of `units` (layer, query) pairs across blocks: the plan of least
// estimated time among every split width (whole tiles per block), where widths
// of 2-8 merge on chip when all clusters of that width can be resident at once
// and otherwise go through the combine kernel.  With allow_partials = false only
// plans that need no workspace qualify (one block, or an on-chip merge).
inline SplitPlan attend_plan(const DevProps& d, int64_t units, int32_t k, bool allow_partials = true) {
  if (units < 1 || k < 1) return SplitPlan{1, kPlanTileRows, false};
  SplitPlan best = split_rows(k, 1);
  double best_t = plan_cost(d, units, k, best);
  for (int n = 2; n <= kPlanMaxSplits; ++n) {
    SplitPlan sp = split_rows(k, n);
    if (sp.n_split == 1) continue;
    sp.merge = merge_fits(d, units, sp.n_split);
    if (!sp.merge && !allow_partials) continue;
    const double t = plan_cost(d, units, k, sp);
    if (t < best_t - 1e-9) {
      best = sp;
      best_t = t;
    }
  }
  return best;
}

// Workspace bytes for the split partials of a plan: per (pair, split) 64 x 512
// fp32 numerators, then 64 x 4 fp32 statistics.
inline size_t partial_bytes(int64_t units, int n_split) {
  const size_t n = (size_t)units * (size_t)n_split;
  return plan_round_up(n * kPlanHeads * kPlanLatent * 4, 256) + plan_round_up(n * kPlanHeads * 4 * 4, 256);
}
inline size_t partial_stats_offset(int64_t units, int n_split) {
  return plan_round_up((size_t)units * (size_t)n_split * kPlanHeads * kPlanLatent * 4, 256);
}

inline size_t attend_ws_bytes(const DevProps& d, int64_t units, int32_t k, bool allow_partials = true) {
  const SplitPlan sp = attend_plan(d, units, k, allow_partials);
  if (sp.n_split <= 1 || sp.merge) return 0;
  return partial_bytes(units, sp.n_split);
}

// Attention workspace for a chunk of n queries and n_layers layers, launched in
// groups of at most kPlanMaxLayers layers (the largest need over the groups).
inline size_t attend_ws_layers(const DevProps& d, int32_t n, int32_t n_layers, int32_t k,
                               bool allow_partials = true) {
  if (n <= 0 || n_layers <= 0 || !allow_partials) return 0;
  const int g = std::min(n_layers, kPlanMaxLayers);
  size_t b = attend_ws_bytes(d, (int64_t)n * g, k);
  const int rem = n_layers % g;
  if (rem) b = std::max(b, attend_ws_bytes(d, (int64_t)n * rem, k));
  return b;
}

// Top-k from the indexer's histogram: each query is spread over S slices,
// enough to fill the GPU but no slice shorter than ~8K candidates.
inline int topk_slices(int sms, int32_t T, int64_t ld) {
  const int64_t by_sms = std::max<int64_t>(1, sms / std::max<int32_t>(1, T));
  const int64_t by_len = std::max<int64_t>(1, (ld + 8191) / 8192);
  return (int)std::min<int64_t>(64, std::min(by_sms, by_len));
}
// Workspace of that path: per (query, slice) kPlanTopkCap keys and positions,
// then the slices' counts, then per query the k-th bin as the filter read it.
// Rows of at most kPlanTopkRowCap scores are selected by one CTA per query from
// shared memory and need none.
inline size_t topk_hist_ws_bytes(int sms, int32_t T, int64_t ld) {
  if (ld <= kPlanTopkRowCap) return 0;
  const size_t ts = (size_t)T * topk_slices(sms, T, ld);
  return 2 * plan_round_up(ts * kPlanTopkCap * 4, 256) + plan_round_up(ts * 4, 256) +
         plan_round_up((size_t)T * 16, 256);
}
inline size_t hist_bytes(int32_t T) { return plan_round_up((size_t)T * kPlanTopkBins * 4, 256); }

// Workspace layout of the fused call:
//   [idx chunk*k i32][count chunk i32][attention partials][hist chunk*2048 u32]
//   [top-k lists][scores chunk*ld f32]
// (idx / count only when the caller passes no idx_out / count_out; the score
// histogram and the top-k lists only for decode groups, q_group = 1).  The
// attention region holds the larger need of a full chunk and of the last one;
// it is empty when the layout restricts the attention to plans without
// partials (a tight workspace).
struct ForwardLayout {
  int32_t chunk = 0;             // queries per chunk (0: nothing fits)
  int32_t n_chunks = 0;
  int32_t last_chunk = 0;        // queries in the final chunk
  bool partials = true;          // the attention may use plans that write partials
  size_t idx_off = SIZE_MAX, cnt_off = SIZE_MAX;
  size_t att_off = 0, att_bytes = 0;
  size_t hist_off = SIZE_MAX, topk_off = SIZE_MAX, topk_bytes = 0;
  size_t scores_off = 0, end = 0;
};

inline ForwardLayout forward_layout_for(const DevProps& d, int32_t T, int64_t ld, int32_t k, int32_t n_layers,
                                        bool own_idx, bool own_count, int32_t chunk, bool partials = true,
                                        bool use_hist = false) {
  ForwardLayout f;
  f.chunk = chunk;
  f.partials = partials;
  f.n_chunks = (T + chunk - 1) / chunk;
  f.last_chunk = T - (f.n_chunks - 1) * chunk;
  size_t off = 0;
  if (own_idx) {
    f.idx_off = off;
    off += plan_round_up((size_t)chunk * k * 4, 256);
  }
  if (own_count) {
    f.cnt_off = off;
    off += plan_round_up((size_t)chunk * 4, 256);
  }
  f.att_off = off;
  f.att_bytes = std::max(attend_ws_layers(d, chunk, n_layers, k, partials),
                         attend_ws_layers(d, f.last_chunk, n_layers, k, partials));
  off += f.att_bytes;
  if (use_hist) {
    f.hist_off = off;
    off += hist_bytes(chunk);
    f.topk_off = off;
    f.topk_bytes = topk_hist_ws_bytes(d.sms, chunk, ld);
    off += f.topk_bytes;
  }
  f.scores_off = off;
  off += plan_round_up((size_t)chunk * (size_t)ld * 4, 256);
  f.end = off;
  return f;
}

// Chunks of (nearly) equal size: for n = 1, 2, 3, ... chunks, the chunk size is
// ceil(T / n) rounded up to a multiple of q_group (T itself when n = 1); the
// first n whose layout fits ws_bytes wins.  Equal chunks keep the last chunk
// from being a small remainder that the attention would split wide (and need
// more partials than the full chunks).  If no chunking fits with the fastest
// attention plans, the search is repeated with plans that need no partials.
// chunk = 0 when nothing fits.
inline ForwardLayout forward_layout(const DevProps& d, int32_t T, int64_t ld, int32_t k, int32_t q_group,
                                    int32_t n_layers, bool own_idx, bool own_count, size_t ws_bytes) {
  if (T <= 0) return ForwardLayout{};
  q_group = std::max(1, q_group);
  const int32_t max_chunks = (T + q_group - 1) / q_group;
  for (int pass = 0; pass < 2; ++pass) {
    const bool partials = pass == 0;
    int32_t prev = -1;
    for (int32_t n = 1; n <= max_chunks; ++n) {
      int32_t c = (T + n - 1) / n;
      if (n > 1) c = (c + q_group - 1) / q_group * q_group;
      c = std::min(c, T);
      if (c == prev) continue;
      prev = c;
      const ForwardLayout f = forward_layout_for(d, T, ld, k, n_layers, own_idx, own_count, c, partials, q_group == 1);
      if (f.end <= ws_bytes) return f;
    }
  }
  ForwardLayout none = forward_layout_for(d, T, ld, k, n_layers, own_idx, own_count, std::min(T, q_group), false,
                                          q_group == 1);
  none.chunk = 0;
  return none;
}

}  // namespace dsa
