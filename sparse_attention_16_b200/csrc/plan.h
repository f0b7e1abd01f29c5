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

// Splits each of `units` (layer, query) pairs so that units x n_split is about
// one wave of the GPU.  The splits merge on chip when all clusters of that size
// can be resident at once; a narrower split that still merges is preferred to
// the combine kernel as long as it keeps at least half the blocks.
inline SplitPlan attend_plan(const DevProps& d, int64_t units, int32_t k) {
  if (units < 1 || k < 1) return SplitPlan{1, kPlanTileRows, false};
  const int want = (int)std::max<int64_t>(1, d.sms / units);
  SplitPlan sp = split_rows(k, want);
  if (sp.n_split == 1) return sp;
  if (merge_fits(d, units, sp.n_split)) {
    sp.merge = true;
    return sp;
  }
  for (int n = std::min(want, kPlanMaxMerge); n >= 2; --n) {
    SplitPlan q = split_rows(k, n);
    if (2 * q.n_split < sp.n_split) break;
    if (merge_fits(d, units, q.n_split)) {
      q.merge = true;
      return q;
    }
  }
  return sp;
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

inline size_t attend_ws_bytes(const DevProps& d, int64_t units, int32_t k) {
  const SplitPlan sp = attend_plan(d, units, k);
  if (sp.n_split <= 1 || sp.merge) return 0;
  return partial_bytes(units, sp.n_split);
}

// Attention workspace for a chunk of n queries and n_layers layers, launched in
// groups of at most kPlanMaxLayers layers (the largest need over the groups).
inline size_t attend_ws_layers(const DevProps& d, int32_t n, int32_t n_layers, int32_t k) {
  if (n <= 0 || n_layers <= 0) return 0;
  const int g = std::min(n_layers, kPlanMaxLayers);
  size_t b = attend_ws_bytes(d, (int64_t)n * g, k);
  const int rem = n_layers % g;
  if (rem) b = std::max(b, attend_ws_bytes(d, (int64_t)n * rem, k));
  return b;
}

// Workspace layout of the fused call:
//   [idx chunk*k i32][count chunk i32][attention partials][scores chunk*ld f32]
// (idx / count only when the caller passes no idx_out / count_out).  The
// attention region holds the larger need of a full chunk and of the last one.
struct ForwardLayout {
  int32_t chunk = 0;             // queries per chunk (0: nothing fits)
  int32_t n_chunks = 0;
  int32_t last_chunk = 0;        // queries in the final chunk
  size_t idx_off = SIZE_MAX, cnt_off = SIZE_MAX;
  size_t att_off = 0, att_bytes = 0;
  size_t scores_off = 0, end = 0;
};

inline ForwardLayout forward_layout_for(const DevProps& d, int32_t T, int64_t ld, int32_t k, int32_t n_layers,
                                        bool own_idx, bool own_count, int32_t chunk) {
  ForwardLayout f;
  f.chunk = chunk;
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
  f.att_bytes = std::max(attend_ws_layers(d, chunk, n_layers, k), attend_ws_layers(d, f.last_chunk, n_layers, k));
  off += f.att_bytes;
  f.scores_off = off;
  off += plan_round_up((size_t)chunk * (size_t)ld * 4, 256);
  f.end = off;
  return f;
}

// The largest chunk (a multiple of q_group, or T itself) whose layout fits
// ws_bytes; then the chunks are evened out (same count, sizes as equal as the
// q_group rule allows).  chunk = 0 when even q_group queries do not fit.
inline ForwardLayout forward_layout(const DevProps& d, int32_t T, int64_t ld, int32_t k, int32_t q_group,
                                    int32_t n_layers, bool own_idx, bool own_count, size_t ws_bytes) {
  if (T <= 0) return ForwardLayout{};
  q_group = std::max(1, q_group);
  auto fits = [&](int32_t c) { return forward_layout_for(d, T, ld, k, n_layers, own_idx, own_count, c).end <= ws_bytes; };
  int32_t c = T;
  while (c > q_group && !fits(c)) {
    const int32_t half = (c / 2 + q_group - 1) / q_group * q_group;
    c = std::max(q_group, std::min(half, c - 1));
  }
  if (c > T) c = T;
  if (!fits(c)) {
    ForwardLayout none = forward_layout_for(d, T, ld, k, n_layers, own_idx, own_count, std::min(T, q_group));
    none.chunk = 0;
    return none;
  }
  const int32_t n_chunks = (T + c - 1) / c;
  int32_t even = (T + n_chunks - 1) / n_chunks;
  even = (even + q_group - 1) / q_group * q_group;
  if (even < c && fits(even) && (T + even - 1) / even == n_chunks) c = even;
  return forward_layout_for(d, T, ld, k, n_layers, own_idx, own_count, c);
}

}  // namespace dsa
