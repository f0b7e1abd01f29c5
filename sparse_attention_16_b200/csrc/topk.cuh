// topk.cuh - per-query top-k over fp32 scores (radix select, exact tie rule).
//
// Selection rule (concept page "Sparse attention": keep the best 2,048 earlier
// positions per query; readings: ties go to the lower position, -0 == +0, NaN
// ranks as -inf): candidates of query t are columns 0..q_pos[t].
//
// Scores are mapped to order-preserving 32-bit keys.  Three histogram passes
// (11 + 11 + 10 bits) find the k-th largest key tau and how many keys equal to
// tau must be taken (need_eq).  A final ordered pass writes the positions of
// keys > tau and of the first need_eq keys == tau, in ascending position order
// (output slot of a kept element = #(> tau before it) + min(#(== tau before it),
// need_eq)), so the result is unique and deterministic.
//
// Three ways to run it:
//  * topk_kernel<CL>: one query per cluster of CL CTAs (CL in {1, 2, 4, 8, 16});
//    each CTA owns a contiguous slice of the candidates and stages its keys in
//    shared memory (whole keys up to 32K per CTA, their top 16 bits up to 64K,
//    where candidates re-read their full key).  The first histogram is summed
//    over the cluster through distributed shared memory; the keys in bins at
//    or above the k-th one are filtered into candidate lists and gathered in
//    rank 0, which finishes alone (or, if they overflow, the cluster runs the
//    passes over its whole slices).
//  * With the first histogram already made by the indexer (its epilogue counts
//    every score it writes), the first pass is free: topk_filter_kernel spreads
//    each query over S slices on every SM, each finding the k-th bin b1 from the
//    histogram and keeping its keys in bins >= b1 (ordered, warp-private lists)
//    in a workspace; topk_select_kernel (one CTA per query) gathers them and
//    runs the last two passes and the ordered output.  If the candidates would
//    exceed kTopkCandCap (a bin full of near-equal scores) or do not add up to
//    the histogram's count, that CTA runs the single-CTA algorithm on the row.
//  * With the histogram and rows of at most kTopkRowCap scores:
//    topk_row_kernel, one CTA per query with the whole row in shared memory
//    (position bitmaps instead of ordered lists; see there).
#pragma once

#include <cooperative_groups.h>

#include "ptx.cuh"

namespace dsa {

namespace cg = cooperative_groups;

constexpr int kTopkThreads = 1024;
constexpr int kTopkBins = 2048;                 // passes 1 and 2 (11 bits); pass 3 uses 1024
constexpr int kTopkStashCap = 32768;            // keys staged in shared memory per CTA
constexpr int kTopkCandCap = 10240;             // (key, position) candidates per CTA
constexpr int kTopkSmemBytes = 2 * kTopkBins * 4 + 1024 + kTopkStashCap * 4 + kTopkCandCap * 8;

struct TopkParams {
  const float* scores;   // [T, ld]
  const int32_t* q_pos;  // [T]
  int32_t* idx;          // [T, k]
  int32_t* count;        // [T]
  int64_t ld;
  int32_t T;
  int32_t k;
};


// Exclusive scan of one uint32 per thread over the whole 1024-thread block.
// `tmp` needs 33 words of shared memory; returns the block total in *total.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* tmp, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = tmp[lane];
    uint32_t s = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    tmp[lane] = s - w;          // exclusive prefix of warp totals
    if (lane == 31) tmp[32] = s;
  }
  __syncthreads();
  const uint32_t r = tmp[warp] + x - v;
  *total = tmp[32];
  __syncthreads();
  return r;
}

// Finds bin b (scanning from the top) with above(b) < need <= above(b) + h[b],
// where above(b) counts elements in bins above b.  Writes (b, above(b)) to res.
// Thread i sums positions [i PER, (i + 1) PER) of the top-down order; a warp
// scan gives the counts above each lane inside its warp, and every warp scans
// the 32 warp totals itself (two barriers in all).
template <int NB>
__device__ __forceinline__ void find_threshold_bin(const uint32_t* h, uint32_t need, uint32_t* tmp,
                                                   uint32_t* res) {
  static_assert(kTopkThreads == 32 * 32, "one warp total per lane of a warp");
  constexpr int PER = NB / kTopkThreads;  // 2 or 1 bins per thread, descending
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t c[PER];
  uint32_t mine = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    c[i] = h[NB - 1 - (threadIdx.x * PER + i)];
    mine += c[i];
  }
  uint32_t x = mine;   // inclusive prefix inside the warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  const uint32_t wt = tmp[lane];
  uint32_t ws = wt;   // inclusive prefix of the warp totals
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, ws, o);
    if (lane >= o) ws += y;
  }
  uint32_t above = __shfl_sync(0xffffffffu, ws - wt, warp) + x - mine;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int b = NB - 1 - (threadIdx.x * PER + i);
    if (above < need && need <= above + c[i]) {
      res[0] = (uint32_t)b;
      res[1] = above;
    }
    above += c[i];
  }
  __syncthreads();
}

template <int CL>
__device__ __forceinline__ void cluster_barrier() {
  if constexpr (CL > 1) {
    cg::this_cluster().sync();
  } else {
    __syncthreads();
  }
}

// Sums the NB-bin histograms of all CTAs in the cluster into `tot` of every
// CTA.  CTA r reduces bins [r NB/CL, (r+1) NB/CL) over all ranks into rank 0's
// `tot`; then every CTA copies rank 0's `tot`.  Each CTA thus reads 2 NB words
// through distributed shared memory instead of CL x NB.
template <int CL, int NB>
__device__ __forceinline__ void cluster_sum_hist(uint32_t* hist, uint32_t* tot) {
  if constexpr (CL > 1) {
    cg::cluster_group cl = cg::this_cluster();
    const int rank = (int)cl.block_rank();
    cluster_barrier<CL>();                 // every histogram is complete
    uint32_t* tot0 = cl.map_shared_rank(tot, 0);
    constexpr int SL = NB / CL;
    for (int b = rank * SL + threadIdx.x; b < (rank + 1) * SL; b += kTopkThreads) {
      uint32_t s = 0;
#pragma unroll
      for (int r = 0; r < CL; ++r) s += cl.map_shared_rank(hist, r)[b];
      tot0[b] = s;
    }
    cluster_barrier<CL>();                 // rank 0 holds the sums; peers' hists no longer read
    if (rank != 0)
      for (int b = threadIdx.x; b < NB; b += kTopkThreads) tot[b] = tot0[b];
    __syncthreads();
  } else {
    __syncthreads();
    for (int b = threadIdx.x; b < NB; b += kTopkThreads) tot[b] = hist[b];
    __syncthreads();
  }
}

// The selection of query t by the CTA of cluster rank `rank` (all CL CTAs of a
// cluster call it for the same t).
template <int CL>
__device__ __forceinline__ void topk_query(const TopkParams& p, int t, int rank) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem_raw);
  uint32_t* tot = hist + kTopkBins;
  uint32_t* tmp = tot + kTopkBins;           // 33 words of scan scratch
  uint32_t* res = tmp + 40;                  // threshold results
  uint32_t* cnt = res + 8;                   // this CTA's (#gt, #eq), read by peers
  uint32_t* stash = reinterpret_cast<uint32_t*>(smem_raw + 2 * kTopkBins * 4 + 1024);

  int qp = p.q_pos[t];
  if (qp >= p.ld) {
    if (threadIdx.x == 0 && rank == 0) raise_error(kErrBadSeq);
    qp = (int)p.ld - 1;
  }
  const int64_t n = (qp < 0) ? 0 : (int64_t)qp + 1;
  int32_t* out = p.idx + (int64_t)t * p.k;

  if (n <= p.k) {  // every candidate is kept
    for (int64_t i = (int64_t)rank * kTopkThreads + threadIdx.x; i < p.k; i += (int64_t)CL * kTopkThreads)
      out[i] = (i < n) ? (int32_t)i : -1;
    if (rank == 0 && threadIdx.x == 0) p.count[t] = (int32_t)n;
    return;
  }

  const float* row = p.scores + (int64_t)t * p.ld;
  const int64_t lo = ((int64_t)rank * n / CL) & ~int64_t(3);
  const int64_t hi = (rank == CL - 1) ? n : (((int64_t)(rank + 1) * n / CL) & ~int64_t(3));
  const int64_t len = hi - lo;
  const bool staged = len <= kTopkStashCap;                          // 32-bit keys
  const bool staged16 = !staged && len <= 2 * kTopkStashCap;       // top 16 bits of each key
  uint16_t* stash16 = reinterpret_cast<uint16_t*>(stash);

  // ---- pass 1: histogram of the top 11 bits (loads batched 4 x float4 per thread)
  for (int b = threadIdx.x; b < kTopkBins; b += kTopkThreads) hist[b] = 0;
  __syncthreads();
  const int64_t n4 = len >> 2;
  const float4* row4 = reinterpret_cast<const float4*>(row + lo);
  for (int64_t i0 = 0; i0 < n4; i0 += 4 * kTopkThreads) {
    float4 f[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t i = i0 + u * kTopkThreads + threadIdx.x;
      f[u] = (i < n4) ? row4[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t i = i0 + u * kTopkThreads + threadIdx.x;
      if (i < n4) {
        const uint32_t k0 = score_key(f[u].x), k1 = score_key(f[u].y), k2 = score_key(f[u].z),
                       k3 = score_key(f[u].w);
        atomicAdd(&hist[k0 >> 21], 1u);
        atomicAdd(&hist[k1 >> 21], 1u);
        atomicAdd(&hist[k2 >> 21], 1u);
        atomicAdd(&hist[k3 >> 21], 1u);
        if (staged) reinterpret_cast<uint4*>(stash)[i] = make_uint4(k0, k1, k2, k3);
        else if (staged16) reinterpret_cast<uint2*>(stash16)[i] = make_uint2((k0 >> 16) | (k1 & 0xFFFF0000u),
                                                                             (k2 >> 16) | (k3 & 0xFFFF0000u));
      }
    }
  }
  for (int64_t i = (n4 << 2) + threadIdx.x; i < len; i += kTopkThreads) {
    const uint32_t kk = score_key(row[lo + i]);
    atomicAdd(&hist[kk >> 21], 1u);
    if (staged) stash[i] = kk;
    else if (staged16) stash16[i] = (uint16_t)(kk >> 16);
  }
  __syncthreads();
  cluster_sum_hist<CL, kTopkBins>(hist, tot);
  find_threshold_bin<kTopkBins>(tot, (uint32_t)p.k, tmp, res);
  const uint32_t b1 = res[0];
  uint32_t above = res[1];
  uint32_t need = (uint32_t)p.k - above;

  // ---- filter: keys in bins >= b1 (all of the selection) with their positions.
  // Warp w owns a contiguous segment of this CTA's slice; pass (a) counts its
  // candidates, pass (b) writes them in position order (ballot compaction).
  uint32_t* cand_key = stash + kTopkStashCap;
  int32_t* cand_pos = reinterpret_cast<int32_t*>(cand_key + kTopkCandCap);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kWarps = kTopkThreads / 32;
  const int64_t seg = ((len + kWarps - 1) / kWarps + 127) & ~int64_t(127);
  const int64_t s_lo = (warp * seg < len) ? warp * seg : len;
  const int64_t s_hi = (s_lo + seg < len) ? s_lo + seg : len;
  auto key_at = [&](int64_t i) -> uint32_t { return staged ? stash[i] : score_key(row[lo + i]); };
  // Four consecutive keys per lane per step: one 16-byte load from the stash
  // (conflict-free) or from the scores, scalar loads only in a segment's tail.
  // With the 16-bit stash the loaded keys hold only their top 16 bits (the
  // filter tests bits 31..21); full keys come from the scores when written.
  auto load4 = [&](int64_t e0, uint32_t (&kk)[4]) {
    if (e0 + 3 < s_hi) {
      if (staged) {
        const uint4 v = reinterpret_cast<const uint4*>(stash)[e0 >> 2];
        kk[0] = v.x; kk[1] = v.y; kk[2] = v.z; kk[3] = v.w;
      } else if (staged16) {
        const uint2 v = reinterpret_cast<const uint2*>(stash16)[e0 >> 2];
        kk[0] = v.x << 16; kk[1] = v.x & 0xFFFF0000u; kk[2] = v.y << 16; kk[3] = v.y & 0xFFFF0000u;
      } else {
        const float4 f = *reinterpret_cast<const float4*>(row + lo + e0);
        kk[0] = score_key(f.x); kk[1] = score_key(f.y); kk[2] = score_key(f.z); kk[3] = score_key(f.w);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) kk[e] = (e0 + e < s_hi) ? key_at(e0 + e) : 0u;
    }
  };
  // (a) count
  uint32_t wcount = 0;
  for (int64_t i0 = s_lo; i0 < s_hi; i0 += 128) {
    const int64_t e0 = i0 + 4 * lane;
    uint32_t kk[4];
    load4(e0, kk);
#pragma unroll
    for (int e = 0; e < 4; ++e) wcount += (e0 + e < s_hi) && ((kk[e] >> 21) >= b1);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wcount += __shfl_xor_sync(0xffffffffu, wcount, o);
  if (lane == 0) tmp[warp] = wcount;
  __syncthreads();
  if (warp == 0) {
    const uint32_t w = tmp[lane];
    uint32_t x = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    tmp[lane] = x - w;                 // exclusive prefix of warp counts
    if (lane == 31) res[4] = x;        // candidates of this CTA
  }
  __syncthreads();
  const uint32_t nc = res[4];
  // (b) write in position order into the local candidate arrays
  if (nc <= (uint32_t)kTopkCandCap) {
    uint32_t wpos = tmp[warp];
    const uint32_t lanes_below = (1u << lane) - 1u;
    for (int64_t i0 = s_lo; i0 < s_hi; i0 += 128) {
      const int64_t e0 = i0 + 4 * lane;
      uint32_t kk[4];
      load4(e0, kk);
      uint32_t flags = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) flags |= ((e0 + e < s_hi) && ((kk[e] >> 21) >= b1)) ? (1u << e) : 0u;
      // Candidates of lower lanes come first (position order): one ballot per
      // element slot gives both this lane's offset and the warp's total.
      uint32_t before = 0, total = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t bal = __ballot_sync(0xffffffffu, (flags >> e) & 1u);
        before += __popc(bal & lanes_below);
        total += __popc(bal);
      }
      uint32_t at = wpos + before;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (flags & (1u << e)) {
          cand_key[at] = staged16 ? score_key(row[lo + e0 + e]) : kk[e];
          cand_pos[at] = (int32_t)(lo + e0 + e);
          ++at;
        }
      }
      wpos += total;
    }
  }
  // ---- gather the cluster's candidates, in rank (= position) order, in rank 0
  if (threadIdx.x == 0) cnt[3] = nc;
  cluster_barrier<CL>();
  uint32_t off = 0, n_all = 0;
  if constexpr (CL > 1) {
    cg::cluster_group cl = cg::this_cluster();
    for (int r = 0; r < CL; ++r) {
      const uint32_t c = cl.map_shared_rank(cnt, r)[3];
      if (r < rank) off += c;
      n_all += c;
    }
  } else {
    n_all = nc;
  }
  const bool overflow = n_all > (uint32_t)kTopkCandCap;   // the same in every CTA
  if (!overflow) {
    if constexpr (CL > 1) {
      if (rank != 0) {
        cg::cluster_group cl = cg::this_cluster();
        uint32_t* dk = cl.map_shared_rank(cand_key, 0);
        int32_t* dp = cl.map_shared_rank(cand_pos, 0);
        for (uint32_t i = threadIdx.x; i < nc; i += kTopkThreads) {
          dk[off + i] = cand_key[i];
          dp[off + i] = cand_pos[i];
        }
      }
    }
    cluster_barrier<CL>();   // rank 0 holds every candidate; the other CTAs are done
    if (rank != 0) return;
  }

  // From here: rank 0 alone on the gathered candidates, or (overflow) every CTA
  // of the cluster on its whole slice with cluster-wide reductions.
  const uint32_t n_items = overflow ? (uint32_t)len : n_all;
  auto item_key = [&](uint32_t i) -> uint32_t { return overflow ? key_at(i) : cand_key[i]; };
  auto item_pos = [&](uint32_t i) -> int32_t { return overflow ? (int32_t)(lo + i) : cand_pos[i]; };
  auto sum_hist = [&](int nb) {
    if (overflow) {
      if (nb == kTopkBins) cluster_sum_hist<CL, kTopkBins>(hist, tot);
      else cluster_sum_hist<CL, 1024>(hist, tot);
    } else {
      __syncthreads();
      for (int b = threadIdx.x; b < nb; b += kTopkThreads) tot[b] = hist[b];
      __syncthreads();
    }
  };

  // ---- pass 2: next 11 bits of keys in bin b1
  for (int b = threadIdx.x; b < kTopkBins; b += kTopkThreads) hist[b] = 0;
  __syncthreads();
  for (uint32_t i = threadIdx.x; i < n_items; i += kTopkThreads) {
    const uint32_t kk = item_key(i);
    if ((kk >> 21) == b1) atomicAdd(&hist[(kk >> 10) & 0x7FFu], 1u);
  }
  __syncthreads();
  sum_hist(kTopkBins);
  find_threshold_bin<kTopkBins>(tot, need, tmp, res);
  const uint32_t pre2 = (b1 << 11) | res[0];
  above += res[1];
  need -= res[1];

  // ---- pass 3: last 10 bits of keys with prefix pre2
  for (int b = threadIdx.x; b < 1024; b += kTopkThreads) hist[b] = 0;
  __syncthreads();
  for (uint32_t i = threadIdx.x; i < n_items; i += kTopkThreads) {
    const uint32_t kk = item_key(i);
    if ((kk >> 10) == pre2) atomicAdd(&hist[kk & 0x3FFu], 1u);
  }
  __syncthreads();
  sum_hist(1024);
  find_threshold_bin<1024>(tot, need, tmp, res);
  const uint32_t tau = (pre2 << 10) | res[0];
  need -= res[1];                 // keys == tau still to take (>= 1)
  const uint32_t need_eq = need;

  // ---- what precedes this CTA's items in position order (only with overflow
  // is the selection spread over several CTAs)
  uint32_t base_gt = 0, base_eq = 0;
  if (overflow) {
    uint32_t my_gt = 0, my_eq = 0;
    for (uint32_t i = threadIdx.x; i < n_items; i += kTopkThreads) {
      const uint32_t kk = item_key(i);
      my_gt += (kk > tau);
      my_eq += (kk == tau);
    }
    uint32_t tg, te;
    block_excl_scan(my_gt, tmp, &tg);
    block_excl_scan(my_eq, tmp, &te);
    if (threadIdx.x == 0) {
      cnt[0] = tg;
      cnt[1] = te;
    }
    cluster_barrier<CL>();
    if constexpr (CL > 1) {
      cg::cluster_group cl = cg::this_cluster();
      for (int r = 0; r < rank; ++r) {
        const uint32_t* pc = cl.map_shared_rank(cnt, r);
        base_gt += pc[0];
        base_eq += pc[1];
      }
    }
    cluster_barrier<CL>();  // peers finished reading cnt (the CTA may exit after this)
  }

  // ---- ordered output: 4 consecutive items (in position order) per thread per round
  for (uint32_t r0 = 0; r0 < n_items; r0 += 4 * kTopkThreads) {
    const uint32_t i0 = r0 + 4 * threadIdx.x;
    uint32_t kk[4];
    uint32_t c_gt = 0, c_eq = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      kk[e] = (i0 + e < n_items) ? item_key(i0 + e) : 0u;
      c_gt += (i0 + e < n_items) && (kk[e] > tau);
      c_eq += (i0 + e < n_items) && (kk[e] == tau);
    }
    uint32_t total;
    const uint32_t ex = block_excl_scan((c_gt << 16) | c_eq, tmp, &total);
    uint32_t g = base_gt + (ex >> 16), q = base_eq + (ex & 0xFFFFu);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (i0 + e < n_items) {
        if (kk[e] > tau) {
          const uint32_t slot = g + min(q, need_eq);
          if (slot < (uint32_t)p.k) out[slot] = item_pos(i0 + e);
          ++g;
        } else if (kk[e] == tau) {
          if (q < need_eq && g + q < (uint32_t)p.k) out[g + q] = item_pos(i0 + e);
          ++q;
        }
      }
    }
    base_gt += total >> 16;
    base_eq += total & 0xFFFFu;
  }
  if (rank == 0 && threadIdx.x == 0) p.count[t] = p.k;
  (void)above;
}

template <int CL>
__global__ void __launch_bounds__(kTopkThreads, 1) topk_kernel(const TopkParams p) {
  griddep_wait();
  const int t = blockIdx.x / CL;
  int rank = 0;
  if constexpr (CL > 1) rank = (int)cg::this_cluster().block_rank();
  if (t >= p.T) return;  // whole clusters only: T * CL blocks are launched
  topk_query<CL>(p, t, rank);
}

// ------------------------------------------------------------------ selection from the indexer's histogram
struct TopkHistParams {
  TopkParams base;
  const uint32_t* hist;   // [T, 2048]: the query's candidate keys counted by their top 11 bits
  uint32_t* cand_key;     // [T, S, kTopkCandCap] candidates of each slice, in position order
  int32_t* cand_pos;      // [T, S, kTopkCandCap]
  uint32_t* cand_cnt;     // [T, S]: candidates of the slice (kTopkNoList: none written)
  uint32_t* bin_info;     // [T, 4]: (b1, keys above bin b1, keys in bin b1) as the filter read them
  int32_t S;              // slices per query
};
constexpr uint32_t kTopkNoList = 0xFFFFFFFFu;

// The float whose order-preserving key is `key` (score_key's inverse on keys
// of non-NaN floats).  For a bin b with 4 <= b: a non-NaN score x has
// score_key(x) >= b << 21 exactly when x >= bin_floor(b), and a NaN score (key
// of -inf, in bin 3) has neither; for b >= 2045 the floor is a NaN, so the
// comparison is false for every score, as no key lies that high.  Bins 0-3
// (every key qualifies, NaN included) need the key itself.
__device__ __forceinline__ float bin_floor(uint32_t b) {
  const uint32_t key = b << 21;
  return __uint_as_float((key & 0x80000000u) ? (key ^ 0x80000000u) : ~key);
}

// Query t's candidate count n (0 when q_pos < 0; clamped to ld, flagged).
__device__ __forceinline__ int64_t topk_row_len(const TopkParams& p, int t, bool report) {
  int qp = p.q_pos[t];
  if (qp >= p.ld) {
    if (report) raise_error(kErrBadSeq);
    qp = (int)p.ld - 1;
  }
  return (qp < 0) ? 0 : (int64_t)qp + 1;
}

// k-th bin of the query's histogram (copied to `h` in shared memory): writes
// (b1, keys in bins above b1, keys in bin b1) to res[0..2].
__device__ __forceinline__ void topk_bin_from_hist(const uint32_t* g_hist, uint32_t* h, uint32_t k, uint32_t* tmp,
                                                   uint32_t* res) {
  for (int b = threadIdx.x; b < kTopkBins; b += kTopkThreads) h[b] = g_hist[b];
  if (threadIdx.x == 0) {
    res[0] = kTopkNoList;
    res[1] = 0;
  }
  __syncthreads();
  find_threshold_bin<kTopkBins>(h, k, tmp, res);
  if (threadIdx.x == 0) res[2] = (res[0] == kTopkNoList) ? 0u : h[res[0]];
  __syncthreads();
}

// The last two radix passes and the ordered output over items gathered in
// shared memory in position order (one CTA): b1 is the k-th key's top-11-bit
// bin and `above` the number of items in higher bins.  Writes the k selected
// positions to out[0..k) in ascending order.
__device__ __forceinline__ void finish_gathered(const uint32_t* gkey, const int32_t* gpos, uint32_t n_items,
                                                uint32_t b1, uint32_t above, uint32_t k, int32_t* out,
                                                uint32_t* hist, uint32_t* tmp, uint32_t* res) {
  uint32_t need = k - above;
  // ---- pass 2: next 11 bits of keys in bin b1
  for (int b = threadIdx.x; b < kTopkBins; b += kTopkThreads) hist[b] = 0;
  __syncthreads();
  for (uint32_t i = threadIdx.x; i < n_items; i += kTopkThreads) {
    const uint32_t kk = gkey[i];
    if ((kk >> 21) == b1) atomicAdd(&hist[(kk >> 10) & 0x7FFu], 1u);
  }
  __syncthreads();
  find_threshold_bin<kTopkBins>(hist, need, tmp, res);
  const uint32_t pre2 = (b1 << 11) | res[0];
  need -= res[1];
  // ---- pass 3: last 10 bits of keys with prefix pre2
  for (int b = threadIdx.x; b < 1024; b += kTopkThreads) hist[b] = 0;
  __syncthreads();
  for (uint32_t i = threadIdx.x; i < n_items; i += kTopkThreads) {
    const uint32_t kk = gkey[i];
    if ((kk >> 10) == pre2) atomicAdd(&hist[kk & 0x3FFu], 1u);
  }
  __syncthreads();
  find_threshold_bin<1024>(hist, need, tmp, res);
  const uint32_t tau = (pre2 << 10) | res[0];
  need -= res[1];
  const uint32_t need_eq = need;
  // ---- ordered output: 4 consecutive items (in position order) per thread per round
  uint32_t base_gt = 0, base_eq = 0;
  for (uint32_t r0 = 0; r0 < n_items; r0 += 4 * kTopkThreads) {
    const uint32_t i0 = r0 + 4 * threadIdx.x;
    uint32_t kk[4];
    uint32_t c_gt = 0, c_eq = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      kk[e] = (i0 + e < n_items) ? gkey[i0 + e] : 0u;
      c_gt += (i0 + e < n_items) && (kk[e] > tau);
      c_eq += (i0 + e < n_items) && (kk[e] == tau);
    }
    uint32_t total;
    const uint32_t ex = block_excl_scan((c_gt << 16) | c_eq, tmp, &total);
    uint32_t g = base_gt + (ex >> 16), q = base_eq + (ex & 0xFFFFu);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (i0 + e < n_items) {
        if (kk[e] > tau) {
          const uint32_t slot = g + min(q, need_eq);
          if (slot < k) out[slot] = gpos[i0 + e];
          ++g;
        } else if (kk[e] == tau) {
          if (q < need_eq && g + q < k) out[g + q] = gpos[i0 + e];
          ++q;
        }
      }
    }
    base_gt += total >> 16;
    base_eq += total & 0xFFFFu;
  }
}

// Keys of one slice with their top 11 bits >= b1, in position order, into
// warp-private lists.  The slice streams into shared memory by bulk copies of
// up to kTopkStashCap scores (issued before the k-th bin is read from the
// histogram, so the copy overlaps it); the last < 4 scores come by plain loads.
__global__ void __launch_bounds__(kTopkThreads, 1) topk_filter_kernel(const TopkHistParams hp) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem_raw);
  uint32_t* tmp = hist + 2 * kTopkBins;
  uint32_t* res = tmp + 40;
  uint64_t* bar = reinterpret_cast<uint64_t*>(res + 8);
  float* chunk = reinterpret_cast<float*>(smem_raw + 2 * kTopkBins * 4 + 1024);     // [kTopkStashCap]
  uint32_t* wkey = reinterpret_cast<uint32_t*>(chunk + kTopkStashCap);                  // warp lists
  int32_t* wposs = reinterpret_cast<int32_t*>(wkey + kTopkCandCap);
  const TopkParams& p = hp.base;
  const int t = blockIdx.x / hp.S;
  const int s = blockIdx.x - t * hp.S;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();
  uint32_t* cnt_out = hp.cand_cnt + (int64_t)t * hp.S + s;
  const int64_t n = topk_row_len(p, t, false);
  if (n <= p.k) {
    if (threadIdx.x == 0) *cnt_out = kTopkNoList;
    return;
  }
  // this slice of the row
  const float* row = p.scores + (int64_t)t * p.ld;
  const int64_t lo = ((int64_t)s * n / hp.S) & ~int64_t(3);
  const int64_t hi = (s == hp.S - 1) ? n : (((int64_t)(s + 1) * n / hp.S) & ~int64_t(3));
  const int64_t len = hi - lo;
  const int64_t len4 = len & ~int64_t(3);                // the part the bulk copies take
  auto issue = [&](int64_t c0) {
    const int64_t c = min((int64_t)kTopkStashCap, len4 - c0);
    if (threadIdx.x == 0 && c > 0) {
      mbar_arrive_expect_tx(bar, (uint32_t)(c * 4));
      bulk_load_g2s(chunk, row + lo + c0, (uint32_t)(c * 4), bar);
    }
  };
  issue(0);
  topk_bin_from_hist(hp.hist + (int64_t)t * kTopkBins, hist, (uint32_t)p.k, tmp, res);
  const uint32_t b1 = res[0];
  const bool give_up = b1 == kTopkNoList || (uint64_t)res[1] + res[2] > (uint64_t)kTopkCandCap;
  if (s == 0 && threadIdx.x < 3) hp.bin_info[(int64_t)t * 4 + threadIdx.x] = res[threadIdx.x];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kWarps = kTopkThreads / 32;
  constexpr uint32_t WCAP = kTopkCandCap / kWarps;
  const uint32_t lanes_below = (1u << lane) - 1u;
  uint32_t* wk = wkey + warp * WCAP;
  int32_t* wp = wposs + warp * WCAP;
  uint32_t wcount = 0;
  bool ok = true;
  uint32_t phase = 0;
  // A score is kept when its key's top 11 bits are >= b1: a float comparison
  // against the bin's floor (keys are made only for the kept scores).
  const bool keep_all = b1 <= 3u;
  const float floor_b1 = bin_floor(b1 & 0x7FFu);
  for (int64_t c0 = 0; c0 < len; c0 += kTopkStashCap) {
    const int c_len = (int)min((int64_t)kTopkStashCap, len - c0);     // scores of this chunk
    const int c_bulk = (int)max((int64_t)0, min((int64_t)c_len, len4 - c0));   // of which came by bulk copy
    if (c_bulk > 0) {
      const bool got = ok && mbar_wait(bar, phase, nullptr);   // every thread waits (bounded)
      ok = __syncthreads_and(got) != 0;                         // the same verdict in every thread
      phase ^= 1u;
    }
    // Warp w owns a contiguous segment of the chunk (a multiple of 128 scores).
    const int seg = ((c_len + kWarps - 1) / kWarps + 127) & ~127;
    const int s_lo = min(warp * seg, c_len);
    const int s_hi = min(s_lo + seg, c_len);
    const float* tail = row + lo + c0;   // scores past the bulk-copied part
    if (!give_up && ok) {
      for (int e0 = s_lo + 4 * lane; e0 - 4 * lane < s_hi; e0 += 128) {
        float f[4];
        if (e0 + 3 < c_bulk) {
          const float4 v = *reinterpret_cast<const float4*>(chunk + e0);
          f[0] = v.x;
          f[1] = v.y;
          f[2] = v.z;
          f[3] = v.w;
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = e0 + e;
            f[e] = (i < s_hi) ? (i < c_bulk ? chunk[i] : tail[i]) : 0.f;
          }
        }
        uint32_t flags = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) flags |= ((e0 + e < s_hi) && (keep_all || f[e] >= floor_b1)) ? (1u << e) : 0u;
        if (__any_sync(0xffffffffu, flags != 0)) {
          uint32_t kk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) kk[e] = score_key(f[e]);
          uint32_t before = 0, total = 0;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t bal = __ballot_sync(0xffffffffu, (flags >> e) & 1u);
            before += __popc(bal & lanes_below);
            total += __popc(bal);
          }
          uint32_t at = wcount + before;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (flags & (1u << e)) {
              if (at < WCAP) {
                wk[at] = kk[e];
                wp[at] = (int32_t)(lo + c0 + e0 + e);
              }
              ++at;
            }
          }
          wcount += total;
        }
      }
    }
    __syncthreads();                     // the chunk is no longer read
    if (ok) issue(c0 + kTopkStashCap);   // the next one (none past the bulk part, none after a failed wait)
  }
  if (give_up || !ok) {
    if (threadIdx.x == 0) *cnt_out = kTopkNoList;   // the select kernel runs the whole row
    return;
  }
  // warp offsets, the slice's count, overflow
  if (lane == 0) tmp[warp] = wcount;
  __syncthreads();
  if (warp == 0) {
    const uint32_t w = tmp[lane];
    uint32_t x = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    const bool over = __any_sync(0xffffffffu, w > WCAP);
    tmp[lane] = x - w;
    if (lane == 31) res[3] = (over || x > (uint32_t)kTopkCandCap) ? kTopkNoList : x;
  }
  __syncthreads();
  const uint32_t nc = res[3];
  if (nc != kTopkNoList) {
    const int64_t base = ((int64_t)t * hp.S + s) * kTopkCandCap + tmp[warp];
    for (uint32_t i = lane; i < wcount; i += 32) {
      hp.cand_key[base + i] = wk[i];
      hp.cand_pos[base + i] = wp[i];
    }
  }
  if (threadIdx.x == 0) *cnt_out = nc;
}

__global__ void __launch_bounds__(kTopkThreads, 1) topk_select_kernel(const TopkHistParams hp) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem_raw);
  uint32_t* tmp = hist + 2 * kTopkBins;
  uint32_t* res = tmp + 40;
  uint32_t* gkey = reinterpret_cast<uint32_t*>(smem_raw + 2 * kTopkBins * 4 + 1024);   // gathered candidates
  int32_t* gpos = reinterpret_cast<int32_t*>(gkey + kTopkCandCap);
  griddep_launch_dependents();   // one CTA per query: the attention may set up on the idle SMs meanwhile
  griddep_wait();
  const TopkParams& p = hp.base;
  const int t = blockIdx.x;
  if (t >= p.T) return;
  const int64_t n = topk_row_len(p, t, threadIdx.x == 0);
  int32_t* out = p.idx + (int64_t)t * p.k;
  if (n <= p.k) {  // every candidate is kept
    for (int64_t i = threadIdx.x; i < p.k; i += kTopkThreads) out[i] = (i < n) ? (int32_t)i : -1;
    if (threadIdx.x == 0) p.count[t] = (int32_t)n;
    return;
  }
  // the k-th bin as the filter read it from the histogram
  const uint32_t b1 = hp.bin_info[(int64_t)t * 4];
  uint32_t above = hp.bin_info[(int64_t)t * 4 + 1];
  const uint32_t n_cand = above + hp.bin_info[(int64_t)t * 4 + 2];
  // Every slice's list must be there and add up to the histogram's count
  // (warp 0: counts, their prefix in `offs`, the verdict in res[4]).
  uint32_t* offs = hist + kTopkBins;   // [S + 1]
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    bool bad = b1 == kTopkNoList || n_cand > (uint32_t)kTopkCandCap;
    uint32_t run = 0;
    for (int s0 = 0; s0 < hp.S; s0 += 32) {
      const int s = s0 + lane;
      const uint32_t c = (s < hp.S) ? hp.cand_cnt[(int64_t)t * hp.S + s] : 0u;
      bad |= __any_sync(0xffffffffu, c == kTopkNoList);
      const uint32_t cc = (c == kTopkNoList) ? 0u : c;
      uint32_t x = cc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (s < hp.S) offs[s] = run + x - cc;
      run += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) {
      offs[hp.S] = run;
      res[4] = (!bad && run == n_cand) ? 1u : 0u;
      res[5] = 0;
      res[6] = 0;
    }
  }
  __syncthreads();
  if (res[4] == 0u) {
    topk_query<1>(p, t, 0);   // the single-CTA algorithm on the whole row
    return;
  }
  // gather the slices' lists in slice (= position) order: item i of the query
  // lies in the slice s with offs[s] <= i < offs[s + 1] (binary search); the
  // keys above and in bin b1 are recounted: they must be the histogram's
  // counts, or b1 is not the row's k-th bin (a histogram that does not belong
  // to these scores)
  {
    // Warp w copies items [w n / 32, (w + 1) n / 32): its first slice is found
    // once, later ones by stepping forward; four items per lane are in flight.
    uint32_t my_gt = 0, my_eq = 0;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int kWarps = kTopkThreads / 32;
    const uint32_t w_lo = (uint32_t)((uint64_t)warp * n_cand / kWarps);
    const uint32_t w_hi = (uint32_t)((uint64_t)(warp + 1) * n_cand / kWarps);
    int s = 0;   // offs[s] <= i < offs[s + 1] for the lane's current item i
    {
      int s_lo = 0, s_hi = hp.S;
      while (s_hi - s_lo > 1) {
        const int mid = (s_lo + s_hi) >> 1;
        if (offs[mid] <= w_lo) s_lo = mid;
        else s_hi = mid;
      }
      s = s_lo;
    }
    const int64_t lists = (int64_t)t * hp.S * kTopkCandCap;
    for (uint32_t i0 = w_lo; i0 < w_hi; i0 += 4 * 32) {
      uint32_t kk[4];
      int32_t pp[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t i = i0 + 32 * e + lane;
        kk[e] = 0u;
        pp[e] = -1;
        if (i < w_hi) {
          while (offs[s + 1] <= i) ++s;
          const int64_t src = lists + (int64_t)s * kTopkCandCap + (i - offs[s]);
          kk[e] = hp.cand_key[src];
          pp[e] = hp.cand_pos[src];
        }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t i = i0 + 32 * e + lane;
        if (i < w_hi) {
          gkey[i] = kk[e];
          gpos[i] = pp[e];
          my_gt += (kk[e] >> 21) > b1;
          my_eq += (kk[e] >> 21) == b1;
        }
      }
    }
    if (my_gt) atomicAdd(&res[5], my_gt);
    if (my_eq) atomicAdd(&res[6], my_eq);
  }
  __syncthreads();
  if (res[5] != above || res[6] != n_cand - above || above >= (uint32_t)p.k) {
    __syncthreads();
    topk_query<1>(p, t, 0);
    return;
  }
  finish_gathered(gkey, gpos, n_cand, b1, above, (uint32_t)p.k, out, hist, tmp, res);
  if (threadIdx.x == 0) p.count[t] = p.k;
}

// ---------------------------------------------------------------------------
// Rows that fit in shared memory (at most kTopkRowCap candidates), with the
// indexer's histogram: one CTA per query stages its whole row once (bulk
// copies, overlapping the read of the histogram) and finishes alone:
//   A  scores above the k-th bin b1 (a float comparison against the bin's
//      floor) are marked in a position bitmap (one warp ballot per 32 positions);
//      keys in b1 are counted by their next 11 bits and their positions listed
//      (each warp appends to its own segment of the list, so no counter is
//      shared);
//   B  over that list: keys above the second threshold bin are marked; keys on
//      it (the prefix of the final threshold) are counted by their last 10 bits
//      and listed again; the short list then gives tau, the keys above it and
//      the ties, of which the lowest-positioned need_eq are kept (a block scan
//      over the tie bitmap's words in position order).
// A last block scan over the bitmap words writes the positions in ascending
// order.  A histogram that does not match the staged keys is replaced by one
// counted from them; lists that overflow fall back to passes over the row.
constexpr int kTopkRowCap = 40960;
constexpr int kTopkRowListCap = 10240;
constexpr int kTopkRowSegCap = kTopkRowListCap / (kTopkThreads / 32);   // list entries per warp
constexpr int kTopkRowList2Cap = kTopkBins;   // the second list reuses the second histogram
constexpr int kTopkRowWords = kTopkRowCap / 32;
constexpr int kTopkRowSmemBytes =
    kTopkRowCap * 4 + 2 * kTopkRowWords * 4 + 2 * kTopkBins * 4 + kTopkRowListCap * 4 + 1024;
static_assert(kTopkRowWords <= 2 * kTopkThreads, "two bitmap words per thread");
static_assert(kTopkRowSmemBytes <= 232448, "shared memory per block");

__global__ void __launch_bounds__(kTopkThreads, 1) topk_row_kernel(const TopkHistParams hp) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  float* row = reinterpret_cast<float*>(smem_raw);                               // [kTopkRowCap] scores
  uint32_t* sel = reinterpret_cast<uint32_t*>(row + kTopkRowCap);                // selected positions
  uint32_t* tie = sel + kTopkRowWords;                                           // keys equal to tau
  uint32_t* h = tie + kTopkRowWords;                                             // [2048] first / third pass
  uint32_t* h2 = h + kTopkBins;                                                  // [2048] second pass, then list 2
  int32_t* list = reinterpret_cast<int32_t*>(h2 + kTopkBins);                    // positions in bin b1
  uint32_t* tmp = reinterpret_cast<uint32_t*>(list + kTopkRowListCap);           // scan scratch (40)
  uint32_t* res = tmp + 40;                                                      // [8]
  uint32_t* cnt = res + 8;                                                       // [4]
  uint32_t* seg_n = cnt + 4;                                                     // [32] list entries per warp
  uint64_t* bar = reinterpret_cast<uint64_t*>(seg_n + kTopkThreads / 32);
  const TopkParams& p = hp.base;
  const int t = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  griddep_launch_dependents();   // the attention may set up on the SMs this launch leaves idle
  griddep_wait();
  const int n = (int)topk_row_len(p, t, tid == 0);   // <= kTopkRowCap
  const uint32_t k = (uint32_t)p.k;
  int32_t* out = p.idx + (int64_t)t * p.k;
  if (n <= (int)k) {   // every candidate is selected
    for (int i = tid; i < (int)k; i += kTopkThreads) out[i] = (i < n) ? i : -1;
    if (tid == 0) p.count[t] = n;
    return;
  }
  const float* grow = p.scores + (int64_t)t * p.ld;
  const int n4 = (n + 3) & ~3;   // <= ld: whole 16-byte pieces of the row
  if (tid == 0) {
    mbar_arrive_expect_tx(bar, (uint32_t)(n4 * 4));
    for (int c0 = 0; c0 < n4; c0 += 8192) bulk_load_g2s(row + c0, grow + c0, (uint32_t)(min(8192, n4 - c0) * 4), bar);
  }
  const int nw = (n + 31) >> 5;
  for (int w = tid; w < nw; w += kTopkThreads) tie[w] = 0u;
  topk_bin_from_hist(hp.hist + (int64_t)t * kTopkBins, h, k, tmp, res);
  uint32_t b1 = res[0], above = res[1], in_b1 = res[2];
  const bool got = mbar_wait(bar, 0, nullptr);
  if (!__syncthreads_and(got)) return;   // timed out (flagged)
  const uint32_t lanes_below = (1u << lane) - 1u;
  auto key_at = [&](int pos) -> uint32_t { return score_key(row[pos]); };
  // ---- pass A.  For 4 <= b1 <= 2043 the bin test is a float comparison
  // against the floors of bins b1 and b1 + 1 (keys only for the scores in b1).
  for (int attempt = 0; attempt < 2; ++attempt) {
    const bool by_floor = b1 >= 4u && b1 <= 2043u;
    const float f_b1 = bin_floor(by_floor ? b1 : 4u), f_b2 = bin_floor(by_floor ? b1 + 1u : 5u);
    for (int b = tid; b < kTopkBins; b += kTopkThreads) h2[b] = 0u;
    if (tid == 0) {
      cnt[0] = 0;
      cnt[1] = 0;
    }
    __syncthreads();
    uint32_t my_gt = 0;
    uint32_t my_eq = 0;   // entries of this warp's list segment (the same in every lane)
    int32_t* seg = list + warp * kTopkRowSegCap;
#pragma unroll 2
    for (int base = 0; base < n; base += kTopkThreads) {
      const int pos = base + tid;
      const bool valid = pos < n;
      const float x = valid ? row[pos] : 0.f;
      bool gt, eq;
      if (by_floor) {
        gt = valid && x >= f_b2;
        eq = valid && !gt && x >= f_b1;
      } else {
        const uint32_t bin = score_key(x) >> 21;
        gt = valid && bin > b1;
        eq = valid && bin == b1;
      }
      const uint32_t bg = __ballot_sync(0xffffffffu, gt);
      if (lane == 0) sel[(base >> 5) + warp] = bg;
      my_gt += __popc(bg);
      const uint32_t be = __ballot_sync(0xffffffffu, eq);
      if (eq) {
        atomicAdd(&h2[(score_key(x) >> 10) & 0x7FFu], 1u);
        const uint32_t at = my_eq + __popc(be & lanes_below);
        if (at < (uint32_t)kTopkRowSegCap) seg[at] = pos;
      }
      my_eq += __popc(be);
    }
    if (lane == 0) {
      seg_n[warp] = my_eq;
      if (my_gt) atomicAdd(&cnt[1], my_gt);
      if (my_eq) atomicAdd(&cnt[0], my_eq);
    }
    __syncthreads();
    if (b1 != kTopkNoList && cnt[1] == above && cnt[0] == in_b1) break;
    // The histogram does not describe these keys: count them here and redo the pass.
    for (int b = tid; b < kTopkBins; b += kTopkThreads) h[b] = 0u;
    __syncthreads();
    for (int pos = tid; pos < n; pos += kTopkThreads) atomicAdd(&h[key_at(pos) >> 21], 1u);
    if (tid == 0) {
      res[0] = kTopkNoList;
      res[1] = 0;
    }
    __syncthreads();
    find_threshold_bin<kTopkBins>(h, k, tmp, res);
    b1 = res[0];
    above = res[1];
    in_b1 = (b1 == kTopkNoList) ? 0u : h[b1];
    __syncthreads();
  }
  bool use_list = true;   // every warp's segment held its entries
#pragma unroll
  for (int w = 0; w < kTopkThreads / 32; ++w) use_list &= seg_n[w] <= (uint32_t)kTopkRowSegCap;
  uint32_t need = k - above;
  find_threshold_bin<kTopkBins>(h2, need, tmp, res);
  const uint32_t b2 = res[0];
  need -= res[1];
  const uint32_t pre2 = (b1 << 11) | b2;
  // ---- pass B over the keys of bin b1
  int32_t* list2 = reinterpret_cast<int32_t*>(h2);   // h2 is no longer needed
  for (int b = tid; b < 1024; b += kTopkThreads) h[b] = 0u;
  if (tid == 0) cnt[2] = 0;
  __syncthreads();
  auto visit_b = [&](int pos, uint32_t key) {
    const uint32_t sub = (key >> 10) & 0x7FFu;
    if (sub > b2) {
      atomicOr(&sel[pos >> 5], 1u << (pos & 31));
    } else if (sub == b2) {
      atomicAdd(&h[key & 0x3FFu], 1u);
      const uint32_t at = atomicAdd(&cnt[2], 1u);
      if (at < (uint32_t)kTopkRowList2Cap) list2[at] = pos;
    }
  };
  if (use_list) {
    // warp w walks segment w
    const uint32_t nseg = seg_n[warp];
    const int32_t* seg = list + warp * kTopkRowSegCap;
    for (uint32_t i = lane; i < nseg; i += 32) {
      const int pos = seg[i];
      visit_b(pos, key_at(pos));
    }
  } else {
    for (int pos = tid; pos < n; pos += kTopkThreads) {
      const uint32_t key = key_at(pos);
      if ((key >> 21) == b1) visit_b(pos, key);
    }
  }
  __syncthreads();
  find_threshold_bin<1024>(h, need, tmp, res);
  const uint32_t tau = (pre2 << 10) | res[0];
  const uint32_t need_eq = need - res[1];
  const uint32_t n_list2 = cnt[2];
  // keys with prefix pre2 above tau are selected; keys equal to tau are ties
  auto mark = [&](int pos, uint32_t key) {
    if (key > tau) atomicOr(&sel[pos >> 5], 1u << (pos & 31));
    else if (key == tau) atomicOr(&tie[pos >> 5], 1u << (pos & 31));
  };
  if (n_list2 <= (uint32_t)kTopkRowList2Cap) {
    for (uint32_t i = tid; i < n_list2; i += kTopkThreads) {
      const int pos = list2[i];
      mark(pos, key_at(pos));
    }
  } else {
    for (int pos = tid; pos < n; pos += kTopkThreads) {
      const uint32_t key = key_at(pos);
      if ((key >> 10) == pre2) mark(pos, key);
    }
  }
  __syncthreads();
  // ---- ties: the need_eq lowest positions (thread i owns bitmap words 2i, 2i + 1)
  const int w0 = 2 * tid, w1 = w0 + 1;
  {
    const uint32_t t0 = (w0 < nw) ? tie[w0] : 0u, t1 = (w1 < nw) ? tie[w1] : 0u;
    uint32_t total;
    uint32_t before = block_excl_scan((uint32_t)(__popc(t0) + __popc(t1)), tmp, &total);
    uint32_t tw[2] = {t0, t1};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      uint32_t x = tw[e], keep = 0u;
      while (x && before < need_eq) {
        const uint32_t low = x & (0u - x);
        keep |= low;
        x ^= low;
        ++before;
      }
      if (keep) sel[w0 + e] |= keep;   // each word has one owner: no race
    }
  }
  __syncthreads();
  // ---- ordered output
  {
    const uint32_t s0 = (w0 < nw) ? sel[w0] : 0u, s1 = (w1 < nw) ? sel[w1] : 0u;
    uint32_t total;
    uint32_t at = block_excl_scan((uint32_t)(__popc(s0) + __popc(s1)), tmp, &total);
    uint32_t sw[2] = {s0, s1};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      uint32_t x = sw[e];
      while (x) {
        const int b = __ffs(x) - 1;
        x &= x - 1u;
        if (at < k) out[at] = 32 * (w0 + e) + b;
        ++at;
      }
    }
    if (total != k && tid == 0) raise_error(kErrBadIndex);   // cannot happen: the passes count exactly k
    for (uint32_t i = total + tid; i < k; i += kTopkThreads) out[i] = -1;
    if (tid == 0) p.count[t] = (int32_t)min(total, k);
  }
}

// ------------------------------------------------------------------ context-parallel decode
// Report's serving section (context-parallel decode: each rank selects among
// its own positions, the candidates are exchanged, then merged).

// A rank's selection as (score, global position) candidates: for i < count[t],
// out_score[t, i] = scores[t, idx[t, i]] and out_pos = idx[t, i] + pos_offset;
// -inf / -1 elsewhere (also for -1 entries).
__global__ void __launch_bounds__(256) topk_export_kernel(const float* scores, int64_t ld, const int32_t* idx,
                                                          const int32_t* count, int32_t T, int32_t k,
                                                          int64_t pos_offset, float* out_score, int32_t* out_pos) {
  griddep_wait();
  const int t = blockIdx.x;
  if (t >= T) return;
  int c = count[t];
  c = c < 0 ? 0 : (c > k ? k : c);
  for (int i = threadIdx.x; i < k; i += blockDim.x) {
    const int32_t q = (i < c) ? idx[(int64_t)t * k + i] : -1;
    const bool ok = q >= 0 && q < ld;
    out_score[(int64_t)t * k + i] = ok ? scores[(int64_t)t * ld + q] : -INFINITY;
    out_pos[(int64_t)t * k + i] = ok ? (int32_t)(q + pos_offset) : -1;
  }
}

constexpr int kMergeCap = 16384;   // candidates per query the merge holds (in the stash region)

struct MergeParams {
  const float* cand_score;   // [R, T, kr]
  const int32_t* cand_pos;   // [R, T, kr]: global positions, -1 = empty slot
  int64_t shard_lo;          // this rank's positions [shard_lo, shard_hi)
  int64_t shard_hi;
  int32_t* idx_global;       // [T, k] or null
  int32_t* idx_local;        // [T, k] or null: the selected positions inside the shard, as
                             // position - shard_lo, ascending and compacted, -1 after them
  int32_t* count_local;      // [T] (with idx_local): how many there are
  int32_t* count;            // [T]
  int32_t R, T, kr, k;
};

// Global top-k of one query from every rank's candidates (ranks hold disjoint
// position ranges in rank order and list their candidates in ascending order,
// so the concatenation is in position order).  Same rule as topk_kernel:
// higher score first, ties to the lower position, -0 == +0, NaN as -inf.
__global__ void __launch_bounds__(kTopkThreads, 1) topk_merge_kernel(const MergeParams mp) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem_raw);
  uint32_t* tmp = hist + 2 * kTopkBins;
  uint32_t* res = tmp + 40;
  uint32_t* gkey = reinterpret_cast<uint32_t*>(smem_raw + 2 * kTopkBins * 4 + 1024);   // [kMergeCap]
  int32_t* gpos = reinterpret_cast<int32_t*>(gkey + kMergeCap);                       // [kMergeCap]
  int32_t* sel = gpos + kMergeCap;                                                     // [k]
  griddep_wait();
  const int t = blockIdx.x;
  if (t >= mp.T) return;
  // ordered compaction of the valid candidates: 4 consecutive slots per thread per round
  const uint32_t n_in = (uint32_t)mp.R * (uint32_t)mp.kr;
  uint32_t n_items = 0;
  for (uint32_t r0 = 0; r0 < n_in; r0 += 4 * kTopkThreads) {
    const uint32_t i0 = r0 + 4 * threadIdx.x;
    uint32_t kk[4];
    int32_t pp[4];
    uint32_t c = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      pp[e] = -1;
      kk[e] = 0;
      const uint32_t i = i0 + e;
      if (i < n_in) {
        const uint32_t r = i / (uint32_t)mp.kr, j = i - r * (uint32_t)mp.kr;
        const int64_t src = ((int64_t)r * mp.T + t) * mp.kr + j;
        pp[e] = mp.cand_pos[src];
        if (pp[e] >= 0) kk[e] = score_key(mp.cand_score[src]);
      }
      c += pp[e] >= 0;
    }
    uint32_t total;
    uint32_t at = n_items + block_excl_scan(c, tmp, &total);
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (pp[e] >= 0) {
        gkey[at] = kk[e];
        gpos[at] = pp[e];
        ++at;
      }
    n_items += total;
  }
  __syncthreads();
  const uint32_t k = (uint32_t)mp.k;
  const uint32_t k_eff = n_items < k ? n_items : k;
  if (n_items <= k) {
    for (uint32_t i = threadIdx.x; i < k; i += kTopkThreads) sel[i] = (i < n_items) ? gpos[i] : -1;
  } else {
    // first pass on the items, then the last two and the ordered output
    for (int b = threadIdx.x; b < kTopkBins; b += kTopkThreads) hist[b] = 0;
    __syncthreads();
    for (uint32_t i = threadIdx.x; i < n_items; i += kTopkThreads) atomicAdd(&hist[gkey[i] >> 21], 1u);
    __syncthreads();
    find_threshold_bin<kTopkBins>(hist, k, tmp, res);
    finish_gathered(gkey, gpos, n_items, res[0], res[1], k, sel, hist, tmp, res);
  }
  __syncthreads();
  if (mp.idx_global)
    for (uint32_t i = threadIdx.x; i < k; i += kTopkThreads) mp.idx_global[(int64_t)t * k + i] = sel[i];
  if (mp.idx_local) {
    // this shard's positions, compacted in order (4 consecutive slots per thread per round)
    uint32_t n_loc = 0;
    for (uint32_t r0 = 0; r0 < k; r0 += 4 * kTopkThreads) {
      const uint32_t i0 = r0 + 4 * threadIdx.x;
      int32_t q[4];
      uint32_t c = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        q[e] = (i0 + e < k) ? sel[i0 + e] : -1;
        const bool mine = q[e] >= 0 && q[e] >= mp.shard_lo && q[e] < mp.shard_hi;
        if (!mine) q[e] = -1;
        c += mine;
      }
      uint32_t total;
      uint32_t at = n_loc + block_excl_scan(c, tmp, &total);
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (q[e] >= 0) mp.idx_local[(int64_t)t * k + at++] = (int32_t)(q[e] - mp.shard_lo);
      n_loc += total;
    }
    for (uint32_t i = n_loc + threadIdx.x; i < k; i += kTopkThreads) mp.idx_local[(int64_t)t * k + i] = -1;
    if (threadIdx.x == 0) mp.count_local[t] = (int32_t)n_loc;
  }
  if (threadIdx.x == 0) mp.count[t] = (int32_t)k_eff;
}

}  // namespace dsa
