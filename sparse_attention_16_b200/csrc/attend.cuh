// attend.cuh - absorbed MLA over the selected rows of latent caches (sm_100a).
//
// For query t, head h and layer l (concept page "What to keep", "Sparse
// attention", "Query scaling"):
//   z[h,i] = (q_nope[t,h] . c_{s_i} + q_pe[t,h] . kR_{s_i}) * scale * m[t,h]
//   o[t,h] = sum_i softmax_i(z[h]) c_{s_i}
// Every gathered 1,152-byte row (1,024 on NoPE layers) is read once and used by
// all 64 heads.  One launch covers up to kMaxAttLayers layers that share one
// selection (the concept page's bullet on layers reusing the selection of the
// most recent layer that ran its indexer), so a small decode batch still fills
// the GPU: the work units are (layer, query, split).  RoPE (576-wide rows) and
// NoPE (512-wide) layers may be mixed in one launch.
//
// Heads are the M dimension of both tensor-core products, so each head's
// softmax state lives in one pair of threads.  Tensor memory (512 columns x
// 128 lanes) holds, in lanes 0-15 of every 32-lane quarter, the query Q
// [64 heads x 576] (bf16, two per column) and two logit buffers S [64 heads x
// 64 rows] (f32), and in lanes 16-31 the output O [64 heads x 512] (f32).  That
// leaves shared memory for three 64-row tile buffers (3 x 72 KB), so two tiles
// are in flight while a third is computed on.  Q is gathered into the third
// tile buffer (free until tile 2) and moved to TMEM by the softmax warps.
//
// Work unit = (pair = layer * T + t, split j) = rows [j*R, min(count, (j+1)*R))
// of idx[t].  Per 64-row tile i (buffer i % 3):
//   producer warps 5-7  gather the rows with 16-byte cp.async into a
//                       chunk-major tile: chunk c (64 columns) = 64 rows x 128 B
//                       in the 128-byte-swizzled layout (K-major for the
//                       logits, MN-major for the output product).  The copies
//                       of a row are issued back to back (a warp covers four
//                       whole rows in KCH instructions), so each row reaches
//                       the memory system as one request stream.
//   warp 4              TMEM owner; one thread issues
//                         S = Q . C^T   M = 64 heads, N = 64 rows, K = 576 | 512, Q read from TMEM
//                         O += P . C    M = 64 heads, N = 2 x 256 columns, K = 64 rows
//                       in order of readiness (S of the next tile usually runs
//                       while the softmax of this one does)
//   warps 0-3           softmax: lane L of warp w owns head 16 w + (L & 15) and
//                       rows 32 (L >> 4) .. + 31 of the tile; writes P (bf16,
//                       K-major) to shared memory for the output product.
// The running max is updated lazily: O and the row sums are rescaled only when
// a head's maximum grows by more than 2^8, so p <= 256 and the final
// normalisation uses the same reference for numerator and denominator.
// A single split writes bf16 output directly.  When a query's selection is
// split over 2-8 CTAs, those CTAs form a thread-block cluster: each pushes the
// column slices of its unnormalised O and its per-head (max, sum) into the
// shared memory of the rank that owns those columns, and rank r merges columns
// [r 512 / n, (r + 1) 512 / n) of all heads locally.  Otherwise the splits
// write fp32 partials that a small combine kernel merges.
//
// A selected position is used only if it lies in [0, q_pos[t]] (when q_pos is
// given) and inside the cache; anything else except the -1 padding is skipped
// and flagged (kErrBadIndex).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include <cooperative_groups.h>

#include <climits>
#include <cstddef>

#include "ptx.cuh"

namespace dsa {

constexpr int kHeads = 64;
constexpr int kLatent = 512;
constexpr int kMaxAttLayers = 8;   // layers per attention launch
constexpr int kMaxSplits = 32;     // CTAs per (layer, query)

struct AttCfg {
  static constexpr int KCH_MAX = 9;                      // 64-column chunks of a RoPE row (NoPE: 8)
  static constexpr int ROWS = 64;                        // rows per tile (N of the logit MMA)
  static constexpr int NBUF = 3;                         // tile buffers
  static constexpr int CHUNK_BYTES = ROWS * 128;         // 8 KB: 64 rows x 64 columns
  static constexpr int TILE_BYTES = KCH_MAX * CHUNK_BYTES;   // 72 KB per buffer
  static constexpr int P_BYTES = kHeads * 128;           // P: 64 heads x 64 rows bf16
  static constexpr int DATA_BYTES = NBUF * TILE_BYTES + P_BYTES;
  static constexpr int SCRATCH_BYTES = 1024;
  static constexpr int SMEM_BYTES = DATA_BYTES + SCRATCH_BYTES;
  static constexpr int THREADS = 8 * 32;
  static constexpr int PRODUCERS = 96;                   // warps 5-7
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t Q_COL = 0;                   // lanes 0-15: Q, KCH x 32 columns
  static constexpr uint32_t S_COL = KCH_MAX * 32;        // lanes 0-15: S buffer b at S_COL + 64 b
  static constexpr uint32_t O_LANE = 16;                 // lanes 16-31: O, 512 columns
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(kHeads, ROWS, 0, 0);
  static constexpr uint32_t IDESC_O = idesc_bf16_f32(kHeads, 256, 0, 1);
  static_assert(S_COL + 2 * ROWS <= TMEM_COLS, "Q and two logit buffers must fit in 512 columns");
  static_assert(SMEM_BYTES <= 232448, "shared memory per block");
  static_assert(kHeads == ROWS, "Q is staged as one tile of 64 'rows' (heads)");
};

// One attention layer of a launch.
struct AttLayer {
  const __nv_bfloat16* q_nope;    // [T, 64, 512]
  const __nv_bfloat16* q_pe;      // [T, 64, 64] (RoPE layers) or null
  const float* qmul;              // [T, 64]
  const __nv_bfloat16* cache;     // [n_rows, ld_c] bf16, or FP8 rows of ld_c bytes (attend_kernel<true>)
  __nv_bfloat16* out;             // [T, 64, 512]
  float* lse;                     // [T, 64] or null
  int64_t ld_c;                   // row stride of the cache: elements (bf16) or bytes (FP8 rows)
  int32_t d_rope;                 // 64 (RoPE) or 0 (NoPE)
  int32_t out_f32;                // 1: `out` is fp32 [T, 64, 512] (partial outputs to combine later)
};

// Stores four output values of (t, h) at column c (a multiple of 4) in the layer's output type.
__device__ __forceinline__ void store_out4(const AttLayer& L, int64_t th, int c, float a, float b, float cc, float d) {
  if (L.out_f32) {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(L.out) + th * kLatent + c) = make_float4(a, b, cc, d);
  } else {
    uint2 o;
    o.x = pack_bf16x2(a, b);
    o.y = pack_bf16x2(cc, d);
    *reinterpret_cast<uint2*>(L.out + th * kLatent + c) = o;
  }
}

struct AttendParams {
  AttLayer layer[kMaxAttLayers];
  const int64_t* seq_row_start;   // [B]
  const int32_t* q_seq;           // [T]
  const int32_t* q_pos;           // [T] or null: positions beyond q_pos[t] are rejected
  const int32_t* idx;             // [T, k]
  const int32_t* count;           // [T]
  float* ws_o;                    // [units, n_split, 64, 512] partial numerators (combine path)
  float* ws_ml;                   // [units, n_split, 64, 4] (max in log2 units, sum of the bf16 weights,
                                  //  sum of the fp32 weights, unused)
  int64_t n_rows;
  uint64_t wait_limit_ns;         // limit of the pipeline waits (kWaitLimitNs unless a test lowers it)
  float scale_log2e;              // softmax_scale * log2(e)
  int32_t n_layers;
  int32_t B;
  int32_t T;
  int32_t k;
  int32_t n_split;
  int32_t rows_per_split;         // multiple of 64
  int32_t merge;                  // 1: the n_split CTAs of a (layer, query) are a cluster and merge in DSMEM
  int32_t q_early;                // 1: Q may be read before the dependency wait (no earlier kernel of the
                                  //    stream that can still be running writes Q)
  int32_t stall_tile;             // testing hook: >= 0 -> that tile is never gathered, so its wait runs out
};

struct AttScratch {
  uint64_t q_smem;                // Q has landed in tile buffer 2 (96 producer arrivals)
  uint64_t q_full;                // Q is in tensor memory (128 arrivals)
  uint64_t s_full[2];             // logits of a tile are in S buffer b
  uint64_t s_free[2];             // S buffer b has been read by the softmax (128 arrivals)
  uint64_t p_full;                // P of a tile is in shared memory (128 arrivals)
  uint64_t o_done;                // the output product of a tile has completed
  uint64_t mma_done;
  uint64_t merge_bar;             // cluster merge: the other ranks' blocks have landed (transaction bytes)
  uint64_t full[3];               // tile buffer b loaded
  uint64_t free_[3];              // tile buffer b no longer read
  uint32_t tmem_slot;
  int abort_flag;
  int merge_have_o;               // cluster merge: O of this CTA is complete
};
static_assert(sizeof(AttScratch) <= 1024, "scratch overflow");

__device__ __forceinline__ void unit_rows(const AttendParams& p, int t, int j, int& r_begin,
                                          int& r_end, bool report) {
  int cnt = p.count[t];
  if (cnt < 0 || cnt > p.k) {
    if (report) raise_error(kErrBadIndex);
    cnt = cnt < 0 ? 0 : p.k;
  }
  r_begin = j * p.rows_per_split;
  r_end = min(cnt, r_begin + p.rows_per_split);
  if (r_end < r_begin) r_end = r_begin;
}

// Two E4M3 codes (bits 0-7: the first, bits 8-15: the second) to two floats;
// every E4M3 value is exact in f16 and in f32.
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t codes) {
  float lo, hi;
  asm("{\n\t.reg .b16 c, l, h;\n\t.reg .b32 x;\n\t"
      "cvt.u16.u32 c, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 x, c;\n\t"
      "mov.b32 {l, h}, x;\n\t"
      "cvt.f32.f16 %0, l;\n\t"
      "cvt.f32.f16 %1, h;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(codes));
  return make_float2(lo, hi);
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// tcgen05.st over the 16 lanes [taddr.lane, +16): threads 0-15 write columns
// [col, col + N), threads 16-31 columns [col + N, col + 2N).
__device__ __forceinline__ void tmem_st16x2_32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x32.b32 [%0], 32, "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
      "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]),
      "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]),
      "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st16x2_16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x16.b32 [%0], 16, "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

// D[tmem] (+)= A[tmem] . B[smem]: A read from tensor memory.  A and D must sit
// in the same TMEM lanes (for M = 64: lanes 0-15 of every 32-lane quarter).
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void ld_shared_v4(uint32_t addr, uint32_t& a, uint32_t& b, uint32_t& c,
                                             uint32_t& d) {
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(a), "=r"(b), "=r"(c), "=r"(d) : "r"(addr));
}

// Merge of a (layer, query)'s split partials inside its cluster (n = p.n_split
// CTAs, rank = split), called by every thread of the CTA once all its roles
// are done.  Rank r produces float4 columns [c0(r), c0(r+1)) of every head,
// c0(r) = r 128 / n.  Every CTA holds a receive region of n blocks, one per
// source rank j: [64 heads][nc(r) + 1] float4, the column slice r of O_j
// (unnormalised) and, in the last column, j's per-head (m, l, lx).  A CTA
// writes its own block with plain stores; for every other rank r it stages
// that rank's block in its shared memory (all eight warps read O from tensor
// memory) and moves it with one bulk copy into rank r's region, counted in
// bytes on rank r's barrier.  After the cluster barrier at the start (every
// CTA has left its tile loop, so every tile buffer is free, and every barrier
// is armed with the bytes it will receive) no CTA waits for another except on
// that barrier.  Rank r then merges its slice, consecutive threads on
// consecutive columns:
//   M = max_j m_j,  w_j = 2^(m_j - M),  L = sum_j w_j l_j,
//   o[h, c] = sum_j (w_j / L) O_j[h, c],
//   lse[h] = (M + log2 sum_j w_j lx_j) ln 2 (rank 0)
// (l: sum of the bf16 weights the products used, lx: of the fp32 weights).
__device__ __forceinline__ int merge_c0(int r, int n) { return r * (kLatent / 4) / n; }

__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, int rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
// Bulk copy from this CTA's shared memory to (another CTA's) shared memory in
// the cluster; `bytes` land on the destination CTA's barrier `bar`.  Both
// addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_copy_s2c(uint32_t dst_cluster, uint32_t src, uint32_t bytes,
                                              uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst_cluster),
      "r"(src), "r"(bytes), "r"(bar_cluster)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_group_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void cluster_merge(const AttendParams& p, const AttLayer& L, uint8_t* cs, uint8_t* ps,
                                              AttScratch* sc, uint32_t tmem_base, int t, int rank, bool have_o,
                                              float m_used, float Lsum, float Lx) {
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  const int n = p.n_split;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int half_w = warp >> 2;   // warps w and w + 4 share the lanes of quarter w & 3
  const int hf = lane >> 4;
  const int h = 16 * (warp & 3) + (lane & 15);
  const uint32_t hi_base = tmem_base + ((uint32_t)((warp & 3) * 32 + AttCfg::O_LANE) << 16);
  const bool stats_thread = warp < 4 && hf == 0;   // holds (m, l, lx) of head h
  auto wrow = [&](int r) { return merge_c0(r + 1, n) - merge_c0(r, n) + 1; };
  const int w_own = wrow(rank);
  const int w_max = (kLatent / 4 + n - 1) / n + 1;
  float4* recv = reinterpret_cast<float4*>(cs);                                        // [n sources][64][w_own]
  float4* stage = reinterpret_cast<float4*>(cs + (size_t)n * kHeads * w_max * 16);    // [64][w_max]
  float* wtab = reinterpret_cast<float*>(ps);                                          // [64 heads][8]: w_j / L
  static_assert(kHeads * 8 * 4 <= AttCfg::P_BYTES, "weight table");

  if (tid == 0) {
    mbar_arrive_expect_tx(&sc->merge_bar, (uint32_t)((n - 1) * kHeads * w_own * 16));
    sc->merge_have_o = have_o ? 1 : 0;
  }
  const float4 my_stats = make_float4(have_o ? m_used : -INFINITY, have_o ? Lsum : 0.f, have_o ? Lx : 0.f, 0.f);
  cl.sync();   // every CTA has left its tile loop (receive regions free) and armed its barrier
  const bool ho = sc->merge_have_o != 0;

  // Block for rank r into `dst` ([64][wrow(r)]): O columns [lo, hi) (floats) of
  // head h, read in 64-column tensor-memory blocks (a thread holds columns
  // 64 k + 32 hf + [0, 32) of block k; blocks alternate between the two warps
  // of a quarter), and the stats column.
  auto stage_block = [&](int r, float4* dst) {
    const int W = wrow(r), lo = 4 * merge_c0(r, n), hi = 4 * merge_c0(r + 1, n);
#pragma unroll 1
    for (int k = lo / 64 + half_w; 64 * k < hi; k += 2) {
      uint32_t u[32];
      if (ho) {
        tmem_ld16x2_32(hi_base + 64 * k, u);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) u[c] = 0u;
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int f = 64 * k + 32 * hf + 4 * q;
        if (f >= lo && f < hi)
          dst[h * W + (f - lo) / 4] = make_float4(__uint_as_float(u[4 * q]), __uint_as_float(u[4 * q + 1]),
                                                  __uint_as_float(u[4 * q + 2]), __uint_as_float(u[4 * q + 3]));
      }
    }
    if (stats_thread) dst[h * W + W - 1] = my_stats;
  };
  stage_block(rank, recv + (size_t)rank * kHeads * w_own);   // own block, plain stores
  for (int d = 1; d < n; ++d) {
    const int r = (rank + d) % n;
    if (d >= 2) {   // the staging buffer was read by the previous copy
      if (tid == 0) bulk_wait_group_read<0>();
      __syncthreads();
    }
    stage_block(r, stage);
    fence_proxy_async_smem();   // the staged block is read by the bulk copy (async proxy)
    __syncthreads();
    if (tid == 0) {
      const int W = wrow(r);
      const uint32_t dst = mapa_shared(smem_u32(recv + (size_t)rank * kHeads * W), r);
      bulk_copy_s2c(dst, smem_u32(stage), (uint32_t)(kHeads * W * 16), mapa_shared(smem_u32(&sc->merge_bar), r));
      bulk_commit_group();
    }
  }

  // Every other rank's block has landed (counted on this CTA's barrier).
  mbar_wait(&sc->merge_bar, 0, nullptr, p.wait_limit_ns);
  // Per-head weights (one thread per head), then the slice's float4 columns,
  // consecutive threads on consecutive columns, four outputs per thread at a
  // time with all their loads issued before the arithmetic.
  const int64_t t64 = (int64_t)t * kHeads;
  if (tid < kHeads) {
    const int hh = tid;
    float m[8], l[8], lx[8];
    float M = -INFINITY;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      m[j] = -INFINITY;
      l[j] = lx[j] = 0.f;
      if (j < n) {
        const float4 st = recv[((size_t)j * kHeads + hh) * w_own + w_own - 1];
        m[j] = st.x;
        l[j] = st.y;
        lx[j] = st.z;
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) M = fmaxf(M, m[j]);
    float w[8], Ls = 0.f, Lxs = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      w[j] = (m[j] == -INFINITY) ? 0.f : ex2_approx(m[j] - M);
      Ls += w[j] * l[j];
      Lxs += w[j] * lx[j];
    }
    const float inv = (Ls > 0.f) ? 1.f / Ls : 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) wtab[hh * 8 + j] = w[j] * inv;
    if (rank == 0 && L.lse != nullptr)
      L.lse[t64 + hh] = (Lxs > 0.f) ? (M + lg2_approx(Lxs)) * 0.69314718055994531f : -INFINITY;
  }
  __syncthreads();
  const int c0 = merge_c0(rank, n);
  const int nc = w_own - 1;
  const int total = kHeads * nc;
  const bool pow2 = (nc & (nc - 1)) == 0;
  const int sh = __ffs(nc) - 1;
  constexpr int U = 4;
#pragma unroll 1
  for (int o0 = tid; o0 < total; o0 += U * AttCfg::THREADS) {
    int hh[U], cc[U];
    float4 acc[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int o = min(o0 + u * AttCfg::THREADS, total - 1);
      hh[u] = pow2 ? (o >> sh) : (o / nc);
      cc[u] = o - hh[u] * nc;
      acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j < n) {
        float4 v[U];
        float wj[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          v[u] = recv[((size_t)j * kHeads + hh[u]) * w_own + cc[u]];
          wj[u] = wtab[hh[u] * 8 + j];
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          acc[u].x = fmaf(wj[u], v[u].x, acc[u].x);
          acc[u].y = fmaf(wj[u], v[u].y, acc[u].y);
          acc[u].z = fmaf(wj[u], v[u].z, acc[u].z);
          acc[u].w = fmaf(wj[u], v[u].w, acc[u].w);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (o0 + u * AttCfg::THREADS < total)
        store_out4(L, t64 + hh[u], 4 * (c0 + cc[u]), acc[u].x, acc[u].y, acc[u].z, acc[u].w);
  }
  if (tid == 0) bulk_wait_group_all();   // this CTA's outgoing copies are complete
}

// Q [64 heads x (512 + 64)] of query t into tile buffer 2 in the tile layout
// (heads as rows), by producer warp pw (0-2): 16-byte cp.async copies, then an
// arrival on q_smem once this thread's copies have landed.
template <int KCH>
__device__ __forceinline__ void issue_q(const AttLayer& L, int t, uint32_t cs0, AttScratch* sc, int pw, int lane) {
  using C = AttCfg;
  constexpr int PPR = 8 * KCH;             // 16-byte pieces per row
  constexpr int NQ = C::ROWS / 4;          // row quads per tile
  constexpr int QPW = (NQ + 2) / 3;        // quads per warp, at most
  const char* qn = reinterpret_cast<const char*>(L.q_nope + (int64_t)t * kHeads * kLatent);
  const char* qp = (KCH == 9) ? reinterpret_cast<const char*>(L.q_pe + (int64_t)t * kHeads * 64) : qn;
  const uint32_t qb = cs0 + 2 * C::TILE_BYTES;
#pragma unroll 1
  for (int kq = 0; kq < QPW; ++kq) {
    const int quad = pw + 3 * kq;
    if (quad >= NQ) break;
#pragma unroll
    for (int j = 0; j < KCH; ++j) {
      const int g = 32 * j + lane;
      const int riq = g / PPR;
      const int pr = g - riq * PPR;
      const int h = 4 * quad + riq;
      const uint32_t dst = qb + (pr >> 3) * C::CHUNK_BYTES + h * 128 + (((pr & 7) ^ (h & 7)) << 4);
      const char* src = (pr < 64) ? qn + h * (kLatent * 2) + pr * 16 : qp + h * 128 + (pr - 64) * 16;
      cp_async_16(dst, src, 16u);
    }
  }
  cp_async_arrive_noinc(&sc->q_smem);   // completes once this thread's Q copies have landed
}

// The work of one CTA on one unit; KCH = 64-column chunks per row (9 RoPE, 8 NoPE);
// F8: the cache rows are FP8 (E4M3 codes + block scales) and are widened to bf16
// in shared memory.
template <int KCH, bool F8>
__device__ __forceinline__ void attend_unit(const AttendParams& p, const AttLayer& L, uint8_t* cs, uint8_t* ps,
                                            AttScratch* sc, uint32_t tmem_base, int t, int jsplit,
                                            bool smem_ok) {
  using C = AttCfg;
  volatile int* abort_flag = &sc->abort_flag;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t limit = p.wait_limit_ns;

  int r_begin, r_end;
  unit_rows(p, t, jsplit, r_begin, r_end, threadIdx.x == 0);
  if (!smem_ok) r_end = r_begin;   // nothing is computed; cluster barriers are still met
  const int n_tiles = (r_end - r_begin + C::ROWS - 1) / C::ROWS;
  const int b = p.q_seq[t];
  const bool seq_ok = (b >= 0 && b < p.B);
  const int64_t base = seq_ok ? p.seq_row_start[b] : 0;
  const int32_t qpos = (p.q_pos != nullptr) ? p.q_pos[t] : INT_MAX;

  bool have_o = false;        // softmax threads: O of this unit is complete
  float m_used = -INFINITY;   // reference max of this thread's head, log2 units
  float Lsum = 0.f, Lx = 0.f;

  if (warp >= 5) {
    // ------------------------------------------------------------- producers
    // Warp pw = 0..2 gathers row quads pw, pw + 3, ... of each tile.  The
    // 4 x KCH x 8 sixteen-byte pieces of a quad are KCH warp-wide copies;
    // piece g = 32 j + lane of instruction j is piece g % (8 KCH) of quad row
    // g / (8 KCH).  Lane l holds the index of the warp's row 4 (l >> 2) + (l & 3)
    // (quad pw + 3 (l >> 2)); other lanes read it with a shuffle.
    const int pw = warp - 5;
    constexpr int PPR = 8 * KCH;             // 16-byte pieces per row
    constexpr int NQ = C::ROWS / 4;          // row quads per tile
    constexpr int QPW = (NQ + 2) / 3;        // quads per warp, at most
    static_assert(4 * PPR == 32 * KCH, "a quad is KCH warp-wide copies");
    static_assert(4 * QPW <= 32, "one index per lane");
    if (!seq_ok && threadIdx.x == 160 && n_tiles > 0) raise_error(kErrBadSeq);
    const uint32_t cs0 = smem_u32(cs);
    // Q into tile buffer 2 (already issued before the dependency wait when p.q_early).
    if (n_tiles > 0 && !p.q_early) issue_q<KCH>(L, t, cs0, sc, pw, lane);
    const int my_quad = pw + 3 * (lane >> 2);
    const int my_row = 4 * my_quad + (lane & 3);
    const char* cache_bytes = reinterpret_cast<const char*>(L.cache);
    const int32_t* idx_t = p.idx + (int64_t)t * p.k;
    // The index of this lane's row, loaded one tile ahead so that a global
    // round trip never sits between a buffer becoming free and its copies.
    auto load_idx = [&](int i) -> int32_t {
      const int rr = r_begin + i * C::ROWS + my_row;
      return (i < n_tiles && my_quad < NQ && rr < r_end && seq_ok) ? idx_t[rr] : -1;
    };
    int32_t cur = load_idx(0);
    bool ok = true;
    if constexpr (!F8) {
      for (int i = 0; i < n_tiles; ++i) {
        const int buf = i % C::NBUF;
        if (i >= C::NBUF &&
            !mbar_wait(&sc->free_[buf], (uint32_t)((i / C::NBUF - 1) & 1), abort_flag, limit)) {
          ok = false;
          break;
        }
        // Buffer 2 holds Q until the softmax warps have moved it to TMEM.
        if (i == 2 && !mbar_wait(&sc->q_full, 0, abort_flag, limit)) {
          ok = false;
          break;
        }
        int32_t row = -1;   // row of the cache, or -1: the copy zero-fills
        if (cur >= 0 && cur <= qpos && base + cur < p.n_rows) row = (int32_t)(base + cur);
        else if (cur != -1) raise_error(kErrBadIndex);
        cur = load_idx(i + 1);
        if (i == p.stall_tile) continue;   // testing hook: this tile never arrives
        const uint32_t tb = cs0 + buf * C::TILE_BYTES;
#pragma unroll 1
        for (int kq = 0; kq < QPW; ++kq) {
          const int quad = pw + 3 * kq;
          if (quad >= NQ) break;
#pragma unroll
          for (int j = 0; j < KCH; ++j) {
            const int g = 32 * j + lane;
            const int riq = g / PPR;
            const int pr = g - riq * PPR;
            const int32_t src_row = __shfl_sync(0xffffffffu, row, 4 * kq + riq);
            const int r = 4 * quad + riq;
            const uint32_t dst = tb + (pr >> 3) * C::CHUNK_BYTES + r * 128 + (((pr & 7) ^ (r & 7)) << 4);
            const char* src = src_row >= 0 ? cache_bytes + (int64_t)src_row * L.ld_c * 2 + pr * 16 : cache_bytes;
            cp_async_16(dst, src, src_row >= 0 ? 16u : 0u);
          }
        }
        cp_async_arrive_noinc(&sc->full[buf]);   // lands once this thread's copies so far have
      }
    } else {
      // FP8 rows: the 64 E4M3 codes of a row's 64-column chunk c land in the
      // upper half of that row's 128-byte line of chunk c (pieces 4-7, swizzled
      // like the bf16 pieces) and the row's block scales in registers of the
      // lane that owns the row.  Once a tile's copies have landed, the warp
      // widens every line in place: a lane reads the line's 64 codes, then
      // writes the 64 bf16 values scale * e4m3(code) over the whole line, so the
      // products see the bf16 tile layout.  The copies of tile i are issued
      // before tile i - 1 is widened, so they are in flight meanwhile.
      constexpr int CPR = 4 * KCH;               // 16-byte code pieces per row
      constexpr int NBLK = (KCH == 9) ? 5 : 4;   // fp32 scales per row
      constexpr int SCALE_OFF = 64 * KCH;        // byte offset of the scales in a row
      constexpr int CPI = (4 * CPR + 31) / 32;   // warp-wide copy instructions per quad
      const int rows_w = 4 * ((NQ - pw + 2) / 3);   // rows this warp gathers; local row l = lane l's row
      const int lines_w = rows_w * KCH;
      float sc_next[NBLK], sc_pend[NBLK];
#pragma unroll
      for (int b = 0; b < NBLK; ++b) sc_next[b] = sc_pend[b] = 0.f;
      // Widens the lines of this warp's rows in buffer `buf`; line lane + 32 m
      // is (local row rl, chunk c), rows fastest.
      auto widen = [&](int buf) {
        const uint32_t tb = cs0 + buf * C::TILE_BYTES;
        int rl = lane, c = 0;
        while (rl >= rows_w) {
          rl -= rows_w;
          ++c;
        }
        const int n_it = (lines_w + 31) / 32;
#pragma unroll 1
        for (int it = 0; it < n_it; ++it) {
          const bool active = c < KCH;
          const int blk = (c < 8) ? (c >> 1) : 4;
          float s = 0.f;
#pragma unroll
          for (int b = 0; b < NBLK; ++b) {
            const float v = __shfl_sync(0xffffffffu, sc_pend[b], active ? rl : 0);
            if (b == blk) s = v;
          }
          if (active) {
            const int r = 4 * (pw + 3 * (rl >> 2)) + (rl & 3);
            const uint32_t line = tb + c * C::CHUNK_BYTES + r * 128;
            uint32_t w[16];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj)
              ld_shared_v4(line + (((4 + jj) ^ (r & 7)) << 4), w[4 * jj], w[4 * jj + 1], w[4 * jj + 2], w[4 * jj + 3]);
#pragma unroll
            for (int pp = 0; pp < 8; ++pp) {
              const float2 a = e4m3x2_to_float2(w[2 * pp]);
              const float2 b = e4m3x2_to_float2(w[2 * pp] >> 16);
              const float2 cc = e4m3x2_to_float2(w[2 * pp + 1]);
              const float2 d = e4m3x2_to_float2(w[2 * pp + 1] >> 16);
              st_shared_v4(line + ((pp ^ (r & 7)) << 4), pack_bf16x2(a.x * s, a.y * s), pack_bf16x2(b.x * s, b.y * s),
                           pack_bf16x2(cc.x * s, cc.y * s), pack_bf16x2(d.x * s, d.y * s));
            }
          }
          rl += 32;
          while (rl >= rows_w) {
            rl -= rows_w;
            ++c;
          }
        }
      };
      int pend_buf = -1;   // buffer whose copies are in flight and not yet widened
      for (int i = 0; i < n_tiles; ++i) {
        const int buf = i % C::NBUF;
        if (i >= C::NBUF &&
            !mbar_wait(&sc->free_[buf], (uint32_t)((i / C::NBUF - 1) & 1), abort_flag, limit)) {
          ok = false;
          break;
        }
        if (i == 2 && !mbar_wait(&sc->q_full, 0, abort_flag, limit)) {
          ok = false;
          break;
        }
        int32_t row = -1;
        if (cur >= 0 && cur <= qpos && base + cur < p.n_rows) row = (int32_t)(base + cur);
        else if (cur != -1) raise_error(kErrBadIndex);
        cur = load_idx(i + 1);
        const bool live = i != p.stall_tile;   // testing hook: that tile never arrives
        if (live) {
          const uint32_t tb = cs0 + buf * C::TILE_BYTES;
#pragma unroll 1
          for (int kq = 0; kq < QPW; ++kq) {
            const int quad = pw + 3 * kq;
            if (quad >= NQ) break;
#pragma unroll
            for (int j = 0; j < CPI; ++j) {
              const int g = 32 * j + lane;
              const int riq = min(g / CPR, 3);
              const int32_t src_row = __shfl_sync(0xffffffffu, row, 4 * kq + riq);
              if (g < 4 * CPR) {
                const int pr = g - riq * CPR;
                const int r = 4 * quad + riq;
                const uint32_t dst = tb + (pr >> 2) * C::CHUNK_BYTES + r * 128 + (((4 + (pr & 3)) ^ (r & 7)) << 4);
                const char* src = src_row >= 0 ? cache_bytes + (int64_t)src_row * L.ld_c + pr * 16 : cache_bytes;
                cp_async_16(dst, src, src_row >= 0 ? 16u : 0u);
              }
            }
          }
          if (lane < rows_w && row >= 0) {
            const float* sr = reinterpret_cast<const float*>(cache_bytes + (int64_t)row * L.ld_c + SCALE_OFF);
            const float4 v = __ldg(reinterpret_cast<const float4*>(sr));
            sc_next[0] = v.x;
            sc_next[1] = v.y;
            sc_next[2] = v.z;
            sc_next[3] = v.w;
            if constexpr (NBLK == 5) sc_next[4] = __ldg(sr + 4);
          } else {
#pragma unroll
            for (int b = 0; b < NBLK; ++b) sc_next[b] = 0.f;
          }
        }
        cp_async_commit();
        if (pend_buf >= 0) {
          cp_async_wait_group<1>();   // this lane's copies of the previous tile have landed
          __syncwarp();               // ... and every lane's
          widen(pend_buf);
          fence_proxy_async_smem();   // generic-proxy writes, read by the tensor core
          mbar_arrive(&sc->full[pend_buf]);
        }
        pend_buf = live ? buf : -1;
#pragma unroll
        for (int b = 0; b < NBLK; ++b) sc_pend[b] = sc_next[b];
      }
      if (ok && pend_buf >= 0) {
        cp_async_wait_group<0>();
        __syncwarp();
        widen(pend_buf);
        fence_proxy_async_smem();
        mbar_arrive(&sc->full[pend_buf]);
      }
    }
    if (!ok) *abort_flag = 1;
    cp_async_wait_all();   // nothing may still be landing in shared memory at the barrier below
  } else if (warp == 4) {
    // ------------------------------------------------------------- MMA issuer
    // Issues, in order of readiness, the logit MMAs of the next tile once its
    // rows have landed and the output MMAs of a tile as soon as its softmax
    // weights are in shared memory.  Descriptors are built once; an
    // operand at byte offset d from its base is the base descriptor + (d >> 4)
    // (shared addresses stay below 256 KB, so the start field cannot carry).
    if (lane == 0 && n_tiles > 0) {
      bool ok = mbar_wait(&sc->q_full, 0, abort_flag, limit);
      tc_fence_after();
      const uint64_t s_desc0 = sdesc_sw128(smem_u32(cs), 16, 1024);                 // K-major C
      const uint64_t o_desc0 = sdesc_sw128(smem_u32(cs), C::CHUNK_BYTES, 1024);     // MN-major C
      const uint64_t p_desc = sdesc_sw128(smem_u32(ps), 16, 1024);                  // K-major P
      const uint32_t o_tmem = tmem_base + (C::O_LANE << 16);
      int s_tile = 0;                // next logit product to issue
      bool s_buf_free = true;        // S buffer of s_tile has been read by its previous softmax
      int o_tile = 0;                // next output product to issue
      uint64_t t_idle = 0;
      uint32_t spins = 0;
      while (ok && o_tile < n_tiles) {
        bool progressed = false;
        // Output product of tile o_tile once its P is written.
        if (o_tile < s_tile && mbar_test(&sc->p_full, (uint32_t)(o_tile & 1))) {
          tc_fence_after();
          const int buf = o_tile % C::NBUF;
#pragma unroll
          for (int kk = 0; kk < C::ROWS / 16; ++kk) {
#pragma unroll
            for (int nh = 0; nh < 2; ++nh)
              mma_bf16_ss(o_tmem + nh * 256, p_desc + (uint64_t)((kk * 32) >> 4),
                          o_desc0 + (uint64_t)((buf * C::TILE_BYTES + 4 * nh * C::CHUNK_BYTES + kk * 2048) >> 4),
                          C::IDESC_O, (o_tile > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&sc->free_[buf]);
          mma_commit(&sc->o_done);
          ++o_tile;
          progressed = true;
        }
        // Logits of tile s_tile once its rows have landed and its S buffer has
        // been read by the softmax of tile s_tile - 2: all KCH x 4 MMAs at once.
        if (s_tile < n_tiles) {
          const int sb = s_tile & 1;
          if (!s_buf_free)
            s_buf_free = mbar_test(&sc->s_free[sb], (uint32_t)(((s_tile - 2) >> 1) & 1));
          const int buf = s_tile % C::NBUF;
          if (s_buf_free && mbar_test(&sc->full[buf], (uint32_t)((s_tile / C::NBUF) & 1))) {
            fence_proxy_async_smem();   // cp.async wrote the tile through the generic proxy
            tc_fence_after();
            const uint64_t sbd = s_desc0 + (uint64_t)((buf * C::TILE_BYTES) >> 4);
            const uint32_t d = tmem_base + C::S_COL + 64 * sb;
#pragma unroll 1
            for (int c = 0; c < KCH; ++c) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ts(d, tmem_base + C::Q_COL + 32 * c + 8 * kk,
                            sbd + (uint64_t)((c * C::CHUNK_BYTES + kk * 32) >> 4), C::IDESC_S, (c | kk) ? 1u : 0u);
            }
            mma_commit(&sc->s_full[sb]);
            ++s_tile;
            s_buf_free = s_tile < 2;
            progressed = true;
          }
        }
        if (progressed) {
          spins = 0;
        } else if ((++spins & 255u) == 0) {
          // The idle clock starts at the first check after progress stopped.
          const uint64_t now = global_timer_ns();
          if (*abort_flag) ok = false;
          else if (spins == 256u) t_idle = now;
          else if (now - t_idle > limit) {
            raise_error(kErrTimeout);
            ok = false;
          }
        }
      }
      if (!ok) *abort_flag = 1;
      mma_commit(&sc->mma_done);
      mbar_wait(&sc->mma_done, 0, nullptr);   // every issued MMA has finished (default limit)
    }
  } else {
    // ------------------------------------------------------------- softmax
    // Lane L of warp w owns head h = 16 w + (L & 15) and rows 32 hf .. 32 hf + 31
    // of each tile, hf = L >> 4 (the 16x32bx2 TMEM access pattern).
    const int hf = lane >> 4;
    const int h = 16 * warp + (lane & 15);
    const uint32_t lo_base = tmem_base + ((uint32_t)(warp * 32) << 16);          // Q, S lanes
    const uint32_t hi_base = tmem_base + ((uint32_t)(warp * 32 + C::O_LANE) << 16);  // O lanes
    const float fac = L.qmul[(int64_t)t * kHeads + h] * p.scale_log2e;
    if (n_tiles > 0) {
      // Q[t, h] into TMEM from its staging copy in tile buffer 2: this thread
      // moves elements [128 s + 64 hf, + 64) of the NoPE part (chunk 2 s + hf)
      // and [32 hf, + 32) of the rotary part (chunk 8, pieces 4 hf ..).
      const bool got_q = mbar_wait(&sc->q_smem, 0, abort_flag, limit);
      const uint32_t qrow = smem_u32(cs + 2 * C::TILE_BYTES) + h * 128;
#pragma unroll 1
      for (int s = 0; s < 4; ++s) {
        uint32_t v[32];
        const uint32_t ca = qrow + (2 * s + hf) * C::CHUNK_BYTES;
#pragma unroll
        for (int u = 0; u < 8; ++u) ld_shared_v4(ca + ((u ^ (h & 7)) << 4), v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
        tmem_st16x2_32(lo_base + C::Q_COL + 64 * s, v);
      }
      if (KCH == 9) {
        uint32_t v[16];
        const uint32_t ca = qrow + 8 * C::CHUNK_BYTES;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          ld_shared_v4(ca + (((4 * hf + u) ^ (h & 7)) << 4), v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
        tmem_st16x2_16(lo_base + C::Q_COL + 256, v);
      }
      if (!got_q) *abort_flag = 1;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sc->q_full);
    }
    // Rows that take part: a real position of the sequence inside the unit
    // (entries of -1 inside the counted prefix are skipped).  Lane L tests
    // rows L and 32 + L; a ballot gives every lane the masks of both halves.
    auto valid_mask = [&](int i) -> uint32_t {
      uint32_t m[2];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int rr = r_begin + i * C::ROWS + 32 * half + lane;
        const int32_t sidx = (i < n_tiles && rr < r_end && seq_ok) ? p.idx[(int64_t)t * p.k + rr] : -1;
        m[half] = __ballot_sync(0xffffffffu, sidx >= 0 && sidx <= qpos && base + sidx < p.n_rows);
      }
      return hf ? m[1] : m[0];
    };
    const uint32_t pbase = smem_u32(ps) + h * 128;
    float l_sum = 0.f;          // this thread's share of the row sum of the bf16 weights (normalises o)
    float l_ex = 0.f;           // ... and of the fp32 weights (gives lse)
    uint32_t vm_next = valid_mask(0);
    bool ok = true;
    for (int i = 0; i < n_tiles && ok; ++i) {
      const int sbuf = i & 1;
      const uint32_t vm = vm_next;
      vm_next = valid_mask(i + 1);
      const bool got_s = mbar_wait(&sc->s_full[sbuf], (uint32_t)((i >> 1) & 1), abort_flag, limit);
      if (named_bar_or(1, 128, !got_s)) { ok = false; break; }   // leave together
      tc_fence_after();
      uint32_t v[32];
      tmem_ld16x2_32(lo_base + C::S_COL + 64 * sbuf, v);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&sc->s_free[sbuf]);
      float z[32];
      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        z[c] = ((vm >> c) & 1u) ? __uint_as_float(v[c]) * fac : -INFINITY;
        mt = fmaxf(mt, z[c]);
      }
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
      // Lazy reference: move it only when the tile max exceeds it by more than 2^8.
      float alpha = 1.f;
      bool resc = false;
      if (mt > m_used + 8.f) {
        alpha = (m_used == -INFINITY) ? 0.f : ex2_approx(m_used - mt);
        resc = (m_used != -INFINITY);
        m_used = mt;
        l_sum *= alpha;
        l_ex *= alpha;
      }
      uint32_t pk[16];
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        const float p0 = ((vm >> c) & 1u) ? ex2_approx(z[c] - m_used) : 0.f;
        const float p1 = ((vm >> (c + 1)) & 1u) ? ex2_approx(z[c + 1] - m_used) : 0.f;
        l_ex += p0 + p1;
        pk[c >> 1] = pack_bf16x2(p0, p1);
      }
      if (i > 0) {
        // O(i-1) finished: P of the previous tile is no longer read, and O may
        // be rescaled in place.
        const bool got_o = mbar_wait(&sc->o_done, (uint32_t)((i - 1) & 1), abort_flag, limit);
        if (named_bar_or(1, 128, !got_o)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, resc)) {
#pragma unroll 1
          for (int cb = 0; cb < kLatent; cb += 64) {
            uint32_t u[32];
            tmem_ld16x2_32(hi_base + cb, u);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) u[c] = __float_as_uint(__uint_as_float(u[c]) * alpha);
            tmem_st16x2_32(hi_base + cb, u);
          }
          tmem_wait_st();
        }
      }
      // P row h, rows 32 hf .. + 31 of the tile = 16-byte pieces 4 hf .. 4 hf + 3,
      // and the row sum of the rounded weights the tensor core multiplies.
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const int q = 4 * hf + q4;
        st_shared_v4(pbase + ((q ^ (h & 7)) << 4), pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
      }
#pragma unroll
      for (int c = 0; c < 16; ++c)
        l_sum += __uint_as_float(pk[c] << 16) + __uint_as_float(pk[c] & 0xFFFF0000u);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&sc->p_full);
    }
    if (!ok) *abort_flag = 1;
    have_o = ok && n_tiles > 0;
    if (have_o) {
      const bool got_o = mbar_wait(&sc->o_done, (uint32_t)((n_tiles - 1) & 1), abort_flag, limit);
      have_o = !named_bar_or(1, 128, !got_o);
    }
    Lsum = l_sum + __shfl_xor_sync(0xffffffffu, l_sum, 16);
    Lx = l_ex + __shfl_xor_sync(0xffffffffu, l_ex, 16);
    if (threadIdx.x == 0) sc->merge_have_o = have_o ? 1 : 0;   // for the warps that did not compute it
  }

  // Every role is done: the producers' copies have landed (cp.async.wait_all),
  // every MMA has completed (mma_done), so the tile buffers may be reused for
  // staging and O may be read from TMEM.
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t hi_base = tmem_base + ((uint32_t)((warp & 3) * 32 + C::O_LANE) << 16);
  if (p.merge) {
    cluster_merge(p, L, cs, ps, sc, tmem_base, t, jsplit, have_o, m_used, Lsum, Lx);
    return;
  }
  const int64_t unit = blockIdx.x;   // (pair, split)
  if (p.n_split > 1) {
    // ---- fp32 partial of this split, [64 heads][512] in the workspace.  All
    // eight warps stage O in shared memory (rows padded by 16 bytes, so the
    // 16 heads a half-warp writes at once fall in different banks; warps w and
    // w + 4 read the same TMEM lanes and take alternate 64-column blocks), then
    // the CTA copies the rows out with whole-line stores.
    constexpr int SROW = kLatent + 4;
    float* stg = reinterpret_cast<float*>(cs);
    const bool ho = sc->merge_have_o != 0;
    const int hf = lane >> 4;
    const int h = 16 * (warp & 3) + (lane & 15);
#pragma unroll 1
    for (int cb = 64 * (warp >> 2); cb < kLatent; cb += 128) {
      uint32_t u[32];
      if (ho) {
        tmem_ld16x2_32(hi_base + cb, u);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) u[c] = 0u;
      }
      float4* dst = reinterpret_cast<float4*>(stg + h * SROW + cb + 32 * hf);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        dst[q] = make_float4(__uint_as_float(u[4 * q]), __uint_as_float(u[4 * q + 1]), __uint_as_float(u[4 * q + 2]),
                             __uint_as_float(u[4 * q + 3]));
    }
    if (warp < 4 && hf == 0) {
      float* ml = p.ws_ml + (unit * kHeads + h) * 4;
      ml[0] = have_o ? m_used : -INFINITY;
      ml[1] = have_o ? Lsum : 0.f;
      ml[2] = have_o ? Lx : 0.f;
    }
    __syncthreads();
    float4* wo = reinterpret_cast<float4*>(p.ws_o + unit * kHeads * kLatent);
#pragma unroll 4
    for (int i = threadIdx.x; i < kHeads * kLatent / 4; i += C::THREADS) {
      const int hh = i / (kLatent / 4), c4 = i % (kLatent / 4);
      wo[i] = reinterpret_cast<const float4*>(stg + hh * SROW)[c4];
    }
    return;
  }
  if (warp >= 4) return;

  // ---- epilogue (softmax warps): normalised output
  const int hf = lane >> 4;
  const int h = 16 * warp + (lane & 15);
  auto read_o = [&](int cb, uint32_t (&u)[32]) {
    if (have_o) {
      tmem_ld16x2_32(hi_base + cb, u);
      tmem_wait_ld();
    } else {
#pragma unroll
      for (int c = 0; c < 32; ++c) u[c] = 0u;
    }
  };
  if (p.n_split == 1) {
    const float inv = (have_o && Lsum > 0.f) ? 1.f / Lsum : 0.f;
    const int64_t th = (int64_t)t * kHeads + h;
#pragma unroll 1
    for (int cb = 0; cb < kLatent; cb += 64) {
      uint32_t u[32];
      read_o(cb, u);
      if (L.out_f32) {
        float4* o_t = reinterpret_cast<float4*>(reinterpret_cast<float*>(L.out) + th * kLatent + 32 * hf + cb);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          o_t[q] = make_float4(__uint_as_float(u[4 * q]) * inv, __uint_as_float(u[4 * q + 1]) * inv,
                               __uint_as_float(u[4 * q + 2]) * inv, __uint_as_float(u[4 * q + 3]) * inv);
      } else {
        uint4* o_t = reinterpret_cast<uint4*>(L.out + th * kLatent + 32 * hf);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(u[8 * q]) * inv, __uint_as_float(u[8 * q + 1]) * inv);
          w.y = pack_bf16x2(__uint_as_float(u[8 * q + 2]) * inv, __uint_as_float(u[8 * q + 3]) * inv);
          w.z = pack_bf16x2(__uint_as_float(u[8 * q + 4]) * inv, __uint_as_float(u[8 * q + 5]) * inv);
          w.w = pack_bf16x2(__uint_as_float(u[8 * q + 6]) * inv, __uint_as_float(u[8 * q + 7]) * inv);
          o_t[cb / 8 + q] = w;
        }
      }
    }
    if (L.lse != nullptr && hf == 0)
      L.lse[(int64_t)t * kHeads + h] =
          (have_o && Lx > 0.f) ? (m_used + lg2_approx(Lx)) * 0.69314718055994531f : -INFINITY;
  }
}

// F8: every layer of the launch keeps its latent cache in FP8 rows.
template <bool F8>
__global__ void __launch_bounds__(AttCfg::THREADS, 1)
    attend_kernel(const __grid_constant__ AttendParams p) {
  using C = AttCfg;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // The swizzled layouts need 1024-byte alignment; dynamic shared memory starts
  // there when the kernel has no static shared memory.
  const bool smem_ok = (smem_u32(smem_raw) & 1023u) == 0;
  if (!smem_ok && threadIdx.x == 0) raise_error(kErrBadSeq);
  uint8_t* cs = smem_raw;                               // three tile buffers
  uint8_t* ps = cs + C::NBUF * C::TILE_BYTES;
  AttScratch* sc = reinterpret_cast<AttScratch*>(ps + C::P_BYTES);

  const int warp = threadIdx.x >> 5;
  const int pair = blockIdx.x / p.n_split;
  const int jsplit = blockIdx.x % p.n_split;
  const int lyr = pair / p.T;
  const int t = pair - lyr * p.T;
  const AttLayer& L = p.layer[lyr];

  if (threadIdx.x == 0) {
    mbar_init(&sc->q_smem, C::PRODUCERS);
    mbar_init(&sc->q_full, 128);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sc->s_full[b], 1);
      mbar_init(&sc->s_free[b], 128);
    }
    mbar_init(&sc->p_full, 128);
    mbar_init(&sc->o_done, 1);
    mbar_init(&sc->mma_done, 1);
    mbar_init(&sc->merge_bar, 1);
    for (int b = 0; b < C::NBUF; ++b) {
      mbar_init(&sc->full[b], C::PRODUCERS);
      mbar_init(&sc->free_[b], 1);
    }
    sc->abort_flag = 0;
    fence_mbar_init();
  }
  if (p.q_early) {
    // Q is not written by the kernels this launch may overlap: its copies start
    // now, while the previous kernel finishes.
    __syncthreads();   // the barriers are initialised
    if (warp >= 5 && smem_ok) {
      if (L.d_rope == 64) issue_q<9>(L, t, smem_u32(cs), sc, warp - 5, threadIdx.x & 31);
      else issue_q<8>(L, t, smem_u32(cs), sc, warp - 5, threadIdx.x & 31);
    }
  }
  // Tensor memory before the dependency wait (a launch as a programmatic
  // dependent sets up while the previous kernel finishes; only this library's
  // attention uses tensor memory, and its blocks never share an SM).
  if (warp == 4) {
    tmem_alloc(&sc->tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  griddep_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = sc->tmem_slot;

  if (L.d_rope == 64) attend_unit<9, F8>(p, L, cs, ps, sc, tmem_base, t, jsplit, smem_ok);
  else attend_unit<8, F8>(p, L, cs, ps, sc, tmem_base, t, jsplit, smem_ok);

  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// Merges the split partials of each (layer, query, head): o = sum_j 2^(m_j - M) O_j / L,
// L = sum_j 2^(m_j - M) l_j, lse = (M + log2 sum_j 2^(m_j - M) lx_j) ln 2.  One block per
// (pair, head); each of the 128 threads owns 4 latent columns.
__global__ void __launch_bounds__(128) attend_combine_kernel(const __grid_constant__ AttendParams p) {
  griddep_wait();
  const int pair = blockIdx.x / kHeads;
  const int h = blockIdx.x % kHeads;
  const int lyr = pair / p.T;
  const int t = pair - lyr * p.T;
  const AttLayer& L = p.layer[lyr];
  const int ns = p.n_split;
  // The first PF partials of this thread's 4 columns are loaded before the
  // weights are known, so their L2 round trips overlap each other and the
  // statistics' round trip.  Every warp computes the weights itself (lane j:
  // split j), so no barrier separates them from the sums.
  constexpr int PF = 8;
  static_assert(kMaxSplits <= 32, "one split per lane");
  const int d = threadIdx.x * 4;
  const float* po = p.ws_o + ((int64_t)pair * ns * kHeads + h) * kLatent + d;   // split j at + j 64 512
  float4 pre[PF];
#pragma unroll
  for (int j = 0; j < PF; ++j)
    pre[j] = (j < ns) ? *reinterpret_cast<const float4*>(po + (int64_t)j * kHeads * kLatent)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
  const int lane = threadIdx.x & 31;
  const int64_t u = (int64_t)pair * ns + lane;
  const float m = (lane < ns) ? p.ws_ml[(u * kHeads + h) * 4] : -INFINITY;
  const float l = (lane < ns) ? p.ws_ml[(u * kHeads + h) * 4 + 1] : 0.f;
  const float lx = (lane < ns) ? p.ws_ml[(u * kHeads + h) * 4 + 2] : 0.f;
  float M = m;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float sc = (m == -INFINITY) ? 0.f : ex2_approx(m - M);
  float Ls = sc * l, Lx = sc * lx;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    Ls += __shfl_xor_sync(0xffffffffu, Ls, o);
    Lx += __shfl_xor_sync(0xffffffffu, Lx, o);
  }
  const float w_lane = (Ls > 0.f) ? sc / Ls : 0.f;   // weight of split `lane`
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int j = 0; j < PF; ++j) {
    const float wj = __shfl_sync(0xffffffffu, w_lane, j);   // 0 for j >= ns
    acc.x = fmaf(wj, pre[j].x, acc.x);
    acc.y = fmaf(wj, pre[j].y, acc.y);
    acc.z = fmaf(wj, pre[j].z, acc.z);
    acc.w = fmaf(wj, pre[j].w, acc.w);
  }
  for (int j = PF; j < ns; ++j) {
    const float wj = __shfl_sync(0xffffffffu, w_lane, j);
    const float4 o4 = *reinterpret_cast<const float4*>(po + (int64_t)j * kHeads * kLatent);
    acc.x = fmaf(wj, o4.x, acc.x);
    acc.y = fmaf(wj, o4.y, acc.y);
    acc.z = fmaf(wj, o4.z, acc.z);
    acc.w = fmaf(wj, o4.w, acc.w);
  }
  store_out4(L, (int64_t)t * kHeads + h, d, acc.x, acc.y, acc.z, acc.w);
  if (threadIdx.x == 0 && L.lse != nullptr)
    L.lse[(int64_t)t * kHeads + h] = (Lx > 0.f) ? (M + lg2_approx(Lx)) * 0.69314718055994531f : -INFINITY;
}

// Context-parallel output combine (report's serving section): R ranks each
// attended over their own part of one selection, giving o_r (normalised over
// that part, fp32) and lse_r.  Over the whole selection
//   lse = log sum_r exp(lse_r),  o = sum_r exp(lse_r - lse) o_r
// (a part with lse_r = -inf contributes nothing; all parts empty: o = 0,
// lse = -inf).  One block per (query, head); 128 threads x 4 columns.
struct LseCombineParams {
  const float* o_parts;       // [R, T, 64, 512]
  const float* lse_parts;     // [R, T, 64]
  __nv_bfloat16* out;         // [T, 64, 512]
  float* lse;                 // [T, 64] or null
  int32_t R, T;
};

__global__ void __launch_bounds__(128) lse_combine_kernel(const LseCombineParams cp) {
  griddep_wait();
  const int t = blockIdx.x / kHeads;
  const int h = blockIdx.x % kHeads;
  __shared__ float wr[64];
  __shared__ float stat;
  if (threadIdx.x < 32) {
    float M = -INFINITY;
    for (int r = threadIdx.x; r < cp.R; r += 32) M = fmaxf(M, cp.lse_parts[((int64_t)r * cp.T + t) * kHeads + h]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float S = 0.f;
    for (int r = threadIdx.x; r < cp.R; r += 32) {
      const float l = cp.lse_parts[((int64_t)r * cp.T + t) * kHeads + h];
      const float w = (l == -INFINITY) ? 0.f : ex2_approx((l - M) * 1.4426950408889634f);
      wr[r] = w;
      S += w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
    __syncwarp();
    for (int r = threadIdx.x; r < cp.R; r += 32) wr[r] = (S > 0.f) ? wr[r] / S : 0.f;
    if (threadIdx.x == 0) stat = (S > 0.f) ? M + lg2_approx(S) * 0.69314718055994531f : -INFINITY;
  }
  __syncthreads();
  const int d = threadIdx.x * 4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int r = 0; r < cp.R; ++r) {
    const float w = wr[r];
    if (w == 0.f) continue;
    const float4 o4 = *reinterpret_cast<const float4*>(cp.o_parts + (((int64_t)r * cp.T + t) * kHeads + h) * kLatent + d);
    acc.x = fmaf(w, o4.x, acc.x);
    acc.y = fmaf(w, o4.y, acc.y);
    acc.z = fmaf(w, o4.z, acc.z);
    acc.w = fmaf(w, o4.w, acc.w);
  }
  uint2 o;
  o.x = pack_bf16x2(acc.x, acc.y);
  o.y = pack_bf16x2(acc.z, acc.w);
  *reinterpret_cast<uint2*>(cp.out + ((int64_t)t * kHeads + h) * kLatent + d) = o;
  if (threadIdx.x == 0 && cp.lse != nullptr) cp.lse[(int64_t)t * kHeads + h] = stat;
}

}  // namespace dsa
