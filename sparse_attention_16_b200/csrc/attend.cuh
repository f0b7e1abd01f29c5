// attend.cuh - absorbed MLA over the selected rows of a latent cache (sm_100a).
//
// For query t and head h (concept page "What to keep", "Sparse attention",
// "Query scaling"):
//   z[h,i] = (q_nope[t,h] . c_{s_i} + q_pe[t,h] . kR_{s_i}) * scale * m[t,h]
//   o[t,h] = sum_i softmax_i(z[h]) c_{s_i}
// Every gathered 1,152-byte row (1,024 on NoPE layers) is read once and used by
// all 64 heads.
//
// Work unit = (query t, split j): rows [j*R, min(count, (j+1)*R)) of idx[t], in
// tiles of 128 rows.  Per tile:
//   producer warps 5-7   gather the 128 rows with 16-byte cp.async into a
//                        chunk-major tile: chunk c (64 columns) holds 128 rows x
//                        128 B in the 128-byte-swizzled layout the tensor core
//                        reads (K-major for the logits, MN-major for the output)
//   warp 4               TMEM owner; one thread issues
//                          S^T[128 rows x 64 heads] = C[rows, 576] . Q^T   (K-major A, B)
//                          O^T[512 x 64] += C^T[512, rows] . P^T[rows, 64] (MN-major A, B)
//   warps 0-3            softmax: TMEM lane r = row r holds that row's 64 head
//                        logits; per-head maxima come from warp max-reductions;
//                        exp2 with scale*m*log2(e) folded in; P^T (bf16) is
//                        written to shared memory for the second product.
// The running max is updated lazily: O and the row sums are rescaled only when
// a head's maximum grows by more than 2^8, so p <= 256 and the final
// normalisation uses the same reference for numerator and denominator.
// The rotary chunk of the tile is no longer needed once S^T is done, so P^T is
// written over it on RoPE layers.  Splits write fp32 partials (o, max, sum)
// that a small combine kernel merges; a single split writes bf16 output
// directly.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include <cstddef>

#include "ptx.cuh"

namespace dsa {

constexpr int kHeads = 64;
constexpr int kLatent = 512;

template <int DR>
struct AttCfg {
  static constexpr int KCH = (kLatent + DR) / 64;        // 64-column chunks: 9 or 8
  static constexpr int ROWS = 64;                        // rows per tile (M of the logit MMA)
  static constexpr int CHUNK_BYTES = ROWS * 128;         // 8 KB: 64 rows x 64 columns
  static constexpr int TILE_BYTES = KCH * CHUNK_BYTES;   // 72 KB (RoPE) / 64 KB (NoPE)
  static constexpr int QCHUNK_BYTES = kHeads * 128;      // 8 KB
  static constexpr int Q_BYTES = KCH * QCHUNK_BYTES;
  static constexpr int P_BYTES = ROWS * 128;             // P^T: 64 rows x 64 heads bf16
  static constexpr int DATA_BYTES = Q_BYTES + 2 * TILE_BYTES + P_BYTES;
  static constexpr int SCRATCH_BYTES = 2048;
  static constexpr int SMEM_BYTES = DATA_BYTES + SCRATCH_BYTES;
  static constexpr int THREADS = 8 * 32;
  static constexpr int PRODUCERS = 96;                   // warps 5-7
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t S_COL = 0;                   // S^T of tile j in TMEM lane half (j & 1)
  static constexpr uint32_t O_COL = 128;                 // O^T: 4 blocks x 64 columns
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(64, kHeads, 0, 0);
  static constexpr uint32_t IDESC_O = idesc_bf16_f32(128, kHeads, 1, 1);
};

struct AttendParams {
  const __nv_bfloat16* cache;     // [n_rows, ld_c]
  const float* qmul;              // [T, 64]
  const int64_t* seq_row_start;   // [B]
  const int32_t* q_seq;           // [T]
  const int32_t* idx;             // [T, k]
  const int32_t* count;           // [T]
  __nv_bfloat16* out;             // [T, 64, 512]
  float* lse;                     // [T, 64] or null
  float* ws_o;                    // [T, n_split, 64, 512] partial numerators (n_split > 1)
  float* ws_ml;                   // [T, n_split, 64, 2] (max in log2 units, sum)
  int64_t ld_c;
  int64_t n_rows;
  float scale_log2e;              // softmax_scale * log2(e)
  int32_t B;
  int32_t T;
  int32_t k;
  int32_t n_split;
  int32_t rows_per_split;         // multiple of 64
};

struct AttScratch {
  uint64_t q_full;
  uint64_t s_full[2];             // S^T of a tile is in TMEM (per lane half)
  uint64_t p_full;                // P^T of a tile is in shared memory
  uint64_t o_done;                // the output product of a tile has completed
  uint64_t mma_done;
  uint64_t full[2][9];            // chunk c of tile buffer b loaded
  uint64_t free_[2];              // tile buffer no longer read (per buffer)
  uint32_t tmem_slot;
  int abort_flag;
  alignas(16) float fac[64];      // scale * m[t,h] * log2(e)   (read as float4)
  alignas(16) float m_used[64];   // running (lazy) max per head, log2 units (float4)
  alignas(16) float alpha[64];    // rescale factor of the current tile
  alignas(16) int32_t red[4][64]; // per-warp head maxima (order-mapped ints) / sums
};
static_assert(sizeof(AttScratch) <= 2048, "scratch overflow");
static_assert(offsetof(AttScratch, fac) % 16 == 0 && offsetof(AttScratch, m_used) % 16 == 0,
              "vector-read arrays must be 16-byte aligned");

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

// Work unit = (query t, split j) = rows [j*R, min(count, (j+1)*R)) of idx[t], in
// tiles of 64 rows held in two buffers:
//   producers (warps 5-7) gather tile j into buffer j & 1 with 16-byte cp.async,
//     in the 128-byte-swizzled chunk-major layout (chunk = 64 rows x 64 columns)
//   the MMA thread (warp 4) issues, per tile,
//     S^T[64 rows x 64 heads] = C . Q^T     M = 64, into TMEM lane half (j & 1)
//     O^T[512 x 64] += C^T . P^T            M = 128 latent columns x 4, K = 64 rows
//     and issues S(j+1) before O(j), so the logits of the next tile are ready
//     while the softmax of this one runs and the tile after that is loading
//   softmax warps 0-3: lane L of warp w holds row 16 w + (L & 15) of the tile
//     whose lane half is L >> 4.
template <int DR>
__global__ void __launch_bounds__(AttCfg<DR>::THREADS, 1)
    attend_kernel(const __grid_constant__ CUtensorMap qn_map, const __grid_constant__ CUtensorMap qp_map,
                  const AttendParams p) {
  using C = AttCfg<DR>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // The swizzled layouts need 1024-byte alignment; dynamic shared memory starts
  // there when the kernel has no static shared memory.
  if ((smem_u32(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) raise_error(kErrBadSeq);
    return;
  }
  uint8_t* qs = smem_raw;
  uint8_t* cs = smem_raw + C::Q_BYTES;                  // two tile buffers
  uint8_t* ps = cs + 2 * C::TILE_BYTES;
  AttScratch* sc = reinterpret_cast<AttScratch*>(ps + C::P_BYTES);
  volatile int* abort_flag = &sc->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x / p.n_split;
  const int jsplit = blockIdx.x % p.n_split;

  if (threadIdx.x == 0) {
    mbar_init(&sc->q_full, 1);
    mbar_init(&sc->s_full[0], 1);
    mbar_init(&sc->s_full[1], 1);
    mbar_init(&sc->p_full, 128);
    mbar_init(&sc->o_done, 1);
    mbar_init(&sc->mma_done, 1);
    for (int b = 0; b < 2; ++b) {
      for (int c = 0; c < C::KCH; ++c) mbar_init(&sc->full[b][c], C::PRODUCERS);
      mbar_init(&sc->free_[b], 1);
    }
    sc->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(&sc->tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = sc->tmem_slot;

  int r_begin, r_end;
  unit_rows(p, t, jsplit, r_begin, r_end, threadIdx.x == 0);
  const int n_tiles = (r_end - r_begin + C::ROWS - 1) / C::ROWS;

  if (warp >= 5) {
    // ------------------------------------------------------------- producers
    // Thread pt copies 16-byte piece (lane & 7) of rows prow, prow + 12, ... of
    // every chunk.  Destination offsets (with the 128-byte swizzle) depend only
    // on the row; source row addresses are computed once per tile.
    const int pt = threadIdx.x - 160;  // 0..95
    if (pt == 0 && n_tiles > 0) {
      prefetch_tmap(&qn_map);
      mbar_arrive_expect_tx(&sc->q_full, C::Q_BYTES);
      for (int c = 0; c < 8; ++c)
        tma_load_2d(qs + c * C::QCHUNK_BYTES, &qn_map, c * 64, t * kHeads, &sc->q_full);
      if (DR == 64) {
        prefetch_tmap(&qp_map);
        tma_load_2d(qs + 8 * C::QCHUNK_BYTES, &qp_map, 0, t * kHeads, &sc->q_full);
      }
    }
    const int b = p.q_seq[t];
    const bool seq_ok = (b >= 0 && b < p.B);
    if (!seq_ok && pt == 0 && n_tiles > 0) raise_error(kErrBadSeq);
    const int64_t base = seq_ok ? p.seq_row_start[b] : 0;
    const int prow = 4 * (warp - 5) + (lane >> 3);  // rows prow + 12 jj
    const int piece = lane & 7;
    constexpr int RPT = (C::ROWS + 11) / 12;          // 6 rows per thread at most
    const uint32_t cs0 = smem_u32(cs);
    uint32_t dst[RPT];
#pragma unroll
    for (int jj = 0; jj < RPT; ++jj) {
      const int r = prow + 12 * jj;
      dst[jj] = r * 128 + ((piece ^ (r & 7)) << 4);
    }
    const char* cache_bytes = reinterpret_cast<const char*>(p.cache);
    const int32_t* idx_t = p.idx + (int64_t)t * p.k;
    // Index loads are software-pipelined one tile ahead so that a global
    // round trip never sits between a buffer becoming free and its copies.
    // Rows of the tile three ahead are bulk-prefetched into L2, so their
    // cp.async copies later hit L2.
    constexpr int kPrefetchTiles = 3;
    auto load_rows = [&](int i, int32_t (&out)[RPT]) {
      const int r0 = r_begin + i * C::ROWS;
#pragma unroll
      for (int jj = 0; jj < RPT; ++jj) {
        const int r = prow + 12 * jj;
        out[jj] = (i < n_tiles && r < C::ROWS && r0 + r < r_end && seq_ok) ? idx_t[r0 + r] : -1;
      }
    };
    auto load_pf = [&](int i) -> int32_t {
      const int rr = r_begin + i * C::ROWS + pt;
      return (i < n_tiles && pt < C::ROWS && rr < r_end && seq_ok) ? idx_t[rr] : -1;
    };
    auto prefetch_row = [&](int32_t sidx) {
      if (sidx >= 0 && base + sidx < p.n_rows)
        prefetch_l2_bulk(cache_bytes + (base + sidx) * p.ld_c * 2, (kLatent + DR) * 2);
    };
    for (int i = 0; i < kPrefetchTiles && i < n_tiles; ++i) prefetch_row(load_pf(i));
    int32_t cur[RPT];
    load_rows(0, cur);
    int32_t pf_next = load_pf(kPrefetchTiles);
    bool ok = true;
    for (int i = 0; i < n_tiles; ++i) {
      const int buf = i & 1;
      prefetch_row(pf_next);
      pf_next = load_pf(i + kPrefetchTiles + 1);
      if (i >= 2 && !mbar_wait(&sc->free_[buf], (uint32_t)(((i >> 1) - 1) & 1), abort_flag)) {
        ok = false;
        break;
      }
      const char* src[RPT];
      uint32_t nbytes[RPT];
#pragma unroll
      for (int jj = 0; jj < RPT; ++jj) {
        const int32_t sidx = cur[jj];
        src[jj] = cache_bytes;
        nbytes[jj] = 0;
        if (sidx >= 0 && base + sidx < p.n_rows) {
          src[jj] = cache_bytes + ((base + sidx) * p.ld_c) * 2 + piece * 16;
          nbytes[jj] = 16;
        } else if (sidx != -1 && piece == 0) {
          raise_error(kErrBadIndex);
        }
      }
      load_rows(i + 1, cur);   // next tile's indices, in flight while this tile is copied
      const uint32_t tb = cs0 + buf * C::TILE_BYTES;
#pragma unroll 1
      for (int c = 0; c < C::KCH; ++c) {
#pragma unroll
        for (int jj = 0; jj < RPT; ++jj) {
          if (prow + 12 * jj < C::ROWS)
            cp_async_16(tb + c * C::CHUNK_BYTES + dst[jj], src[jj] + (nbytes[jj] ? c * 128 : 0), nbytes[jj]);
        }
        cp_async_arrive_noinc(&sc->full[buf][c]);   // lands once this thread's copies so far have
      }
    }
    if (!ok) *abort_flag = 1;
    cp_async_wait_all();   // nothing may still be landing in shared memory at exit
    if (pt == 0 && n_tiles > 0) mbar_wait(&sc->q_full, 0, nullptr);
  } else if (warp == 4) {
    // ------------------------------------------------------------- MMA issuer
    // Issues, in order of readiness, the logit MMAs of the next tile chunk by
    // chunk as its rows land, and the output MMAs of a tile as soon as its
    // softmax weights are in shared memory.  Descriptors are built once; an
    // operand at byte offset d from its base is the base descriptor + (d >> 4)
    // (shared addresses stay below 256 KB, so the start field cannot carry).
    if (lane == 0 && n_tiles > 0) {
      bool ok = mbar_wait(&sc->q_full, 0, abort_flag);
      const uint64_t q_desc = sdesc_sw128(smem_u32(qs), 16, 1024);
      const uint64_t s_desc0 = sdesc_sw128(smem_u32(cs), 16, 1024);                        // K-major C
      const uint64_t o_desc0 = sdesc_sw128(smem_u32(cs), C::CHUNK_BYTES, 1024);            // MN-major C^T
      const uint64_t p_desc = sdesc_sw128(smem_u32(ps), C::CHUNK_BYTES, 1024);             // MN-major P^T
      int s_tile = 0, s_chunk = 0;   // next logit chunk to issue
      int o_tile = 0;                // next output product to issue
      uint64_t t_idle = global_timer_ns();
      uint32_t spins = 0;
      while (ok && o_tile < n_tiles) {
        bool progressed = false;
        // Output product of tile o_tile once its P^T is written.
        if (o_tile < s_tile && mbar_test(&sc->p_full, (uint32_t)(o_tile & 1))) {
          tc_fence_after();
          fence_proxy_async_smem();     // P^T was written with st.shared
          const uint64_t ob = o_desc0 + (uint64_t)(((o_tile & 1) * C::TILE_BYTES) >> 4);
#pragma unroll
          for (int blk = 0; blk < 4; ++blk) {
#pragma unroll
            for (int kk = 0; kk < C::ROWS / 16; ++kk)
              mma_bf16_ss(tmem_base + C::O_COL + blk * 64,
                          ob + (uint64_t)((2 * blk * C::CHUNK_BYTES + kk * 2048) >> 4),
                          p_desc + (uint64_t)((kk * 2048) >> 4), C::IDESC_O, (o_tile > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&sc->free_[o_tile & 1]);
          mma_commit(&sc->o_done);
          ++o_tile;
          progressed = true;
        }
        // Logits of tile s_tile, one chunk at a time.  Its TMEM lane half was
        // last read by the softmax of tile s_tile - 2, whose weights the
        // output product o_tile > s_tile - 2 has already consumed.
        if (s_tile < n_tiles && o_tile >= s_tile - 1) {
          const int buf = s_tile & 1;
          if (mbar_test(&sc->full[buf][s_chunk], (uint32_t)((s_tile >> 1) & 1))) {
            fence_proxy_async_smem();   // cp.async wrote through the generic proxy
            tc_fence_after();
            const uint64_t sb = s_desc0 + (uint64_t)((buf * C::TILE_BYTES + s_chunk * C::CHUNK_BYTES) >> 4);
            const uint64_t qb = q_desc + (uint64_t)((s_chunk * C::QCHUNK_BYTES) >> 4);
            const uint32_t d = tmem_base + ((uint32_t)(16 * buf) << 16) + C::S_COL;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16_ss(d, sb + (uint64_t)((kk * 32) >> 4), qb + (uint64_t)((kk * 32) >> 4), C::IDESC_S,
                          (s_chunk | kk) ? 1u : 0u);
            if (++s_chunk == C::KCH) {
              mma_commit(&sc->s_full[buf]);
              s_chunk = 0;
              ++s_tile;
            }
            progressed = true;
          }
        }
        if (progressed) {
          spins = 0;
          t_idle = global_timer_ns();
        } else if ((++spins & 255u) == 0) {
          if (*abort_flag) ok = false;
          else if (global_timer_ns() - t_idle > kWaitLimitNs) {
            raise_error(kErrTimeout);
            ok = false;
          }
        }
      }
      if (!ok) *abort_flag = 1;
      mma_commit(&sc->mma_done);
      mbar_wait(&sc->mma_done, 0, nullptr);
    }
  } else {
    // ------------------------------------------------------------- softmax + epilogue
    // Lane L of warp w owns row 16 w + (L & 15) of the current tile and heads
    // 32 (L >> 4) .. 32 (L >> 4) + 31 (the 16x32bx2 TMEM load pattern).
    const int st = threadIdx.x;                // 0..127
    const int sw = warp;                       // softmax warp 0..3 == TMEM lane quarter
    const int hh = lane >> 4;                  // head half
    const int row = 16 * warp + (lane & 15);   // tile row
    const int r = 32 * warp + lane;            // epilogue: latent column within a 128-block
    const uint32_t lane_base = tmem_base + ((uint32_t)(warp * 32) << 16);
    const int sb = p.q_seq[t];
    const bool seq_ok = (sb >= 0 && sb < p.B);
    const int64_t seq_base = seq_ok ? p.seq_row_start[sb] : 0;
    if (st < kHeads) {
      sc->fac[st] = p.qmul[(int64_t)t * kHeads + st] * p.scale_log2e;
      sc->m_used[st] = -INFINITY;
    }
    named_bar_sync(1, 128);
    float fac[32], mref[32], l_part[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      fac[c] = sc->fac[hh * 32 + c];
      mref[c] = -INFINITY;
      l_part[c] = 0.f;
    }
    const uint32_t pbase = smem_u32(ps) + row * 128;
    // A row takes part only if its index is a real position of the sequence
    // (entries of -1 inside the counted prefix are skipped).  The index of the
    // next tile's row is loaded one tile ahead.
    auto row_index = [&](int i) -> int32_t {
      const int rr = r_begin + i * C::ROWS + row;
      return (i < n_tiles && rr < r_end && seq_ok) ? p.idx[(int64_t)t * p.k + rr] : -1;
    };
    int32_t sidx_next = row_index(0);
    bool ok = true;
    for (int i = 0; i < n_tiles && ok; ++i) {
      const int buf = i & 1;
      const int32_t sidx = sidx_next;
      sidx_next = row_index(i + 1);
      const bool valid = sidx >= 0 && seq_base + sidx < p.n_rows;
      const bool got_s = mbar_wait(&sc->s_full[buf], (uint32_t)((i >> 1) & 1), abort_flag);
      if (named_bar_or(1, 128, !got_s)) { ok = false; break; }   // leave together
      tc_fence_after();
      uint32_t v[32];
      tmem_ld16x2_32(lane_base + ((uint32_t)(16 * buf) << 16) + C::S_COL, v);
      tmem_wait_ld();
      // Speculative weights against the current references; valid unless a
      // logit exceeds its head's reference by more than 2^8.
      float dmax = -INFINITY;
      uint32_t pk[16];
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        const float d0 = fmaf(__uint_as_float(v[c]), fac[c], -mref[c]);
        const float d1 = fmaf(__uint_as_float(v[c + 1]), fac[c + 1], -mref[c + 1]);
        dmax = fmaxf(dmax, fmaxf(d0, d1));
        pk[c >> 1] = pack_bf16x2(ex2_approx(d0), ex2_approx(d1));
      }
      const bool grow = named_bar_or(1, 128, valid && !(dmax <= 8.f));
      if (grow) {
        // Exact per-head maxima of the tile (always on the first tile).
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float z = valid ? __uint_as_float(v[c]) * fac[c] : -INFINITY;
          const int zl = (hh == 0) ? f2ord(z) : f2ord(-INFINITY);
          const int zh = (hh == 1) ? f2ord(z) : f2ord(-INFINITY);
          const int m_lo = warp_max_s32(zl);   // head c      over this warp's 16 rows
          const int m_hi = warp_max_s32(zh);   // head 32 + c over this warp's 16 rows
          if (lane == c) {
            sc->red[sw][c] = m_lo;
            sc->red[sw][32 + c] = m_hi;
          }
        }
        named_bar_sync(1, 128);
        bool resc = false;
        if (st < kHeads) {
          float tmax = ord2f(sc->red[0][st]);
#pragma unroll
          for (int w2 = 1; w2 < 4; ++w2) tmax = fmaxf(tmax, ord2f(sc->red[w2][st]));
          const float mo = sc->m_used[st];
          float al = 1.f;
          if (tmax > mo) {
            al = (mo == -INFINITY) ? 0.f : ex2_approx(mo - tmax);
            resc = (mo != -INFINITY);
            sc->m_used[st] = tmax;
          }
          sc->alpha[st] = al;
        }
        const bool any_resc = named_bar_or(1, 128, resc);
        if (any_resc) {
          // O(i-1) must be complete before O^T is rescaled in place.
          const bool got_o = mbar_wait(&sc->o_done, (uint32_t)((i - 1) & 1), abort_flag);
          if (named_bar_or(1, 128, !got_o)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int blk = 0; blk < 4; ++blk) {
#pragma unroll 1
            for (int h2 = 0; h2 < 2; ++h2) {
              uint32_t u[32];
              const uint32_t a = lane_base + C::O_COL + blk * 64 + h2 * 32;
              tmem_ld32(a, u);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 32; ++c)
                u[c] = __float_as_uint(__uint_as_float(u[c]) * sc->alpha[h2 * 32 + c]);
              tmem_st32(a, u);
            }
          }
          tmem_wait_st();
        }
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          l_part[c] *= sc->alpha[hh * 32 + c];
          mref[c] = sc->m_used[hh * 32 + c];
        }
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float d0 = fmaf(__uint_as_float(v[c]), fac[c], -mref[c]);
          const float d1 = fmaf(__uint_as_float(v[c + 1]), fac[c + 1], -mref[c + 1]);
          pk[c >> 1] = pack_bf16x2(ex2_approx(d0), ex2_approx(d1));
        }
      }
      if (!valid) {
#pragma unroll
        for (int c = 0; c < 16; ++c) pk[c] = 0u;
      }
      if (i > 0) {
        // O(i-1) finished: P^T of the previous tile is no longer read.
        const bool got_o = mbar_wait(&sc->o_done, (uint32_t)((i - 1) & 1), abort_flag);
        if (named_bar_or(1, 128, !got_o)) { ok = false; break; }
        tc_fence_after();
      }
      // This thread's 32 heads of the row's P^T (bf16) and the row sums of the
      // rounded weights the tensor core multiplies.
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const int q = hh * 4 + q4;   // 16-byte group of 8 heads
        st_shared_v4(pbase + ((q ^ (row & 7)) << 4), pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
      }
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        l_part[2 * c] += __uint_as_float(pk[c] << 16);
        l_part[2 * c + 1] += __uint_as_float(pk[c] & 0xFFFF0000u);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&sc->p_full);
    }
    if (!ok) *abort_flag = 1;

    // ---- epilogue: per-head row sums, then normalised output or partials
    bool have_o = ok && n_tiles > 0;
    if (have_o) {
      const bool got_o = mbar_wait(&sc->o_done, (uint32_t)((n_tiles - 1) & 1), abort_flag);
      have_o = !named_bar_or(1, 128, !got_o);
      tc_fence_after();
    }
    float* lsum = reinterpret_cast<float*>(&sc->red[0][0]);
    named_bar_sync(1, 128);
    // Sum each head over the 16 rows of this warp (lanes sharing a head half).
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      float s = l_part[c];
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      l_part[c] = s;
    }
    if ((lane & 15) == 0) {
#pragma unroll
      for (int c = 0; c < 32; ++c) lsum[sw * kHeads + hh * 32 + c] = l_part[c];
    }
    named_bar_sync(1, 128);
    if (st < kHeads) {
      const float L = lsum[st] + lsum[kHeads + st] + lsum[2 * kHeads + st] + lsum[3 * kHeads + st];
      sc->alpha[st] = L;   // reuse: final row sum per head
    }
    named_bar_sync(1, 128);
    const int64_t unit = (int64_t)t * p.n_split + jsplit;
    if (p.n_split == 1) {
      __nv_bfloat16* o_t = p.out + (int64_t)t * kHeads * kLatent;
#pragma unroll 1
      for (int blk = 0; blk < 4; ++blk) {
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t u[32];
          if (have_o) {
            tmem_ld32(lane_base + C::O_COL + blk * 64 + hh * 32, u);
            tmem_wait_ld();
          }
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int h = hh * 32 + c;
            const float L = sc->alpha[h];
            const float o = (have_o && L > 0.f) ? __uint_as_float(u[c]) / L : 0.f;
            o_t[(int64_t)h * kLatent + blk * 128 + r] = __float2bfloat16_rn(o);
          }
        }
      }
      if (p.lse != nullptr && st < kHeads) {
        const float L = sc->alpha[st];
        p.lse[(int64_t)t * kHeads + st] =
            (have_o && L > 0.f) ? (sc->m_used[st] + lg2_approx(L)) * 0.69314718055994531f : -INFINITY;
      }
    } else {
      float* wo = p.ws_o + unit * kHeads * kLatent;
#pragma unroll 1
      for (int blk = 0; blk < 4; ++blk) {
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t u[32];
          if (have_o) {
            tmem_ld32(lane_base + C::O_COL + blk * 64 + hh * 32, u);
            tmem_wait_ld();
          }
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int h = hh * 32 + c;
            wo[(int64_t)h * kLatent + blk * 128 + r] = have_o ? __uint_as_float(u[c]) : 0.f;
          }
        }
      }
      if (st < kHeads) {
        float* ml = p.ws_ml + (unit * kHeads + st) * 2;
        ml[0] = have_o ? sc->m_used[st] : -INFINITY;
        ml[1] = have_o ? sc->alpha[st] : 0.f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// Merges the split partials of each (query, head): o = sum_j 2^(m_j - M) O_j / L,
// L = sum_j 2^(m_j - M) l_j, lse = (M + log2 L) ln 2.  One block per
// (query, head); each of the 128 threads owns 4 latent columns.
constexpr int kMaxSplits = 32;
__global__ void __launch_bounds__(128) attend_combine_kernel(const AttendParams p) {
  const int t = blockIdx.x / kHeads;
  const int h = blockIdx.x % kHeads;
  const int ns = p.n_split;
  __shared__ float wsc[kMaxSplits];
  __shared__ float stats[2];
  if (threadIdx.x < 32) {
    const int j = threadIdx.x;
    const int64_t u = (int64_t)t * ns + j;
    const float m = (j < ns) ? p.ws_ml[(u * kHeads + h) * 2] : -INFINITY;
    const float l = (j < ns) ? p.ws_ml[(u * kHeads + h) * 2 + 1] : 0.f;
    float M = m;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float sc = (m == -INFINITY) ? 0.f : ex2_approx(m - M);
    float L = sc * l;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    wsc[j] = (L > 0.f) ? sc / L : 0.f;
    if (j == 0) {
      stats[0] = M;
      stats[1] = L;
    }
  }
  __syncthreads();
  const int d = threadIdx.x * 4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < ns; ++j) {
    const float wj = wsc[j];
    const float4 o4 = *reinterpret_cast<const float4*>(p.ws_o + (((int64_t)t * ns + j) * kHeads + h) * kLatent + d);
    acc.x = fmaf(wj, o4.x, acc.x);
    acc.y = fmaf(wj, o4.y, acc.y);
    acc.z = fmaf(wj, o4.z, acc.z);
    acc.w = fmaf(wj, o4.w, acc.w);
  }
  __nv_bfloat16* o = p.out + ((int64_t)t * kHeads + h) * kLatent + d;
  *reinterpret_cast<__nv_bfloat162*>(o) = __floats2bfloat162_rn(acc.x, acc.y);
  *reinterpret_cast<__nv_bfloat162*>(o + 2) = __floats2bfloat162_rn(acc.z, acc.w);
  if (threadIdx.x == 0 && p.lse != nullptr) {
    const float L = stats[1];
    p.lse[(int64_t)t * kHeads + h] = (L > 0.f) ? (stats[0] + lg2_approx(L)) * 0.69314718055994531f : -INFINITY;
  }
}

}  // namespace dsa
