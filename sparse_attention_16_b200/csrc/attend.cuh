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

#include "ptx.cuh"

namespace dsa {

constexpr int kHeads = 64;
constexpr int kLatent = 512;

template <int DR>
struct AttCfg {
  static constexpr int KCH = (kLatent + DR) / 64;        // 64-column chunks: 9 or 8
  static constexpr int ROWS = 128;                       // rows per tile (MMA M)
  static constexpr int CHUNK_BYTES = ROWS * 128;         // 16 KB
  static constexpr int QCHUNK_BYTES = kHeads * 128;      // 8 KB
  static constexpr int Q_BYTES = KCH * QCHUNK_BYTES;
  static constexpr int C_BYTES = KCH * CHUNK_BYTES;
  static constexpr bool P_IN_ROPE = (DR == 64);
  static constexpr int P_BYTES = ROWS * 128;
  static constexpr int DATA_BYTES = Q_BYTES + C_BYTES + (P_IN_ROPE ? 0 : P_BYTES);
  static constexpr int SCRATCH_BYTES = 4096;
  static constexpr int SMEM_BYTES = 1024 + DATA_BYTES + SCRATCH_BYTES;
  static constexpr int THREADS = 8 * 32;
  static constexpr int PRODUCERS = 96;   // warps 5-7
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t S_COL = 0;
  static constexpr uint32_t O_COL = 128;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(128, kHeads, 0, 0);
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
  int32_t rows_per_split;         // multiple of 128
};

struct AttScratch {
  uint64_t q_full;
  uint64_t s_full;
  uint64_t p_full;
  uint64_t o_done;
  uint64_t mma_done;
  uint64_t c_full[9];
  uint64_t c_free[9];
  uint32_t tmem_slot;
  int abort_flag;
  int32_t rowidx[128];            // absolute cache row per tile row (-1 = empty)
  float fac[64];                  // scale * m[t,h] * log2(e)
  float m_used[64];               // running (lazy) max per head, log2 units
  float alpha[64];                // rescale factor of the current tile
  int32_t red[4][64];             // per-warp head maxima (order-mapped ints) / sums
};

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

template <int DR>
__global__ void __launch_bounds__(AttCfg<DR>::THREADS, 1)
    attend_kernel(const __grid_constant__ CUtensorMap qn_map, const __grid_constant__ CUtensorMap qp_map,
                  const AttendParams p) {
  using C = AttCfg<DR>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* qs = smem;
  uint8_t* cs = smem + C::Q_BYTES;
  uint8_t* ps = C::P_IN_ROPE ? (cs + 8 * C::CHUNK_BYTES) : (cs + C::C_BYTES);
  AttScratch* sc = reinterpret_cast<AttScratch*>(smem + C::DATA_BYTES);
  volatile int* abort_flag = &sc->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x / p.n_split;
  const int jsplit = blockIdx.x % p.n_split;

  if (threadIdx.x == 0) {
    mbar_init(&sc->q_full, 1);
    mbar_init(&sc->s_full, 1);
    mbar_init(&sc->p_full, 128);
    mbar_init(&sc->o_done, 1);
    mbar_init(&sc->mma_done, 1);
    for (int c = 0; c < C::KCH; ++c) {
      mbar_init(&sc->c_full[c], C::PRODUCERS);
      mbar_init(&sc->c_free[c], 1);
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
    // every chunk.  The destination offsets (with the 128-byte swizzle) depend
    // only on the row, so they are computed once; the source row addresses once
    // per tile; each copy then costs two adds.
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
    const int prow = 4 * (warp - 5) + (lane >> 3);  // rows prow + 12 j
    const int piece = lane & 7;                       // 16-byte piece of the 128-byte chunk row
    constexpr int RPT = (C::ROWS + 11) / 12;          // rows per thread (10 or 11)
    const uint32_t cs0 = smem_u32(cs);
    uint32_t dst[RPT];
#pragma unroll
    for (int j = 0; j < RPT; ++j) {
      const int r = prow + 12 * j;
      dst[j] = cs0 + r * 128 + ((piece ^ (r & 7)) << 4);
    }
    const char* cache_bytes = reinterpret_cast<const char*>(p.cache);
    bool ok = true;
    for (int i = 0; i < n_tiles && ok; ++i) {
      const int r0 = r_begin + i * C::ROWS;
      const int nvalid = min(C::ROWS, r_end - r0);
      const char* src[RPT];
      uint32_t nbytes[RPT];
#pragma unroll
      for (int j = 0; j < RPT; ++j) {
        const int r = prow + 12 * j;
        src[j] = cache_bytes;
        nbytes[j] = 0;
        if (r < C::ROWS && r < nvalid && seq_ok) {
          const int32_t sidx = p.idx[(int64_t)t * p.k + r0 + r];
          if (sidx >= 0 && base + sidx < p.n_rows) {
            src[j] = cache_bytes + ((base + sidx) * p.ld_c) * 2 + piece * 16;
            nbytes[j] = 16;
          } else if (sidx != -1 && piece == 0) {
            raise_error(kErrBadIndex);
          }
        }
      }
      for (int c = 0; c < C::KCH; ++c) {
        if (i > 0 && !mbar_wait(&sc->c_free[c], (uint32_t)((i - 1) & 1), abort_flag)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int j = 0; j < RPT; ++j) {
          if (prow + 12 * j < C::ROWS)
            cp_async_16(dst[j] + c * C::CHUNK_BYTES, src[j] + (nbytes[j] ? c * 128 : 0), nbytes[j]);
        }
        cp_async_arrive_noinc(&sc->c_full[c]);
      }
    }
    if (!ok) *abort_flag = 1;
    cp_async_wait_all();   // nothing may still be landing in shared memory at exit
    if (pt == 0 && n_tiles > 0) mbar_wait(&sc->q_full, 0, nullptr);
  } else if (warp == 4) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0 && n_tiles > 0) {
      bool ok = mbar_wait(&sc->q_full, 0, abort_flag);
      const uint32_t qaddr = smem_u32(qs);
      const uint32_t caddr = smem_u32(cs);
      const uint32_t paddr = smem_u32(ps);
      for (int i = 0; i < n_tiles && ok; ++i) {
        const uint32_t ph = (uint32_t)(i & 1);
        for (int c = 0; c < C::KCH; ++c) {
          if (!mbar_wait(&sc->c_full[c], ph, abort_flag)) { ok = false; break; }
          fence_proxy_async_smem();   // cp.async wrote through the generic proxy
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = sdesc_sw128(caddr + c * C::CHUNK_BYTES + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(qaddr + c * C::QCHUNK_BYTES + kk * 32, 16, 1024);
            mma_bf16_ss(tmem_base + C::S_COL, ad, bd, C::IDESC_S, (c | kk) ? 1u : 0u);
          }
        }
        if (!ok) break;
        mma_commit(&sc->s_full);
        if (!mbar_wait(&sc->p_full, ph, abort_flag)) { ok = false; break; }
        tc_fence_after();
        fence_proxy_async_smem();     // P^T was written with st.shared
#pragma unroll 1
        for (int blk = 0; blk < 4; ++blk) {
#pragma unroll
          for (int kk = 0; kk < C::ROWS / 16; ++kk) {
            const uint64_t ad =
                sdesc_sw128(caddr + 2 * blk * C::CHUNK_BYTES + kk * 2048, C::CHUNK_BYTES, 1024);
            const uint64_t bd = sdesc_sw128(paddr + kk * 2048, C::CHUNK_BYTES, 1024);
            mma_bf16_ss(tmem_base + C::O_COL + blk * 64, ad, bd, C::IDESC_O,
                        (i > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&sc->c_free[2 * blk]);
          mma_commit(&sc->c_free[2 * blk + 1]);
        }
        if (DR == 64) mma_commit(&sc->c_free[8]);
        mma_commit(&sc->o_done);
      }
      if (!ok) *abort_flag = 1;
      mma_commit(&sc->mma_done);
      mbar_wait(&sc->mma_done, 0, nullptr);
    }
  } else {
    // ------------------------------------------------------------- softmax + epilogue
    const int st = threadIdx.x;                // 0..127
    const int sw = warp;                       // softmax warp 0..3
    const int quarter = warp;
    const int r = quarter * 32 + lane;         // tile row == TMEM lane
    const uint32_t lane_base = tmem_base + ((uint32_t)(quarter * 32) << 16);
    const int sb = p.q_seq[t];
    const bool seq_ok = (sb >= 0 && sb < p.B);
    const int64_t seq_base = seq_ok ? p.seq_row_start[sb] : 0;
    if (st < kHeads) {
      sc->fac[st] = p.qmul[(int64_t)t * kHeads + st] * p.scale_log2e;
      sc->m_used[st] = -INFINITY;
    }
    named_bar_sync(1, 128);
    float l_part[kHeads];
#pragma unroll
    for (int h = 0; h < kHeads; ++h) l_part[h] = 0.f;
    const uint32_t pbase = smem_u32(ps) + r * 128;
    const float4* fac4 = reinterpret_cast<const float4*>(sc->fac);
    const float4* mu4 = reinterpret_cast<const float4*>(sc->m_used);
    bool ok = true;
    for (int i = 0; i < n_tiles && ok; ++i) {
      const uint32_t ph = (uint32_t)(i & 1);
      const int nvalid = min(C::ROWS, r_end - (r_begin + i * C::ROWS));
      // A row takes part only if its index is a real position of the sequence
      // (entries of -1 inside the counted prefix are skipped).
      bool valid = false;
      if (r < nvalid && seq_ok) {
        const int32_t sidx = p.idx[(int64_t)t * p.k + r_begin + i * C::ROWS + r];
        valid = sidx >= 0 && seq_base + sidx < p.n_rows;
      }
      const bool got_s = mbar_wait(&sc->s_full, ph, abort_flag);
      if (named_bar_or(1, 128, !got_s)) { ok = false; break; }   // leave together
      tc_fence_after();

      // Common case: every logit of this tile is at most 2^8 above the head's
      // reference m_used (the first tile always fails this test: m_used = -inf).
      float dmax = -INFINITY;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t v[32];
        tmem_ld32(lane_base + C::S_COL + half * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
          const float4 f = fac4[half * 8 + q4];
          const float4 m = mu4[half * 8 + q4];
          dmax = fmaxf(dmax, fmaf(__uint_as_float(v[4 * q4 + 0]), f.x, -m.x));
          dmax = fmaxf(dmax, fmaf(__uint_as_float(v[4 * q4 + 1]), f.y, -m.y));
          dmax = fmaxf(dmax, fmaf(__uint_as_float(v[4 * q4 + 2]), f.z, -m.z));
          dmax = fmaxf(dmax, fmaf(__uint_as_float(v[4 * q4 + 3]), f.w, -m.w));
        }
      }
      const bool grow = named_bar_or(1, 128, valid && !(dmax <= 8.f));
      if (grow) {
        // Exact per-head maxima of the tile: warp max-reductions, then across warps.
        int mine0 = 0, mine1 = 0;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t v[32];
          tmem_ld32(lane_base + C::S_COL + half * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int h = half * 32 + c;
            const float z = valid ? __uint_as_float(v[c]) * sc->fac[h] : -INFINITY;
            const int m = warp_max_s32(f2ord(z));
            if (lane == c) {
              if (half == 0) mine0 = m; else mine1 = m;
            }
          }
        }
        sc->red[sw][lane] = mine0;
        sc->red[sw][32 + lane] = mine1;
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
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              uint32_t u[32];
              const uint32_t a = lane_base + C::O_COL + blk * 64 + half * 32;
              tmem_ld32(a, u);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 32; ++c)
                u[c] = __float_as_uint(__uint_as_float(u[c]) * sc->alpha[half * 32 + c]);
              tmem_st32(a, u);
            }
          }
          tmem_wait_st();
#pragma unroll
          for (int h = 0; h < kHeads; ++h) l_part[h] *= sc->alpha[h];
        }
      }
      if (i > 0) {
        // O(i-1) finished: P^T of the previous tile is no longer read.
        const bool got_o = mbar_wait(&sc->o_done, (uint32_t)((i - 1) & 1), abort_flag);
        if (named_bar_or(1, 128, !got_o)) { ok = false; break; }
        tc_fence_after();
      }
      // p = 2^(z - m), this row of P^T (64 heads, bf16), and the row sums.
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t v[32];
        tmem_ld32(lane_base + C::S_COL + half * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = q8 * 8 + 2 * e;
            const int h0 = half * 32 + c;
            const float4 f = fac4[h0 >> 2];
            const float4 m = mu4[h0 >> 2];
            const float f0 = (h0 & 2) ? f.z : f.x, f1 = (h0 & 2) ? f.w : f.y;
            const float m0 = (h0 & 2) ? m.z : m.x, m1 = (h0 & 2) ? m.w : m.y;
            const float p0 = valid ? ex2_approx(fmaf(__uint_as_float(v[c]), f0, -m0)) : 0.f;
            const float p1 = valid ? ex2_approx(fmaf(__uint_as_float(v[c + 1]), f1, -m1)) : 0.f;
            pk[e] = pack_bf16x2(p0, p1);
            // Sum the bf16-rounded weights the tensor core multiplies, so the
            // numerator and the denominator of the softmax use the same values.
            l_part[h0] += __uint_as_float(pk[e] << 16);
            l_part[h0 + 1] += __uint_as_float(pk[e] & 0xFFFF0000u);
          }
          const int q = half * 4 + q8;   // 16-byte group of 8 heads
          st_shared_v4(pbase + ((q ^ (r & 7)) << 4), pk[0], pk[1], pk[2], pk[3]);
        }
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
#pragma unroll
    for (int h = 0; h < kHeads; ++h) {
      float s = l_part[h];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      l_part[h] = s;
    }
    if (lane == 0) {
#pragma unroll
      for (int h = 0; h < kHeads; ++h) lsum[sw * kHeads + h] = l_part[h];
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
        for (int half = 0; half < 2; ++half) {
          uint32_t u[32];
          if (have_o) {
            tmem_ld32(lane_base + C::O_COL + blk * 64 + half * 32, u);
            tmem_wait_ld();
          }
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int h = half * 32 + c;
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
        for (int half = 0; half < 2; ++half) {
          uint32_t u[32];
          if (have_o) {
            tmem_ld32(lane_base + C::O_COL + blk * 64 + half * 32, u);
            tmem_wait_ld();
          }
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int h = half * 32 + c;
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
// (query, group of 8 heads), one thread per latent column.
__global__ void __launch_bounds__(512) attend_combine_kernel(const AttendParams p) {
  const int t = blockIdx.x;
  const int d = threadIdx.x;
  const int ns = p.n_split;
  for (int h = blockIdx.y * 8; h < blockIdx.y * 8 + 8; ++h) {
    float M = -INFINITY;
    for (int j = 0; j < ns; ++j) M = fmaxf(M, p.ws_ml[(((int64_t)t * ns + j) * kHeads + h) * 2]);
    float L = 0.f, acc = 0.f;
    if (M != -INFINITY) {
      for (int j = 0; j < ns; ++j) {
        const int64_t u = (int64_t)t * ns + j;
        const float m = p.ws_ml[(u * kHeads + h) * 2];
        if (m == -INFINITY) continue;
        const float sc = ex2_approx(m - M);
        L += sc * p.ws_ml[(u * kHeads + h) * 2 + 1];
        acc += sc * p.ws_o[(u * kHeads + h) * kLatent + d];
      }
    }
    const float o = (L > 0.f) ? acc / L : 0.f;
    p.out[((int64_t)t * kHeads + h) * kLatent + d] = __float2bfloat16_rn(o);
    if (d == 0 && p.lse != nullptr)
      p.lse[(int64_t)t * kHeads + h] = (L > 0.f) ? (M + lg2_approx(L)) * 0.69314718055994531f : -INFINITY;
  }
}

}  // namespace dsa
