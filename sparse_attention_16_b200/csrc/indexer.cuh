// indexer.cuh - the DSA lightning indexer on sm_100a tensor cores.
//
// Computes I[t,s] = sum_{j<32} w[t,j] * max(0, q[t,j,:] . k[s,:]) (the concept
// page's "Where to look" / "Sparse attention": 32 small heads, 32 x 128
// multiply-adds per scored position).
//
// One tile = 128 consecutive key rows of one sequence x QG queries (QG = 1 for
// decode, 4 for several queries of one sequence decoded together - e.g. the
// verification of drafted tokens - and 8 for chunked prefill).  The 128 x 128 bf16 key tile and the
// (32*QG) x 128 query block are brought into shared memory by TMA with the
// 128-byte swizzle; one tcgen05.mma chain (M = 128 keys, N = 32*QG, K = 128)
// leaves, in TMEM lane r, the 32 head dot products of key r for every query in
// the group.  The epilogue applies ReLU, the head weights and the head sum in
// registers, so each key row costs one TMEM row read and a 32-term FMA chain.
//
// FP8 keys (F8 = true): key rows and query heads are E4M3 codes with one fp32
// scale per key row and per query head (k = k_scale[s] e4m3(k8[s]),
// q_j = q_scale[t,j] e4m3(q8[t,j]); the concept page keeps indexer keys in FP8,
// "1M-token serving scenario", without a scale convention).  Both scales are
// positive, so ReLU commutes with them: the MMA runs on the raw codes
// (kind::f8f6f4, K = 32), q_scale is folded into the head weights and k_scale
// multiplies each key's head sum.  A key row is 128 B, one swizzle row, so a
// key tile is 16 KB and twice as many tiles are in flight.
//
// Warp roles (persistent CTA, one per SM, contiguous range of tiles):
//   warp 0        TMA producer (key tiles ring, query block buffers)
//   warp 1        TMEM owner + single-thread MMA issuer (FP8 decode: a second
//                 issuer warp after the epilogue warps takes every other tile)
//   warps 2..     epilogue (4, 8 or 12 warps), two or six TMEM accumulators in flight
#pragma once

#include <cuda.h>

#include "ptx.cuh"

namespace dsa {

constexpr int kIdxHeads = 32;
constexpr int kIdxDim = 128;
constexpr int kKeyTile = 128;

// Instruction descriptor of tcgen05.mma kind::f8f6f4 with E4M3 A and B (format
// code 0), f32 accumulate, both K-major.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4)                          // D format: f32
         | ((uint32_t)(N >> 3) << 17)       // N / 8
         | ((uint32_t)(M >> 4) << 24);      // M / 16
}

template <int QG, bool F8 = false>
struct IdxCfg {
  static constexpr int N = 32 * QG;                     // MMA N: heads x queries
  static constexpr int KBLK = F8 ? 1 : 2;               // 128-byte column blocks per row
  static constexpr int STAGES = F8 ? ((QG == 1) ? 12 : 8) : ((QG == 1) ? 6 : 4);   // key tiles in flight
  static constexpr int QBUFS = (QG == 8) ? 1 : 2;       // query blocks in flight
  static constexpr int KHALF = kKeyTile * 128;          // bytes of one 128-byte column block
  static constexpr int KT_BYTES = KBLK * KHALF;         // 32 KB (bf16) / 16 KB (fp8) per key tile
  static constexpr int QHALF = N * 128;
  static constexpr int Q_BYTES = KBLK * QHALF;
  static constexpr int KSTEPS = F8 ? kIdxDim / 32 : kIdxDim / 16;   // MMAs per tile (K = 32 / 16)
  // Epilogue warps.  QG 4: four warps x four queries; QG 8: two halves of four warps, four
  // queries each; FP8 decode: three sets of four warps take the accumulators (tiles) in turn
  // (measured at 1M keys per query: one set 130 us, two 112 us, three 110 us).
  static constexpr int EPI_SETS = (F8 && QG == 1) ? 3 : 1;
  static constexpr int EPI_WARPS = (QG == 8) ? 8 : 4 * EPI_SETS;
  // MMA-issuing threads: FP8 decode tiles are small (4 MMAs of M128 N32 K32), so two
  // issuers (warp 1 and the warp after the epilogue) take the tiles in turn.  The
  // issuer count must divide the accumulator and stage counts: every accumulator
  // and stage then always has the same issuer, whose parity waits on it stay in
  // order (an issuer may otherwise wait on a phase two ahead of the barrier and
  // pass at once).  Measured: a third issuer adds nothing.
  static constexpr int ISSUERS = (F8 && QG == 1) ? 2 : 1;
  static constexpr int ISSUER2_WARP = 2 + EPI_WARPS;   // first of the extra issuer warps
  static constexpr int THREADS = 64 + 32 * EPI_WARPS + 32 * (ISSUERS - 1);
  static constexpr int NACC = (F8 && QG == 1) ? 2 * EPI_SETS : 2;   // TMEM accumulators in flight (measured best)
  static constexpr int TMEM_COLS = (NACC * N <= 32) ? 32 : (NACC * N <= 64) ? 64 : (NACC * N <= 128) ? 128
                                   : (NACC * N <= 256) ? 256 : 512;   // allocations are powers of two
  static constexpr int SMEM_TILES = STAGES * KT_BYTES + QBUFS * Q_BYTES;
  static constexpr int W_BYTES = EPI_WARPS * ((QG == 1) ? 1 : 4) * kIdxHeads * 4;
  static constexpr int HIST_BYTES = (QG == 1) ? 2048 * 4 : 0;   // decode: score histogram of the current query
  static constexpr int KS_AHEAD = F8 ? 4 : 0;                    // key-scale loads issued this many tiles ahead
  static constexpr int KS_BYTES = F8 ? EPI_WARPS * (KS_AHEAD + 1) * 32 * 4 : 0;
  static constexpr int SMEM_BYTES = 1024 + SMEM_TILES + 1024 + W_BYTES + HIST_BYTES + KS_BYTES;
  static constexpr uint32_t IDESC = F8 ? idesc_e4m3_f32(128, N) : idesc_bf16_f32(128, N, 0, 0);
  static_assert(NACC % ISSUERS == 0 && STAGES % ISSUERS == 0, "each accumulator and stage has one issuer");
  static_assert(NACC % EPI_SETS == 0, "each accumulator has one epilogue set");
};

struct IndexerParams {
  const float* w;                 // [T, 32]
  const float* q_scale;           // [T, 32] (FP8 keys only)
  const float* k_scale;           // [n_rows] (FP8 keys only)
  const int64_t* seq_row_start;   // [B]
  const int32_t* q_seq;           // [T]
  const int32_t* q_pos;           // [T]
  float* scores;                  // [T, ld]
  uint32_t* hist;                 // [T, 2048] or null (q_group 1): candidates' score keys counted by their
                                  // top 11 bits, accumulated (the caller zeroes it)
  int64_t ld;
  int64_t n_rows;
  int64_t n_units;                // n_groups * n_kt
  int32_t T;
  int32_t B;
  int32_t n_kt;                   // ceil(ld / 128)
};

struct GroupInfo {
  int64_t row_base;   // first key row of the sequence
  int32_t maxpos;     // largest candidate position over the group (-1: none)
};

template <int QG>
__device__ __forceinline__ GroupInfo load_group(const IndexerParams& p, int g, bool report) {
  GroupInfo gi{0, -1};
  const int t0 = g * QG;
  const int b = p.q_seq[t0];
  if (b < 0 || b >= p.B) {
    if (report) raise_error(kErrBadSeq);
    return gi;
  }
  gi.row_base = p.seq_row_start[b];
  int mx = -1;
#pragma unroll
  for (int i = 0; i < QG; ++i) {
    const int t = t0 + i;
    if (t < p.T) {
      if (QG > 1 && p.q_seq[t] != b && report) raise_error(kErrMixedGroup);
      int qp = p.q_pos[t];
      if (qp >= p.ld) {
        if (report) raise_error(kErrBadSeq);
        qp = (int)p.ld - 1;
      }
      mx = max(mx, qp);
    }
  }
  if (mx >= 0 && gi.row_base + mx >= p.n_rows) {
    if (report) raise_error(kErrBadSeq);
  }
  gi.maxpos = mx;
  return gi;
}

// Group and key tile of work unit u (u = g * n_kt + kt).  The FP8 kernel
// advances (g, kt) incrementally instead; on the bf16 kernel the division per
// unit measured faster (its slower issue loop paces the key loads better on
// the decode batches), so it keeps it.
__device__ __forceinline__ void unit_of(int64_t u, int32_t n_kt, int& g, int& kt) {
  g = (int)(u / n_kt);
  kt = (int)(u % n_kt);
}

struct Ring {
  int idx;
  uint32_t phase;
  __device__ __forceinline__ void next(int n) {
    if (++idx == n) {
      idx = 0;
      phase ^= 1u;
    }
  }
};

// D[tmem] (+)= A . B with E4M3 operands from shared memory, fp32 accumulate.
__device__ __forceinline__ void mma_e4m3_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

template <int QG, bool F8>
__global__ void __launch_bounds__(IdxCfg<QG, F8>::THREADS, 1)
    indexer_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                   const IndexerParams p) {
  using C = IdxCfg<QG, F8>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* ktiles = smem;
  uint8_t* qbufs = smem + C::STAGES * C::KT_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_TILES);
  uint64_t* k_full = bars;
  uint64_t* k_empty = k_full + C::STAGES;
  uint64_t* q_full = k_empty + C::STAGES;
  uint64_t* q_empty = q_full + C::QBUFS;
  uint64_t* acc_full = q_empty + C::QBUFS;
  uint64_t* acc_empty = acc_full + C::NACC;
  uint64_t* mma_done = acc_empty + C::NACC;   // [ISSUERS]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + C::ISSUERS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* w_s = reinterpret_cast<float*>(smem + C::SMEM_TILES + 1024);
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(smem + C::SMEM_TILES + 1024 + C::W_BYTES);
  float* ks_s = reinterpret_cast<float*>(smem + C::SMEM_TILES + 1024 + C::W_BYTES + C::HIST_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < C::QBUFS; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], C::ISSUERS);
    }
    for (int i = 0; i < C::NACC; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], C::EPI_WARPS / C::EPI_SETS);
    }
    for (int i = 0; i < C::ISSUERS; ++i) mbar_init(&mma_done[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  griddep_wait();
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int64_t u_begin = (int64_t)blockIdx.x * p.n_units / gridDim.x;
  const int64_t u_end = (int64_t)(blockIdx.x + 1) * p.n_units / gridDim.x;

  if (warp == 0) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tmap(&kmap);
      const uint64_t key_policy = make_policy_evict_first();
      prefetch_tmap(&qmap);
      Ring ks{0, 0}, qs{C::QBUFS - 1, 1u};
      int cur_g = -1;
      GroupInfo gi{0, -1};
      bool kused[C::STAGES] = {};
      uint32_t klast[C::STAGES] = {};
      bool qused[C::QBUFS] = {};
      uint32_t qlast[C::QBUFS] = {};
      bool ok = true;
      int g = (int)(u_begin / p.n_kt), kt = (int)(u_begin % p.n_kt);   // unit u = g * n_kt + kt
      for (int64_t u = u_begin; u < u_end && ok; ++u, kt = (kt + 1 == p.n_kt) ? 0 : kt + 1, g += (kt == 0)) {
        if constexpr (!F8) unit_of(u, p.n_kt, g, kt);
        if (g != cur_g) {
          gi = load_group<QG>(p, g, true);
          cur_g = g;
          qs.next(C::QBUFS);
          if (!mbar_wait(&q_empty[qs.idx], qs.phase ^ 1u, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&q_full[qs.idx], C::Q_BYTES);
          uint8_t* qb = qbufs + qs.idx * C::Q_BYTES;
          for (int blk = 0; blk < C::KBLK; ++blk)   // 128-byte column blocks (64 bf16 / 128 fp8)
            tma_load_2d(qb + blk * C::QHALF, &qmap, blk * 64, g * C::N, &q_full[qs.idx]);
          qused[qs.idx] = true;
          qlast[qs.idx] = qs.phase;
        }
        if (kt * kKeyTile > gi.maxpos) continue;   // nothing to score in this tile
        if (!mbar_wait(&k_empty[ks.idx], ks.phase ^ 1u, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(&k_full[ks.idx], C::KT_BYTES);
        uint8_t* kb = ktiles + ks.idx * C::KT_BYTES;
        const int32_t row0 = (int32_t)(gi.row_base + (int64_t)kt * kKeyTile);
        for (int blk = 0; blk < C::KBLK; ++blk) {
          // decode streams each key once: evict it first, so that the scores this
          // kernel writes stay in L2 for the top-k that reads them next (prefill
          // groups re-read the keys, which then keep the normal policy)
          if constexpr (QG == 1) tma_load_2d_hint(kb + blk * C::KHALF, &kmap, blk * 64, row0, &k_full[ks.idx], key_policy);
          else tma_load_2d(kb + blk * C::KHALF, &kmap, blk * 64, row0, &k_full[ks.idx]);
        }
        kused[ks.idx] = true;
        klast[ks.idx] = ks.phase;
        ks.next(C::STAGES);
      }
      if (!ok) *abort_flag = 1;
      // Never leave the CTA with TMA writes still landing in its shared memory.
      for (int i = 0; i < C::STAGES; ++i)
        if (kused[i]) mbar_wait(&k_full[i], klast[i], nullptr);
      for (int i = 0; i < C::QBUFS; ++i)
        if (qused[i]) mbar_wait(&q_full[i], qlast[i], nullptr);
    }
  } else if (warp == 1 || (C::ISSUERS > 1 && warp >= C::ISSUER2_WARP)) {
    // ------------------------------------------------------------- MMA issuer(s)
    // Issuer j issues the tiles with (work tile number) % ISSUERS == j and only
    // steps the stage / accumulator rings over the others.
    const int issuer = (warp == 1) ? 0 : 1 + warp - C::ISSUER2_WARP;
    if (lane == 0) {
      Ring ks{0, 0}, qs{C::QBUFS - 1, 1u}, as{0, 0};
      int cur_g = -1;
      GroupInfo gi{0, -1};
      bool ok = true;
      uint32_t n_work = 0;
      int g = (int)(u_begin / p.n_kt), kt = (int)(u_begin % p.n_kt);   // unit u = g * n_kt + kt
      for (int64_t u = u_begin; u < u_end && ok; ++u, kt = (kt + 1 == p.n_kt) ? 0 : kt + 1, g += (kt == 0)) {
        if constexpr (!F8) unit_of(u, p.n_kt, g, kt);
        if (*abort_flag) { ok = false; break; }
        if (g != cur_g) {
          gi = load_group<QG>(p, g, false);
          if (cur_g >= 0) mma_commit(&q_empty[qs.idx]);   // old query block free once drained
          cur_g = g;
          qs.next(C::QBUFS);
          if (!mbar_wait(&q_full[qs.idx], qs.phase, abort_flag)) { ok = false; break; }
        }
        if (kt * kKeyTile > gi.maxpos) continue;
        if (C::ISSUERS > 1 && (int)(n_work++ % C::ISSUERS) != issuer) {   // another issuer's tile
          ks.next(C::STAGES);
          as.next(C::NACC);
          continue;
        }
        if (!mbar_wait(&acc_empty[as.idx], as.phase ^ 1u, abort_flag)) { ok = false; break; }
        if (!mbar_wait(&k_full[ks.idx], ks.phase, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kaddr = smem_u32(ktiles + ks.idx * C::KT_BYTES);
        const uint32_t qaddr = smem_u32(qbufs + qs.idx * C::Q_BYTES);
        const uint32_t d_tmem = tmem_base + (uint32_t)(as.idx * C::N);
        // K steps of 32 bytes (16 bf16 or 32 fp8 values) inside each 128-byte block
#pragma unroll
        for (int kk = 0; kk < C::KSTEPS; ++kk) {
          const uint32_t off = (uint32_t)((kk & 3) * 32);
          const uint64_t ad = sdesc_sw128(kaddr + (kk >> 2) * C::KHALF + off, 16, 1024);
          const uint64_t bd = sdesc_sw128(qaddr + (kk >> 2) * C::QHALF + off, 16, 1024);
          if constexpr (F8) mma_e4m3_ss(d_tmem, ad, bd, C::IDESC, kk > 0 ? 1u : 0u);
          else mma_bf16_ss(d_tmem, ad, bd, C::IDESC, kk > 0 ? 1u : 0u);
        }
        mma_commit(&k_empty[ks.idx]);
        mma_commit(&acc_full[as.idx]);
        ks.next(C::STAGES);
        as.next(C::NACC);
      }
      if (!ok) *abort_flag = 1;
      // Drain: every MMA issued by this thread has finished before TMEM is freed.
      mma_commit(&mma_done[issuer]);
      mbar_wait(&mma_done[issuer], 0, nullptr);
    }
  } else {
    // ------------------------------------------------------------- epilogue
    const int epi = warp - 2;                     // 0 .. EPI_WARPS-1
    const int quarter = warp & 3;                 // TMEM lanes this warp may read
    const int row = quarter * 32 + lane;          // key row within the tile
    constexpr int QPW = (QG == 1) ? 1 : 4;        // queries per epilogue warp
    const int qbase = (QG == 1) ? 0 : (epi >> 2) * 4;
    const int set = (C::EPI_SETS > 1) ? (epi >> 2) : 0;   // this warp's tiles: accumulators with idx % EPI_SETS == set
    float* w_my = w_s + epi * (QPW * kIdxHeads);
    // Decode (one query per group): every candidate score is also counted in a
    // shared-memory histogram of its key's top 11 bits, flushed to the query's
    // global histogram when the group changes and at the end (the top-k's first
    // pass).  The flushes are met by every epilogue warp, also after an abort.
    const bool do_hist = (QG == 1) && p.hist != nullptr;
    constexpr int EPI_THREADS = 32 * C::EPI_WARPS;
    const int etid = threadIdx.x - 64;
    auto flush_hist = [&](int g_old) {
      named_bar_sync(1, EPI_THREADS);   // every epilogue warp has counted its scores of g_old
      if (g_old >= 0)
        for (int b = etid; b < 2048; b += EPI_THREADS) {
          const uint32_t v = hist_s[b];
          if (v) {
            atomicAdd(&p.hist[(int64_t)g_old * 2048 + b], v);
            hist_s[b] = 0;
          }
        }
      named_bar_sync(1, EPI_THREADS);   // cleared before anyone counts the next group
    };
    if (do_hist) {
      for (int b = etid; b < 2048; b += EPI_THREADS) hist_s[b] = 0;
    }
    Ring as{0, 0};
    int cur_g = -1;
    GroupInfo gi{0, -1};
    int qpos_q[QPW];
    bool dead = false;   // gave up after an abort: keeps walking the units only to meet the flushes
    // FP8: this thread's key scale of tile kt + KS_AHEAD is copied (cp.async,
    // 4 bytes) into a warp-private ring slot while tile kt is processed, so the
    // global round trip is never on a tile's critical path.  Each thread reads
    // only the slots it wrote itself, after waiting for its own copy group.
    constexpr int KSA = C::KS_AHEAD;
    const uint32_t ks_lane = smem_u32(ks_s) + (uint32_t)((epi * (KSA + 1) * 32 + lane) * 4);
    int ks_head = 0;
    bool ks_reset = true;
    auto issue_ks = [&](int kt2, int slot) {
      const int64_t pos2 = (int64_t)kt2 * kKeyTile + row;
      const bool v = kt2 < p.n_kt && pos2 <= gi.maxpos && gi.row_base + pos2 < p.n_rows;
      const float* src = v ? p.k_scale + gi.row_base + pos2 : p.k_scale;
      asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(ks_lane + (uint32_t)(slot * 128)),
                   "l"(src), "r"(v ? 4 : 0)
                   : "memory");
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    int g = (int)(u_begin / p.n_kt), kt = (int)(u_begin % p.n_kt);   // unit u = g * n_kt + kt
    for (int64_t u = u_begin; u < u_end; ++u, kt = (kt + 1 == p.n_kt) ? 0 : kt + 1, g += (kt == 0)) {
      if constexpr (!F8) unit_of(u, p.n_kt, g, kt);
      if (!dead && *abort_flag) dead = true;
      if (dead && !do_hist) break;
      if (g != cur_g) {
        if (do_hist) flush_hist(cur_g);
        gi = load_group<QG>(p, g, false);
        cur_g = g;
        ks_reset = true;
        // Weights of this warp's queries, in a warp-private slice of shared memory.
        __syncwarp();
#pragma unroll
        for (int qi = 0; qi < QPW; ++qi) {
          const int t = g * QG + qbase + qi;
          float wv = (t < p.T) ? p.w[(int64_t)t * kIdxHeads + lane] : 0.f;
          if (F8 && t < p.T) wv *= p.q_scale[(int64_t)t * kIdxHeads + lane];   // ReLU(a x) = a ReLU(x), a > 0
          w_my[qi * kIdxHeads + lane] = wv;
        }
        __syncwarp();
#pragma unroll
        for (int qi = 0; qi < QPW; ++qi) {
          const int t = g * QG + qbase + qi;
          int qp = (t < p.T) ? p.q_pos[t] : -1;
          qpos_q[qi] = (qp >= p.ld) ? (int)p.ld - 1 : qp;
          if (gi.maxpos < 0) qpos_q[qi] = -1;     // bad sequence id: nothing valid
        }
      }
      if (dead) continue;
      const int64_t pos = (int64_t)kt * kKeyTile + row;
      float res[QPW];
      float kscale = 1.f;
      if constexpr (F8) {
        if (ks_reset) {   // new group: drop what is in flight, fill the ring from this tile on
          asm volatile("cp.async.wait_all;" ::: "memory");
          for (int i = 0; i < KSA; ++i) issue_ks(kt + i, i);
          ks_head = 0;
          ks_reset = false;
        }
        int tail = ks_head + KSA;
        if (tail > KSA) tail -= KSA + 1;
        issue_ks(kt + KSA, tail);
        asm volatile("cp.async.wait_group %0;" ::"n"(KSA) : "memory");   // this tile's copy has landed
        asm volatile("ld.shared.f32 %0, [%1];" : "=f"(kscale) : "r"(ks_lane + (uint32_t)(ks_head * 128)) : "memory");
        if (++ks_head == KSA + 1) ks_head = 0;
      }
      if (kt * kKeyTile <= gi.maxpos) {
        if (C::EPI_SETS > 1 && as.idx % C::EPI_SETS != set) {   // another set's tile: it writes the scores
          as.next(C::NACC);
          continue;
        }
        if (!mbar_wait(&acc_full[as.idx], as.phase, abort_flag)) {
          *abort_flag = 1;
          dead = true;
          continue;
        }
        tc_fence_after();
        // Per query: ReLU of the 32 head dot products, weighted head sum (two
        // partial sums to halve the dependent FMA chain; weights as float4).
        const uint32_t lane_addr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(as.idx * C::N);
#pragma unroll
        for (int qp = 0; qp < QPW; qp += (QPW > 1 ? 2 : 1)) {
          uint32_t v[2][32];
#pragma unroll
          for (int u = 0; u < (QPW > 1 ? 2 : 1); ++u)
            tmem_ld32(lane_addr + (uint32_t)((qbase + qp + u) * 32), v[u]);
          tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < (QPW > 1 ? 2 : 1); ++u) {
            const float4* wq = reinterpret_cast<const float4*>(w_my + (qp + u) * kIdxHeads);
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
              const float4 wv = wq[j4];
              s0 = fmaf(wv.x, fmaxf(__uint_as_float(v[u][4 * j4 + 0]), 0.f), s0);
              s1 = fmaf(wv.y, fmaxf(__uint_as_float(v[u][4 * j4 + 1]), 0.f), s1);
              s0 = fmaf(wv.z, fmaxf(__uint_as_float(v[u][4 * j4 + 2]), 0.f), s0);
              s1 = fmaf(wv.w, fmaxf(__uint_as_float(v[u][4 * j4 + 3]), 0.f), s1);
            }
            res[qp + u] = (s0 + s1) * kscale;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[as.idx]);
        as.next(C::NACC);
      } else {
        if (C::EPI_SETS > 1 && set != 0) continue;   // past the causal range: the first set fills it
#pragma unroll
        for (int qi = 0; qi < QPW; ++qi) res[qi] = -INFINITY;
      }
      if (pos < p.ld) {
#pragma unroll
        for (int qi = 0; qi < QPW; ++qi) {
          const int t = g * QG + qbase + qi;
          if (t < p.T) p.scores[(int64_t)t * p.ld + pos] = (pos <= qpos_q[qi]) ? res[qi] : -INFINITY;
        }
        if (do_hist && pos <= qpos_q[0]) atomicAdd(&hist_s[score_key(res[0]) >> 21], 1u);
      }
    }
    if (do_hist) flush_hist(cur_g);
    if constexpr (F8) asm volatile("cp.async.wait_all;" ::: "memory");   // no copy lands after the CTA ends
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace dsa
