// dsa_api.cu - host side of the C ABI declared in include/dsa.h: argument
// validation, TMA descriptor encoding, launch configuration and the fused
// indexer -> top-k -> per-layer attention sequence.  Every step of the hot
// path runs in the kernels included below; nothing here computes on the host.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <utility>

#include <nvtx3/nvToolsExt.h>

#include "dsa.h"
#include "attend.cuh"
#include "indexer.cuh"
#include "topk.cuh"

namespace {

thread_local std::string g_last_error;
std::atomic<uint64_t> g_launches{0};

dsa_status_t fail(dsa_status_t st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

#define DSA_REQUIRE(cond, ...)                                   \
  do {                                                           \
    if (!(cond)) return fail(DSA_ERR_INVALID_ARG, __VA_ARGS__);  \
  } while (0)

#define DSA_CUDA(call)                                                                      \
  do {                                                                                      \
    cudaError_t e_ = (call);                                                                \
    if (e_ != cudaSuccess) return fail(DSA_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

constexpr int kMaxK = 16384;

int sm_count() {
  static std::atomic<int> cached[64] = {};
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64 && (n = cached[dev].load(std::memory_order_relaxed)) > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  if (dev >= 0 && dev < 64) cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 tensor map with the 128-byte swizzle: `inner` contiguous elements
// per row, `outer` rows `row_bytes` apart, box of box_inner x box_outer.
dsa_status_t make_tmap(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                       uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  auto enc = encode_fn();
  if (enc == nullptr) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return DSA_OK;
}

// NVTX range around each C-ABI call (header-only NVTX 3: free unless a
// profiler is attached), so traces show the library's calls by name.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Raises a kernel's dynamic shared-memory limit once per device (the
// attribute persists, so later launches skip the driver call).
template <auto Kernel>
dsa_status_t set_smem(int bytes) {
  static std::atomic<uint64_t> done{0};   // one flag set per kernel (not per signature)
  int dev = 0;
  DSA_CUDA(cudaGetDevice(&dev));
  const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t(1) << dev) : 0;
  if (bit && (done.load(std::memory_order_relaxed) & bit)) return DSA_OK;
  DSA_CUDA(cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  if (bit) done.fetch_or(bit, std::memory_order_relaxed);
  return DSA_OK;
}

// Launches a kernel, as clusters of cl CTAs for cl > 1.  With DSA_PDL=1 in the
// environment the launch also allows programmatic stream serialization: every
// kernel waits in griddepcontrol.wait before touching global memory, so it may
// be scheduled while the previous kernel of the stream drains.  Off by
// default: on the decode and prefill steps measured it gained nothing (the
// kernels' set-up is short and each fills the GPU).
bool pdl_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("DSA_PDL");
    return v != nullptr && v[0] == '1';
  }();
  return on;
}

template <typename... KArgs, typename... Args>
dsa_status_t launch(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t stream,
                    unsigned cl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cl > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cl;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  DSA_CUDA(cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...));
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return DSA_OK;
}

// ----------------------------------------------------------------- indexer
// F8: q_idx / k_idx hold E4M3 codes (one byte per value) and q_scale / k_scale
// their per-head / per-row scales; otherwise bf16 values and null scales.
template <int QG, bool F8>
dsa_status_t launch_indexer(const void* q_idx, const float* q_scale, const float* w, const void* k_idx,
                            const float* k_scale, int64_t n_rows, const int64_t* seq_row_start, int32_t B,
                            const int32_t* q_seq, const int32_t* q_pos, int32_t T, float* scores, int64_t ld,
                            cudaStream_t stream) {
  using C = dsa::IdxCfg<QG, F8>;
  // One 128-byte swizzled block per box row: 64 bf16 or 128 fp8 values.  TMA
  // moves bytes, so an fp8 row (128 B) is described as 64 two-byte elements:
  // the same bytes and the same swizzle as a bf16 half row.
  const uint64_t row_elems = F8 ? dsa::kIdxDim / 2 : dsa::kIdxDim;
  const uint64_t row_bytes = F8 ? dsa::kIdxDim : dsa::kIdxDim * 2;
  CUtensorMap kmap, qmap;
  dsa_status_t st = make_tmap(&kmap, k_idx, row_elems, (uint64_t)n_rows, row_bytes, 64, dsa::kKeyTile);
  if (st != DSA_OK) return st;
  st = make_tmap(&qmap, q_idx, row_elems, (uint64_t)T * dsa::kIdxHeads, row_bytes, 64, C::N);
  if (st != DSA_OK) return st;
  dsa::IndexerParams p;
  p.w = w;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.seq_row_start = seq_row_start;
  p.q_seq = q_seq;
  p.q_pos = q_pos;
  p.scores = scores;
  p.ld = ld;
  p.n_rows = n_rows;
  p.T = T;
  p.B = B;
  p.n_kt = (int32_t)((ld + dsa::kKeyTile - 1) / dsa::kKeyTile);
  const int64_t n_groups = (T + QG - 1) / QG;
  p.n_units = n_groups * p.n_kt;
  const int grid = (int)std::min<int64_t>(p.n_units, sm_count());
  st = set_smem<dsa::indexer_kernel<QG, F8>>(C::SMEM_BYTES);
  if (st != DSA_OK) return st;
  return launch(dsa::indexer_kernel<QG, F8>, (unsigned)grid, C::THREADS, C::SMEM_BYTES, stream, 1, kmap, qmap,
                p);
}

dsa_status_t indexer_impl(const void* q_idx, const float* w, const void* k_idx, int64_t n_rows,
                          const int64_t* seq_row_start, int32_t B, const int32_t* q_seq,
                          const int32_t* q_pos, int32_t T, int32_t q_group, float* scores,
                          int64_t ld, cudaStream_t stream) {
  if (q_group == 8)
    return launch_indexer<8, false>(q_idx, nullptr, w, k_idx, nullptr, n_rows, seq_row_start, B, q_seq, q_pos,
                                    T, scores, ld, stream);
  return launch_indexer<1, false>(q_idx, nullptr, w, k_idx, nullptr, n_rows, seq_row_start, B, q_seq, q_pos, T,
                                  scores, ld, stream);
}

// ----------------------------------------------------------------- top-k
template <int CL>
dsa_status_t launch_topk_cl(const dsa::TopkParams& p, cudaStream_t stream) {
  dsa_status_t st = set_smem<dsa::topk_kernel<CL>>(dsa::kTopkSmemBytes);
  if (st != DSA_OK) return st;
  if (CL > 8) {
    static std::once_flag once;
    cudaError_t e = cudaSuccess;
    std::call_once(once, [&] {
      e = cudaFuncSetAttribute(dsa::topk_kernel<CL>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    });
    if (e != cudaSuccess) return fail(DSA_ERR_CUDA, "cluster attribute: %s", cudaGetErrorString(e));
  }
  return launch(dsa::topk_kernel<CL>, (unsigned)(p.T * CL), dsa::kTopkThreads, dsa::kTopkSmemBytes, stream,
                (unsigned)CL, p);
}

// How many top-k clusters of CL CTAs can be resident at once (16 needs the
// non-portable attribute and a GPC with 16 free SMs); 0 if none.
template <int CL>
int topk_max_clusters_t() {
  static std::atomic<int> count{-1};
  const int known = count.load(std::memory_order_relaxed);
  if (known >= 0) return known;
  int n = 0;
  bool ok = cudaFuncSetAttribute(dsa::topk_kernel<CL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 dsa::kTopkSmemBytes) == cudaSuccess;
  if (ok && CL > 8)
    ok = cudaFuncSetAttribute(dsa::topk_kernel<CL>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
         cudaSuccess;
  if (ok) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(CL);
    cfg.blockDim = dim3(dsa::kTopkThreads);
    cfg.dynamicSmemBytes = dsa::kTopkSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, dsa::topk_kernel<CL>, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  count.store(n, std::memory_order_relaxed);
  return n;
}

int topk_max_clusters(int CL) {
  switch (CL) {
    case 1: return sm_count();
    case 2: return topk_max_clusters_t<2>();
    case 4: return topk_max_clusters_t<4>();
    case 8: return topk_max_clusters_t<8>();
    case 16: return topk_max_clusters_t<16>();
    default: return 0;
  }
}

// CTAs per query: enough that each CTA owns at least ~16K candidates' worth of
// work while the batch stays within one wave (T x CL <= SMs, every cluster
// resident at once); more (up to 16) when a query's slice would not fit the
// shared-memory key stash.
int topk_cluster_size(int32_t T, int64_t ld) {
  const int sms = sm_count();
  auto fits = [&](int c) { return (int64_t)T * c <= sms && T <= topk_max_clusters(c); };
  int cl = 1;
  while (cl < 8 && (ld + cl - 1) / cl > 16384 && fits(cl * 2)) cl *= 2;
  while (cl < 16 && (ld + cl - 1) / cl > dsa::kTopkStashCap && fits(cl * 2)) cl *= 2;
  return cl;
}

dsa_status_t topk_impl(const float* scores, int64_t ld, const int32_t* q_pos, int32_t T, int32_t k,
                       int32_t* idx, int32_t* count, cudaStream_t stream) {
  dsa::TopkParams p;
  p.scores = scores;
  p.q_pos = q_pos;
  p.idx = idx;
  p.count = count;
  p.ld = ld;
  p.T = T;
  p.k = k;
  switch (topk_cluster_size(T, ld)) {
    case 1: return launch_topk_cl<1>(p, stream);
    case 2: return launch_topk_cl<2>(p, stream);
    case 4: return launch_topk_cl<4>(p, stream);
    case 8: return launch_topk_cl<8>(p, stream);
    default: return launch_topk_cl<16>(p, stream);   // chosen only when its clusters fit
  }
}

// ----------------------------------------------------------------- attention
struct SplitPlan {
  int n_split;
  int rows_per_split;
  bool merge;   // the n_split CTAs of a query form a cluster and merge in distributed shared memory
};

// How many clusters of CL attention CTAs (one per SM, 225 KB of shared memory
// each) can be resident at once (0: none, or CL outside 2..8).  A cluster must
// sit inside one GPC, so this can be well below SMs / CL.
int attend_max_clusters(int CL) {
  static std::atomic<int> count[9] = {-1, -1, -1, -1, -1, -1, -1, -1, -1};
  if (CL < 2 || CL > 8) return 0;
  const int known = count[CL].load(std::memory_order_relaxed);
  if (known >= 0) return known;
  using C = dsa::AttCfg<64>;
  int n = 0;
  if (cudaFuncSetAttribute(dsa::attend_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::SMEM_BYTES) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(CL);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, dsa::attend_kernel<64>, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  count[CL].store(n, std::memory_order_relaxed);
  return n;
}

// Splits each query's selection across CTAs so that T x n_split is about one
// wave of the GPU; rows per split are a multiple of the 64-row tile.
SplitPlan attend_plan(int32_t T, int32_t k) {
  const int tile = dsa::AttCfg<64>::ROWS;
  const int max_tiles = (k + tile - 1) / tile;
  int want = std::max(1, sm_count() / std::max(1, T));
  want = std::min(want, std::min(max_tiles, dsa::kMaxSplits));
  int tiles_per = (max_tiles + want - 1) / want;
  SplitPlan sp;
  sp.rows_per_split = tiles_per * tile;
  sp.n_split = (k + sp.rows_per_split - 1) / sp.rows_per_split;
  // Merge in clusters only when every query's cluster is resident at once;
  // otherwise the partials go through the workspace and the combine kernel.
  sp.merge = sp.n_split >= 2 && sp.n_split <= 8 && T <= attend_max_clusters(sp.n_split);
  return sp;
}

size_t attend_ws_bytes(int32_t T, int32_t k) {
  const SplitPlan sp = attend_plan(T, k);
  if (sp.n_split <= 1 || sp.merge) return 0;
  const size_t units = (size_t)T * sp.n_split;
  return round_up(units * dsa::kHeads * dsa::kLatent * 4, 256) + round_up(units * dsa::kHeads * 4 * 4, 256);
}

template <int DR>
dsa_status_t launch_attend(const void* q_nope, const void* q_pe, const float* qmul, float scale,
                           const void* cache, int64_t n_rows, int32_t ld_c,
                           const int64_t* seq_row_start, int32_t B, const int32_t* q_seq,
                           const int32_t* idx, const int32_t* count, int32_t T, int32_t k, void* out,
                           float* lse, void* ws, cudaStream_t stream) {
  using C = dsa::AttCfg<DR>;
  CUtensorMap qn_map, qp_map;
  dsa_status_t st = make_tmap(&qn_map, q_nope, dsa::kLatent, (uint64_t)T * dsa::kHeads,
                              dsa::kLatent * 2, 64, dsa::kHeads);
  if (st != DSA_OK) return st;
  if (DR == 64) {
    st = make_tmap(&qp_map, q_pe, 64, (uint64_t)T * dsa::kHeads, 128, 64, dsa::kHeads);
    if (st != DSA_OK) return st;
  } else {
    qp_map = qn_map;  // unused on NoPE layers
  }
  const SplitPlan sp = attend_plan(T, k);
  dsa::AttendParams p;
  p.q_nope = static_cast<const __nv_bfloat16*>(q_nope);
  p.q_pe = static_cast<const __nv_bfloat16*>(q_pe);
  p.cache = static_cast<const __nv_bfloat16*>(cache);
  p.qmul = qmul;
  p.seq_row_start = seq_row_start;
  p.q_seq = q_seq;
  p.idx = idx;
  p.count = count;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.ld_c = ld_c;
  p.n_rows = n_rows;
  p.scale_log2e = scale * 1.4426950408889634f;
  p.B = B;
  p.T = T;
  p.k = k;
  p.n_split = sp.n_split;
  p.rows_per_split = sp.rows_per_split;
  p.merge = sp.merge ? 1 : 0;
  p.ws_o = nullptr;
  p.ws_ml = nullptr;
  if (sp.n_split > 1 && !sp.merge) {
    const size_t units = (size_t)T * sp.n_split;
    p.ws_o = static_cast<float*>(ws);
    p.ws_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) +
                                       round_up(units * dsa::kHeads * dsa::kLatent * 4, 256));
  }
  st = set_smem<dsa::attend_kernel<DR>>(C::SMEM_BYTES);
  if (st != DSA_OK) return st;
  st = launch(dsa::attend_kernel<DR>, (unsigned)(T * sp.n_split), C::THREADS, C::SMEM_BYTES, stream,
              sp.merge ? (unsigned)sp.n_split : 1u, qn_map, qp_map, p);
  if (st != DSA_OK || sp.n_split == 1 || sp.merge) return st;
  return launch(dsa::attend_combine_kernel, (unsigned)(T * dsa::kHeads), 128, 0, stream, 1, p);
}

dsa_status_t attend_impl(const void* q_nope, const void* q_pe, const float* qmul, float scale,
                         const void* cache, int64_t n_rows, int32_t ld_c, int32_t d_rope,
                         const int64_t* seq_row_start, int32_t B, const int32_t* q_seq,
                         const int32_t* idx, const int32_t* count, int32_t T, int32_t k, void* out,
                         float* lse, void* ws, cudaStream_t stream) {
  if (d_rope == 64)
    return launch_attend<64>(q_nope, q_pe, qmul, scale, cache, n_rows, ld_c, seq_row_start, B, q_seq,
                             idx, count, T, k, out, lse, ws, stream);
  return launch_attend<0>(q_nope, q_pe, qmul, scale, cache, n_rows, ld_c, seq_row_start, B, q_seq,
                          idx, count, T, k, out, lse, ws, stream);
}

// ----------------------------------------------------------------- validation helpers
dsa_status_t check_index_args(const void* q_idx, const float* w, const void* k_idx, int64_t n_rows,
                              const int64_t* seq_row_start, int32_t B, const int32_t* q_seq,
                              const int32_t* q_pos, int32_t T, int32_t q_group, int64_t ld) {
  DSA_REQUIRE(T >= 0, "T must be >= 0 (got %d)", T);
  DSA_REQUIRE(q_idx && w && k_idx && seq_row_start && q_seq && q_pos, "null pointer argument");
  DSA_REQUIRE(aligned(q_idx, 16) && aligned(k_idx, 16), "q_idx and k_idx must be 16-byte aligned");
  DSA_REQUIRE(aligned(w, 4) && aligned(seq_row_start, 8) && aligned(q_seq, 4) && aligned(q_pos, 4),
              "misaligned w / seq_row_start / q_seq / q_pos");
  DSA_REQUIRE(B >= 1, "B must be >= 1");
  DSA_REQUIRE(n_rows >= 1 && n_rows < (int64_t(1) << 31) - 256, "n_rows out of range");
  DSA_REQUIRE(ld >= 4 && ld % 4 == 0 && ld < (int64_t(1) << 31), "ld must be a multiple of 4 in [4, 2^31)");
  DSA_REQUIRE(q_group == 1 || q_group == 8, "q_group must be 1 or 8");
  DSA_REQUIRE((int64_t)T * dsa::kIdxHeads < (int64_t(1) << 31), "T too large");
  return DSA_OK;
}

dsa_status_t check_topk_args(const float* scores, int64_t ld, const int32_t* q_pos, int32_t T,
                             int32_t k, int32_t* idx, int32_t* count) {
  DSA_REQUIRE(T >= 0, "T must be >= 0");
  DSA_REQUIRE(scores && q_pos && idx && count, "null pointer argument");
  DSA_REQUIRE(aligned(scores, 16), "scores must be 16-byte aligned");
  DSA_REQUIRE(aligned(idx, 4) && aligned(count, 4) && aligned(q_pos, 4), "misaligned idx/count/q_pos");
  DSA_REQUIRE(ld >= 4 && ld % 4 == 0 && ld < (int64_t(1) << 31), "ld must be a multiple of 4 in [4, 2^31)");
  DSA_REQUIRE(k >= 1 && k <= kMaxK, "k must be in [1, %d]", kMaxK);
  return DSA_OK;
}

dsa_status_t check_attend_args(const void* q_nope, const void* q_pe, const float* qmul,
                               const void* cache, int64_t n_rows, int32_t ld_c, int32_t d_rope,
                               const int64_t* seq_row_start, int32_t B, const int32_t* q_seq,
                               const int32_t* idx, const int32_t* count, int32_t T, int32_t k,
                               void* out) {
  DSA_REQUIRE(T >= 0, "T must be >= 0");
  DSA_REQUIRE(d_rope == 0 || d_rope == 64, "d_rope must be 0 or 64 (got %d)", d_rope);
  DSA_REQUIRE(q_nope && qmul && cache && seq_row_start && q_seq && idx && count && out,
              "null pointer argument");
  DSA_REQUIRE((q_pe != nullptr) == (d_rope == 64), "q_pe must be given iff d_rope == 64");
  DSA_REQUIRE(aligned(q_nope, 16) && aligned(cache, 16) && aligned(out, 16) &&
                  (q_pe == nullptr || aligned(q_pe, 16)),
              "q_nope, q_pe, cache and out must be 16-byte aligned");
  DSA_REQUIRE(aligned(qmul, 4) && aligned(idx, 4) && aligned(count, 4) && aligned(q_seq, 4) &&
                  aligned(seq_row_start, 8),
              "misaligned qmul/idx/count/q_seq/seq_row_start");
  DSA_REQUIRE(ld_c >= dsa::kLatent + d_rope && ld_c % 8 == 0, "ld_c must be >= 512 + d_rope and a multiple of 8");
  DSA_REQUIRE(n_rows >= 1 && n_rows * (int64_t)ld_c < (int64_t(1) << 62), "n_rows out of range");
  DSA_REQUIRE(n_rows < (int64_t(1) << 31), "n_rows must be < 2^31");
  DSA_REQUIRE(B >= 1, "B must be >= 1");
  DSA_REQUIRE(k >= 1 && k <= kMaxK, "k must be in [1, %d]", kMaxK);
  DSA_REQUIRE((int64_t)T * dsa::kHeads < (int64_t(1) << 31), "T too large");
  return DSA_OK;
}

}  // namespace

// =================================================================== no-allocation variant
// Scratch for sparse_mla_attend_noalloc: the split partials (numerators, then
// four statistics per head) of at most kNoAllocMaxPartials (query, split) work units, in
// the layout launch_attend expects of a workspace.  Every GPU that loads this
// library holds the array until the process exits.
constexpr int kNoAllocMaxPartials = DSA_NOALLOC_MAX_PARTIALS;
static __device__ __align__(256) float g_noalloc_scratch[(size_t)kNoAllocMaxPartials * 64 * (512 + 4)];

namespace {

std::mutex g_noalloc_mu;
constexpr int kNoAllocMaxDevices = 64;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per
// device (host code cannot use the array's name as a device pointer).
dsa_status_t noalloc_scratch(void** out) {
  int dev = 0;
  DSA_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kNoAllocMaxDevices)
    return fail(DSA_ERR_UNSUPPORTED, "device %d: sparse_mla_attend_noalloc supports devices 0..%d", dev,
                kNoAllocMaxDevices - 1);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(DSA_ERR_CUDA, "cudaGetSymbolAddress(scratch) failed: %s", cudaGetErrorString(e));
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return DSA_OK;
}

}  // namespace

// =================================================================== C ABI
extern "C" {

dsa_status_t dsa_index_scores(const void* q_idx, const float* w, const void* k_idx, int64_t n_rows,
                              const int64_t* seq_row_start, int32_t B, const int32_t* q_seq,
                              const int32_t* q_pos, int32_t T, int32_t q_group, float* scores,
                              int64_t ld, void* stream) {
  NvtxRange nvtx_range("dsa_index_scores");
  dsa_status_t st = check_index_args(q_idx, w, k_idx, n_rows, seq_row_start, B, q_seq, q_pos, T,
                                     q_group, ld);
  if (st != DSA_OK) return st;
  DSA_REQUIRE(scores && aligned(scores, 16), "scores must be non-null and 16-byte aligned");
  if (T == 0) return DSA_OK;
  return indexer_impl(q_idx, w, k_idx, n_rows, seq_row_start, B, q_seq, q_pos, T, q_group, scores, ld,
                      static_cast<cudaStream_t>(stream));
}

dsa_status_t dsa_index_scores_fp8(const void* q8, const float* q_scale, const float* w, const void* k8,
                                  const float* k_scale, int64_t n_rows, const int64_t* seq_row_start,
                                  int32_t B, const int32_t* q_seq, const int32_t* q_pos, int32_t T,
                                  int32_t q_group, float* scores, int64_t ld, void* stream) {
  NvtxRange nvtx_range("dsa_index_scores_fp8");
  dsa_status_t st = check_index_args(q8, w, k8, n_rows, seq_row_start, B, q_seq, q_pos, T, q_group, ld);
  if (st != DSA_OK) return st;
  DSA_REQUIRE(q_scale && k_scale && aligned(q_scale, 4) && aligned(k_scale, 4),
              "q_scale and k_scale must be non-null and 4-byte aligned");
  DSA_REQUIRE(scores && aligned(scores, 16), "scores must be non-null and 16-byte aligned");
  if (T == 0) return DSA_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (q_group == 8)
    return launch_indexer<8, true>(q8, q_scale, w, k8, k_scale, n_rows, seq_row_start, B, q_seq, q_pos, T,
                                   scores, ld, s);
  return launch_indexer<1, true>(q8, q_scale, w, k8, k_scale, n_rows, seq_row_start, B, q_seq, q_pos, T, scores,
                                 ld, s);
}

size_t dsa_topk_workspace_size(int32_t, int64_t, int32_t) { return 0; }

dsa_status_t dsa_topk(const float* scores, int64_t ld, const int32_t* q_pos, int32_t T, int32_t k,
                      int32_t* idx, int32_t* count, void* workspace, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("dsa_topk");
  (void)workspace;
  (void)ws_bytes;
  dsa_status_t st = check_topk_args(scores, ld, q_pos, T, k, idx, count);
  if (st != DSA_OK) return st;
  if (T == 0) return DSA_OK;
  return topk_impl(scores, ld, q_pos, T, k, idx, count, static_cast<cudaStream_t>(stream));
}

size_t sparse_mla_workspace_size(int32_t T, int32_t k) {
  if (T <= 0 || k <= 0) return 0;
  return attend_ws_bytes(T, k);
}

dsa_status_t sparse_mla_attend(const void* q_nope, const void* q_pe, const float* qmul,
                               float softmax_scale, const void* cache, int64_t n_rows, int32_t ld_c,
                               int32_t d_rope, const int64_t* seq_row_start, int32_t B,
                               const int32_t* q_seq, const int32_t* idx, const int32_t* count,
                               int32_t T, int32_t k, void* out, float* lse, void* workspace,
                               size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("sparse_mla_attend");
  dsa_status_t st = check_attend_args(q_nope, q_pe, qmul, cache, n_rows, ld_c, d_rope, seq_row_start, B,
                                      q_seq, idx, count, T, k, out);
  if (st != DSA_OK) return st;
  DSA_REQUIRE(lse == nullptr || aligned(lse, 4), "misaligned lse");
  if (T == 0) return DSA_OK;
  const size_t need = attend_ws_bytes(T, k);
  if (need > 0 && (workspace == nullptr || ws_bytes < need || !aligned(workspace, 256)))
    return fail(DSA_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned (got %zu)", need, ws_bytes);
  return attend_impl(q_nope, q_pe, qmul, softmax_scale, cache, n_rows, ld_c, d_rope, seq_row_start, B,
                     q_seq, idx, count, T, k, out, lse, workspace, static_cast<cudaStream_t>(stream));
}

// Same computation as sparse_mla_attend, for callers that may not allocate:
// the split partials go to the library's fixed scratch array instead of a
// caller workspace.  Launches exactly the kernels sparse_mla_attend launches.
dsa_status_t sparse_mla_attend_noalloc(const void* q_nope, const void* q_pe, const float* qmul,
                                       float softmax_scale, const void* cache, int64_t n_rows,
                                       int32_t ld_c, int32_t d_rope, const int64_t* seq_row_start,
                                       int32_t B, const int32_t* q_seq, const int32_t* idx,
                                       const int32_t* count, int32_t T, int32_t k, void* out,
                                       float* lse, void* stream) {
  NvtxRange nvtx_range("sparse_mla_attend_noalloc");
  dsa_status_t st = check_attend_args(q_nope, q_pe, qmul, cache, n_rows, ld_c, d_rope, seq_row_start, B,
                                      q_seq, idx, count, T, k, out);
  if (st != DSA_OK) return st;
  DSA_REQUIRE(lse == nullptr || aligned(lse, 4), "misaligned lse");
  if (T == 0) return DSA_OK;
  const SplitPlan sp = attend_plan(T, k);
  void* scratch = nullptr;
  if (sp.n_split > 1 && !sp.merge) {
    const int64_t partials = (int64_t)T * sp.n_split;
    if (partials > kNoAllocMaxPartials)
      return fail(DSA_ERR_WORKSPACE,
                  "sparse_mla_attend_noalloc: %d queries split %d ways need %lld partials; its fixed "
                  "scratch holds %d (use sparse_mla_attend with a workspace, or fewer queries per call)",
                  T, sp.n_split, (long long)partials, kNoAllocMaxPartials);
    st = noalloc_scratch(&scratch);
    if (st != DSA_OK) return st;
  }
  return attend_impl(q_nope, q_pe, qmul, softmax_scale, cache, n_rows, ld_c, d_rope, seq_row_start, B,
                     q_seq, idx, count, T, k, out, lse, scratch, static_cast<cudaStream_t>(stream));
}

// Workspace of the fused call for a chunk of Tc queries:
//   [idx Tc*k i32][count Tc i32][attention partials][scores Tc*ld f32]
static size_t forward_chunk_bytes(int32_t Tc, int64_t ld, int32_t k, bool own_idx, bool own_count) {
  size_t b = 0;
  if (own_idx) b += round_up((size_t)Tc * k * 4, 256);
  if (own_count) b += round_up((size_t)Tc * 4, 256);
  b += attend_ws_bytes(Tc, k);
  b += round_up((size_t)Tc * ld * 4, 256);
  return b;
}

size_t dsa_forward_workspace_size(int32_t T, int64_t ld, int32_t k, int32_t q_group) {
  (void)q_group;
  if (T <= 0 || ld <= 0 || k <= 0) return 0;
  return forward_chunk_bytes(T, ld, k, true, true);
}

dsa_status_t dsa_sparse_mla_forward(const void* q_idx, const float* w, const void* k_idx, int64_t n_rows,
                                    const int64_t* seq_row_start, int32_t B, const int32_t* q_seq,
                                    const int32_t* q_pos, int32_t T, int32_t q_group, int64_t ld,
                                    int32_t n_layers, const dsa_layer_args* layers,
                                    float softmax_scale, int32_t k, int32_t* idx_out,
                                    int32_t* count_out, void* workspace, size_t ws_bytes,
                                    void* stream) {
  NvtxRange nvtx_range("dsa_sparse_mla_forward");
  dsa_status_t st = check_index_args(q_idx, w, k_idx, n_rows, seq_row_start, B, q_seq, q_pos, T,
                                     q_group, ld);
  if (st != DSA_OK) return st;
  DSA_REQUIRE(k >= 1 && k <= kMaxK, "k must be in [1, %d]", kMaxK);
  DSA_REQUIRE(n_layers >= 0 && (n_layers == 0 || layers != nullptr), "bad layer list");
  DSA_REQUIRE(idx_out == nullptr || aligned(idx_out, 4), "misaligned idx_out");
  DSA_REQUIRE(count_out == nullptr || aligned(count_out, 4), "misaligned count_out");
  for (int l = 0; l < n_layers; ++l) {
    const dsa_layer_args& L = layers[l];
    st = check_attend_args(L.q_nope, L.q_pe, L.qmul, L.cache, n_rows, L.ld_c, L.d_rope, seq_row_start,
                           B, q_seq, q_seq /* idx checked below */, q_pos, T, k, L.out);
    if (st != DSA_OK) return fail(st, "layer %d: %s", l, g_last_error.c_str());
    DSA_REQUIRE(L.lse == nullptr || aligned(L.lse, 4), "layer %d: misaligned lse", l);
  }
  if (T == 0) return DSA_OK;
  DSA_REQUIRE(workspace != nullptr && aligned(workspace, 256), "workspace must be non-null and 256-byte aligned");
  const bool own_idx = idx_out == nullptr, own_count = count_out == nullptr;
  // Largest chunk (a multiple of q_group) whose working set fits the workspace.
  int32_t Tc = T;
  while (Tc > q_group && forward_chunk_bytes(Tc, ld, k, own_idx, own_count) > ws_bytes)
    Tc = std::max<int32_t>(q_group, (Tc / 2 + q_group - 1) / q_group * q_group);
  if (forward_chunk_bytes(Tc, ld, k, own_idx, own_count) > ws_bytes)
    return fail(DSA_ERR_WORKSPACE, "workspace of %zu bytes is too small (need %zu for %d queries)", ws_bytes,
                forward_chunk_bytes(Tc, ld, k, own_idx, own_count), Tc);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* idx_ws = nullptr;
  int32_t* cnt_ws = nullptr;
  size_t off = 0;
  if (own_idx) {
    idx_ws = reinterpret_cast<int32_t*>(ws + off);
    off += round_up((size_t)Tc * k * 4, 256);
  }
  if (own_count) {
    cnt_ws = reinterpret_cast<int32_t*>(ws + off);
    off += round_up((size_t)Tc * 4, 256);
  }
  void* att_ws = ws + off;
  off += attend_ws_bytes(Tc, k);
  float* scores = reinterpret_cast<float*>(ws + off);

  for (int32_t t0 = 0; t0 < T; t0 += Tc) {
    const int32_t n = std::min(Tc, T - t0);
    int32_t* idx_c = own_idx ? idx_ws : idx_out + (int64_t)t0 * k;
    int32_t* cnt_c = own_count ? cnt_ws : count_out + t0;
    st = indexer_impl(static_cast<const __nv_bfloat16*>(q_idx) + (int64_t)t0 * dsa::kIdxHeads * dsa::kIdxDim,
                      w + (int64_t)t0 * dsa::kIdxHeads, k_idx, n_rows, seq_row_start, B, q_seq + t0,
                      q_pos + t0, n, q_group, scores, ld, s);
    if (st != DSA_OK) return st;
    st = topk_impl(scores, ld, q_pos + t0, n, k, idx_c, cnt_c, s);
    if (st != DSA_OK) return st;
    for (int l = 0; l < n_layers; ++l) {
      const dsa_layer_args& L = layers[l];
      const int64_t qo = (int64_t)t0 * dsa::kHeads;
      st = attend_impl(static_cast<const __nv_bfloat16*>(L.q_nope) + qo * dsa::kLatent,
                       L.q_pe ? static_cast<const __nv_bfloat16*>(L.q_pe) + qo * 64 : nullptr,
                       L.qmul + qo, softmax_scale, L.cache, n_rows, L.ld_c, L.d_rope, seq_row_start, B,
                       q_seq + t0, idx_c, cnt_c, n, k,
                       static_cast<__nv_bfloat16*>(L.out) + qo * dsa::kLatent,
                       L.lse ? L.lse + qo : nullptr, att_ws, s);
      if (st != DSA_OK) return st;
    }
  }
  return DSA_OK;
}

dsa_status_t dsa_check_errors(void* stream, uint32_t* bits) {
  DSA_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  unsigned int word = 0;
  DSA_CUDA(cudaMemcpyFromSymbol(&word, dsa::g_dev_error, sizeof(word)));
  if (bits) *bits = word;
  if (word == 0) return DSA_OK;
  const unsigned int zero = 0;
  DSA_CUDA(cudaMemcpyToSymbol(dsa::g_dev_error, &zero, sizeof(zero)));
  if (word & dsa::kErrTimeout) return fail(DSA_ERR_TIMEOUT, "device wait timed out (error word 0x%x)", word);
  return fail(DSA_ERR_DEVICE_CHECK, "device-side check failed (error word 0x%x)", word);
}

uint64_t dsa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* dsa_last_error(void) { return g_last_error.c_str(); }

int32_t dsa_version(void) { return 100; }

}  // extern "C"
