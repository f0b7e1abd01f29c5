// dsa_api.cu - host side of the C ABI declared in include/dsa.h: argument
// validation, TMA descriptor encoding, launch planning and configuration, and
// the fused indexer -> top-k -> per-layer attention sequence.  Every step of
// the hot path runs in the kernels included below; nothing here computes on
// the host.
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
#include "plan.h"
#include "topk.cuh"

static_assert(dsa::kPlanMaxLayers == dsa::kMaxAttLayers, "planner and kernel agree on layers per launch");
static_assert(dsa::kPlanMaxSplits == dsa::kMaxSplits, "planner and kernel agree on the split limit");
static_assert(dsa::kPlanTileRows == dsa::AttCfg::ROWS, "planner and kernel agree on the tile height");
static_assert(dsa::kPlanTopkCap == dsa::kTopkCandCap && dsa::kPlanTopkBins == dsa::kTopkBins,
              "planner and top-k kernels agree on the candidate lists");

namespace {

thread_local std::string g_last_error;
std::atomic<uint64_t> g_launches{0};
std::atomic<uint64_t> g_wait_limit_ns{0};   // 0: kWaitLimitNs (testing hook)
std::atomic<int32_t> g_stall_tile{-1};      // testing hook, off

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

#define DSA_TRY(...)                       \
  do {                                     \
    dsa_status_t st_ = (__VA_ARGS__);      \
    if (st_ != DSA_OK) return st_;         \
  } while (0)

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

constexpr int kMaxK = 16384;

// ----------------------------------------------------------------- driver entry points
template <typename Fn>
Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) == cudaSuccess && q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<Fn>(p);
  return nullptr;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static const auto fn = driver_fn<PFN_cuTensorMapEncodeTiled_v12000>("cuTensorMapEncodeTiled");
  return fn;
}

// Unique id of the calling thread's current context (0: none is current yet).
// Per-device state is keyed by it, so a device reset (a new primary context)
// starts from a clean slate instead of reusing addresses and attributes of the
// old context.
uint64_t current_context_id() {
  static const auto get_cur = driver_fn<PFN_cuCtxGetCurrent_v4000>("cuCtxGetCurrent");
  static const auto get_id = driver_fn<PFN_cuCtxGetId_v12000>("cuCtxGetId");
  if (get_cur == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  if (get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return (uint64_t)id + 1;   // never 0 for a real context
}

// ----------------------------------------------------------------- per-device state
static_assert(dsa::kTopkRowCap == dsa::kPlanTopkRowCap, "planner and kernel agree on the shared-memory row path");

enum KernelId : uint32_t {
  kKIdx1 = 0, kKIdx4, kKIdx8, kKIdx1F8, kKIdx4F8, kKIdx8F8, kKTopk1, kKTopk2, kKTopk4, kKTopk8, kKTopk16, kKAttend, kKAttend8, kKTopkRow, kKTopkFilter,
  kKTopkSelect, kKTopkMerge, kKCount
};

constexpr int kMaxDevices = 64;

struct DevState {
  std::mutex mu;
  uint64_t ctx_id = ~0ull;        // context the cached values belong to
  bool props_ok = false;
  dsa::DevProps props;            // SMs and attention cluster residency
  int topk_clusters[17] = {};     // [CL]: top-k clusters of CL blocks resident at once
  uint32_t smem_done = 0;         // bit per KernelId: dynamic shared-memory limit raised
  void* noalloc_ptr = nullptr;    // device address of the no-allocation scratch array
};
DevState g_dev[kMaxDevices];

// The calling thread's device state, locked, reset when its context changed.
struct DevLock {
  DevState* s = nullptr;
  int dev = 0;
  std::unique_lock<std::mutex> lk;
};

dsa_status_t lock_device(DevLock& L) {
  DSA_CUDA(cudaGetDevice(&L.dev));
  if (L.dev < 0 || L.dev >= kMaxDevices)
    return fail(DSA_ERR_UNSUPPORTED, "device %d: this library supports devices 0..%d", L.dev, kMaxDevices - 1);
  L.s = &g_dev[L.dev];
  L.lk = std::unique_lock<std::mutex>(L.s->mu);
  const uint64_t id = current_context_id();
  if (L.s->ctx_id != id) {
    L.s->ctx_id = id;
    L.s->props_ok = false;
    L.s->smem_done = 0;
    L.s->noalloc_ptr = nullptr;
  }
  return DSA_OK;
}

// Raises a kernel's dynamic shared-memory limit once per device and context.
template <typename K>
dsa_status_t set_smem(DevState& s, KernelId id, K kernel, int bytes) {
  if (s.smem_done & (1u << id)) return DSA_OK;
  DSA_CUDA(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  s.smem_done |= 1u << id;
  return DSA_OK;
}

template <typename K>
int max_active_clusters(K kernel, int threads, int smem, int cl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cl);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) n = 0;
  cudaGetLastError();
  return n;
}

// SM count and how many clusters of each size the attention and top-k kernels
// can keep resident (a cluster must sit inside one GPC, so this can be well
// below SMs / size).  Queried once per device and context.
dsa_status_t device_props(DevLock& L, dsa::DevProps* out) {
  DevState& s = *L.s;
  if (!s.props_ok) {
    dsa::DevProps d;
    int n = 0;
    DSA_CUDA(cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, L.dev));
    d.sms = n > 0 ? n : 1;
    // (the FP8-cache variant has the same block size and shared memory, so the same residency)
    DSA_TRY(set_smem(s, kKAttend, dsa::attend_kernel<false>, dsa::AttCfg::SMEM_BYTES));
    for (int c = 2; c <= dsa::kPlanMaxMerge; ++c)
      d.max_clusters[c] =
          max_active_clusters(dsa::attend_kernel<false>, dsa::AttCfg::THREADS, dsa::AttCfg::SMEM_BYTES, c);
    DSA_TRY(set_smem(s, kKTopk2, dsa::topk_kernel<2>, dsa::kTopkSmemBytes));
    DSA_TRY(set_smem(s, kKTopk4, dsa::topk_kernel<4>, dsa::kTopkSmemBytes));
    DSA_TRY(set_smem(s, kKTopk8, dsa::topk_kernel<8>, dsa::kTopkSmemBytes));
    DSA_TRY(set_smem(s, kKTopk16, dsa::topk_kernel<16>, dsa::kTopkSmemBytes));
    DSA_CUDA(cudaFuncSetAttribute(dsa::topk_kernel<16>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
    s.topk_clusters[1] = d.sms;
    s.topk_clusters[2] = max_active_clusters(dsa::topk_kernel<2>, dsa::kTopkThreads, dsa::kTopkSmemBytes, 2);
    s.topk_clusters[4] = max_active_clusters(dsa::topk_kernel<4>, dsa::kTopkThreads, dsa::kTopkSmemBytes, 4);
    s.topk_clusters[8] = max_active_clusters(dsa::topk_kernel<8>, dsa::kTopkThreads, dsa::kTopkSmemBytes, 8);
    s.topk_clusters[16] = max_active_clusters(dsa::topk_kernel<16>, dsa::kTopkThreads, dsa::kTopkSmemBytes, 16);
    s.props = d;
    s.props_ok = true;
  }
  *out = s.props;
  return DSA_OK;
}

// Props for a planning query: the caller's (on any machine) or the current device's.
dsa_status_t props_for_query(const dsa_device_props* given, dsa::DevProps* out) {
  if (given != nullptr) {
    DSA_REQUIRE(given->sms >= 1, "props.sms must be >= 1");
    dsa::DevProps d;
    d.sms = given->sms;
    for (int c = 0; c < 9; ++c) d.max_clusters[c] = std::max(0, given->max_clusters[c]);
    *out = d;
    return DSA_OK;
  }
  DevLock L;
  DSA_TRY(lock_device(L));
  return device_props(L, out);
}

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
dsa_status_t launch_ex(bool pdl, void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem,
                       cudaStream_t stream, unsigned cl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (pdl) {
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

template <typename... KArgs, typename... Args>
dsa_status_t launch(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t stream,
                    unsigned cl, Args&&... args) {
  return launch_ex(pdl_enabled(), kernel, grid, block, smem, stream, cl, std::forward<Args>(args)...);
}

// ----------------------------------------------------------------- indexer
// F8: q_idx / k_idx hold E4M3 codes (one byte per value) and q_scale / k_scale
// their per-head / per-row scales; otherwise bf16 values and null scales.
template <int QG, bool F8>
dsa_status_t launch_indexer(DevLock& L, const void* q_idx, const float* q_scale, const float* w, const void* k_idx,
                            const float* k_scale, int64_t n_rows, const int64_t* seq_row_start, int32_t B,
                            const int32_t* q_seq, const int32_t* q_pos, int32_t T, float* scores, int64_t ld,
                            uint32_t* hist, cudaStream_t stream) {
  using C = dsa::IdxCfg<QG, F8>;
  // One 128-byte swizzled block per box row: 64 bf16 or 128 fp8 values.  TMA
  // moves bytes, so an fp8 row (128 B) is described as 64 two-byte elements:
  // the same bytes and the same swizzle as a bf16 half row.
  const uint64_t row_elems = F8 ? dsa::kIdxDim / 2 : dsa::kIdxDim;
  const uint64_t row_bytes = F8 ? dsa::kIdxDim : dsa::kIdxDim * 2;
  CUtensorMap kmap, qmap;
  DSA_TRY(make_tmap(&kmap, k_idx, row_elems, (uint64_t)n_rows, row_bytes, 64, dsa::kKeyTile));
  DSA_TRY(make_tmap(&qmap, q_idx, row_elems, (uint64_t)T * dsa::kIdxHeads, row_bytes, 64, C::N));
  dsa::IndexerParams p;
  p.w = w;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.seq_row_start = seq_row_start;
  p.q_seq = q_seq;
  p.q_pos = q_pos;
  p.scores = scores;
  p.hist = (QG == 1) ? hist : nullptr;
  p.ld = ld;
  p.n_rows = n_rows;
  p.T = T;
  p.B = B;
  p.n_kt = (int32_t)((ld + dsa::kKeyTile - 1) / dsa::kKeyTile);
  if (p.hist != nullptr) DSA_CUDA(cudaMemsetAsync(hist, 0, (size_t)T * dsa::kTopkBins * 4, stream));
  const int64_t n_groups = (T + QG - 1) / QG;
  p.n_units = n_groups * p.n_kt;
  dsa::DevProps props;
  DSA_TRY(device_props(L, &props));
  const int grid = (int)std::min<int64_t>(p.n_units, props.sms);
  const KernelId id = F8 ? (QG == 8 ? kKIdx8F8 : (QG == 4 ? kKIdx4F8 : kKIdx1F8))
                          : (QG == 8 ? kKIdx8 : (QG == 4 ? kKIdx4 : kKIdx1));
  DSA_TRY(set_smem(*L.s, id, dsa::indexer_kernel<QG, F8>, C::SMEM_BYTES));
  return launch(dsa::indexer_kernel<QG, F8>, (unsigned)grid, C::THREADS, C::SMEM_BYTES, stream, 1, kmap, qmap,
                p);
}

dsa_status_t indexer_impl(DevLock& L, const void* q_idx, const float* w, const void* k_idx, int64_t n_rows,
                          const int64_t* seq_row_start, int32_t B, const int32_t* q_seq,
                          const int32_t* q_pos, int32_t T, int32_t q_group, float* scores,
                          int64_t ld, uint32_t* hist, cudaStream_t stream) {
  if (q_group == 8)
    return launch_indexer<8, false>(L, q_idx, nullptr, w, k_idx, nullptr, n_rows, seq_row_start, B, q_seq, q_pos,
                                    T, scores, ld, nullptr, stream);
  if (q_group == 4)
    return launch_indexer<4, false>(L, q_idx, nullptr, w, k_idx, nullptr, n_rows, seq_row_start, B, q_seq, q_pos,
                                    T, scores, ld, nullptr, stream);
  return launch_indexer<1, false>(L, q_idx, nullptr, w, k_idx, nullptr, n_rows, seq_row_start, B, q_seq, q_pos, T,
                                  scores, ld, hist, stream);
}

// ----------------------------------------------------------------- top-k
template <int CL>
dsa_status_t launch_topk_cl(DevLock& L, KernelId id, const dsa::TopkParams& p, cudaStream_t stream) {
  DSA_TRY(set_smem(*L.s, id, dsa::topk_kernel<CL>, dsa::kTopkSmemBytes));
  return launch(dsa::topk_kernel<CL>, (unsigned)(p.T * CL), dsa::kTopkThreads, dsa::kTopkSmemBytes, stream,
                (unsigned)CL, p);
}

// CTAs per query: enough that each CTA owns at least ~16K candidates' worth of
// work while the batch stays within one wave (T x CL <= SMs, every cluster
// resident at once); more (up to 16) when a query's slice would not fit the
// shared-memory key stash.
int topk_cluster_size(const DevState& s, int sms, int32_t T, int64_t ld) {
  auto fits = [&](int c) { return (int64_t)T * c <= sms && T <= s.topk_clusters[c]; };
  int cl = 1;
  while (cl < 8 && (ld + cl - 1) / cl > 16384 && fits(cl * 2)) cl *= 2;
  while (cl < 16 && (ld + cl - 1) / cl > dsa::kTopkStashCap && fits(cl * 2)) cl *= 2;
  return cl;
}

dsa_status_t topk_impl(DevLock& L, const float* scores, int64_t ld, const int32_t* q_pos, int32_t T, int32_t k,
                       int32_t* idx, int32_t* count, const uint32_t* hist, void* ws, size_t ws_bytes,
                       cudaStream_t stream) {
  dsa::DevProps props;
  DSA_TRY(device_props(L, &props));
  dsa::TopkParams p;
  p.scores = scores;
  p.q_pos = q_pos;
  p.idx = idx;
  p.count = count;
  p.ld = ld;
  p.T = T;
  p.k = k;
  if (hist != nullptr && ld <= dsa::kTopkRowCap) {
    // first pass from the indexer's histogram; the whole row in one CTA's shared memory
    dsa::TopkHistParams hp;
    std::memset(&hp, 0, sizeof(hp));
    hp.base = p;
    hp.hist = hist;
    DSA_TRY(set_smem(*L.s, kKTopkRow, dsa::topk_row_kernel, dsa::kTopkRowSmemBytes));
    return launch(dsa::topk_row_kernel, (unsigned)T, dsa::kTopkThreads, dsa::kTopkRowSmemBytes, stream, 1, hp);
  }
  if (hist != nullptr) {
    // first pass from the indexer's histogram: slices on every SM, then one CTA per query
    const int S = dsa::topk_slices(props.sms, T, ld);
    const size_t need = dsa::topk_hist_ws_bytes(props.sms, T, ld);
    if (ws == nullptr || ws_bytes < need || !aligned(ws, 256))
      return fail(DSA_ERR_WORKSPACE, "top-k with a histogram needs %zu bytes of 256-byte aligned workspace (got %zu)",
                  need, ws_bytes);
    const size_t ts = (size_t)T * S;
    const size_t lists = dsa::plan_round_up(ts * dsa::kTopkCandCap * 4, 256);
    dsa::TopkHistParams hp;
    hp.base = p;
    hp.hist = hist;
    hp.cand_key = static_cast<uint32_t*>(ws);
    hp.cand_pos = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + lists);
    hp.cand_cnt = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + 2 * lists);
    hp.bin_info = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + 2 * lists + dsa::plan_round_up(ts * 4, 256));
    hp.S = S;
    DSA_TRY(set_smem(*L.s, kKTopkFilter, dsa::topk_filter_kernel, dsa::kTopkSmemBytes));
    DSA_TRY(set_smem(*L.s, kKTopkSelect, dsa::topk_select_kernel, dsa::kTopkSmemBytes));
    DSA_TRY(launch(dsa::topk_filter_kernel, (unsigned)(T * S), dsa::kTopkThreads, dsa::kTopkSmemBytes, stream, 1,
                   hp));
    // programmatic dependent launch: the select CTAs are scheduled as the filter's
    // blocks retire and wait (griddepcontrol.wait) for all of its writes
    return launch_ex(true, dsa::topk_select_kernel, (unsigned)T, dsa::kTopkThreads, dsa::kTopkSmemBytes, stream, 1,
                     hp);
  }
  switch (topk_cluster_size(*L.s, props.sms, T, ld)) {
    case 1: return launch_topk_cl<1>(L, kKTopk1, p, stream);
    case 2: return launch_topk_cl<2>(L, kKTopk2, p, stream);
    case 4: return launch_topk_cl<4>(L, kKTopk4, p, stream);
    case 8: return launch_topk_cl<8>(L, kKTopk8, p, stream);
    default: return launch_topk_cl<16>(L, kKTopk16, p, stream);   // chosen only when its clusters fit
  }
}

// ----------------------------------------------------------------- attention
// One launch over up to kMaxAttLayers layers sharing one selection (grid =
// layers x queries x splits), plus the combine kernel when the plan writes
// partials.  `ws` must hold the plan's partials (checked).
dsa_status_t launch_attend(DevLock& L, const dsa_layer_args* layers, int32_t n_layers, float scale,
                           int64_t n_rows, const int64_t* seq_row_start, int32_t B, const int32_t* q_seq,
                           const int32_t* q_pos, const int32_t* idx, const int32_t* count, int32_t T, int32_t k,
                           void* ws, size_t ws_bytes, cudaStream_t stream, bool allow_partials = true,
                           bool q_early = false) {
  using C = dsa::AttCfg;
  dsa::DevProps props;
  DSA_TRY(device_props(L, &props));
  const int64_t units = (int64_t)T * n_layers;
  const dsa::SplitPlan sp = dsa::attend_plan(props, units, k, allow_partials);
  dsa::AttendParams p;
  std::memset(&p, 0, sizeof(p));
  for (int l = 0; l < n_layers; ++l) {
    const dsa_layer_args& a = layers[l];
    p.layer[l].q_nope = static_cast<const __nv_bfloat16*>(a.q_nope);
    p.layer[l].q_pe = static_cast<const __nv_bfloat16*>(a.q_pe);
    p.layer[l].qmul = a.qmul;
    p.layer[l].cache = static_cast<const __nv_bfloat16*>(a.cache);
    p.layer[l].out = static_cast<__nv_bfloat16*>(a.out);
    p.layer[l].lse = a.lse;
    p.layer[l].ld_c = a.ld_c;
    p.layer[l].d_rope = a.d_rope;
    p.layer[l].out_f32 = a.out_f32 ? 1 : 0;
  }
  p.seq_row_start = seq_row_start;
  p.q_seq = q_seq;
  p.q_pos = q_pos;
  p.idx = idx;
  p.count = count;
  p.n_rows = n_rows;
  const uint64_t lim = g_wait_limit_ns.load(std::memory_order_relaxed);
  p.wait_limit_ns = lim ? lim : dsa::kWaitLimitNs;
  p.stall_tile = g_stall_tile.load(std::memory_order_relaxed);
  p.scale_log2e = scale * 1.4426950408889634f;
  p.n_layers = n_layers;
  p.B = B;
  p.T = T;
  p.k = k;
  p.n_split = sp.n_split;
  p.rows_per_split = sp.rows_per_split;
  p.merge = sp.merge ? 1 : 0;
  p.q_early = q_early ? 1 : 0;
  const bool partials = sp.n_split > 1 && !sp.merge;
  if (partials) {
    const size_t need = dsa::partial_bytes(units, sp.n_split);
    if (ws == nullptr || ws_bytes < need || !aligned(ws, 256))
      return fail(DSA_ERR_WORKSPACE, "attention partials need %zu bytes of 256-byte aligned workspace (got %zu)",
                  need, ws_bytes);
    p.ws_o = static_cast<float*>(ws);
    p.ws_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + dsa::partial_stats_offset(units, sp.n_split));
  }
  const unsigned grid = (unsigned)(units * sp.n_split);
  const unsigned cluster = sp.merge ? (unsigned)sp.n_split : 1u;
  // programmatic dependent launch: the CTAs may be scheduled while the previous kernel (the top-k)
  // still runs on other SMs; they set up and then wait (griddepcontrol.wait) before reading memory
  if (layers[0].cache_fp8) {   // every layer of a call has the same cache format (checked)
    DSA_TRY(set_smem(*L.s, kKAttend8, dsa::attend_kernel<true>, C::SMEM_BYTES));
    DSA_TRY(launch_ex(true, dsa::attend_kernel<true>, grid, C::THREADS, C::SMEM_BYTES, stream, cluster, p));
  } else {
    DSA_TRY(set_smem(*L.s, kKAttend, dsa::attend_kernel<false>, C::SMEM_BYTES));
    DSA_TRY(launch_ex(true, dsa::attend_kernel<false>, grid, C::THREADS, C::SMEM_BYTES, stream, cluster, p));
  }
  if (!partials) return DSA_OK;
  // programmatic dependent launch: scheduled while the attention drains, waits for its writes
  return launch_ex(true, dsa::attend_combine_kernel, (unsigned)(units * dsa::kHeads), 128, 0, stream, 1, p);
}

// Several layers over one selection: launches of up to kMaxAttLayers layers
// each, in order on the stream (they reuse the same partials region).
dsa_status_t attend_layers_impl(DevLock& L, const dsa_layer_args* layers, int32_t n_layers, float scale,
                                int64_t n_rows, const int64_t* seq_row_start, int32_t B, const int32_t* q_seq,
                                const int32_t* q_pos, const int32_t* idx, const int32_t* count, int32_t T,
                                int32_t k, int64_t q_offset, void* ws, size_t ws_bytes, cudaStream_t stream,
                                bool allow_partials = true, bool q_early = false) {
  for (int l0 = 0; l0 < n_layers; l0 += dsa::kMaxAttLayers) {
    const int g = std::min(dsa::kMaxAttLayers, n_layers - l0);
    dsa_layer_args sub[dsa::kMaxAttLayers];
    const int64_t qo = q_offset * dsa::kHeads;
    for (int i = 0; i < g; ++i) {
      const dsa_layer_args& a = layers[l0 + i];
      sub[i] = a;
      sub[i].q_nope = static_cast<const __nv_bfloat16*>(a.q_nope) + qo * dsa::kLatent;
      sub[i].q_pe = a.q_pe ? static_cast<const __nv_bfloat16*>(a.q_pe) + qo * 64 : nullptr;
      sub[i].qmul = a.qmul + qo;
      sub[i].out = a.out_f32 ? static_cast<void*>(static_cast<float*>(a.out) + qo * dsa::kLatent)
                             : static_cast<void*>(static_cast<__nv_bfloat16*>(a.out) + qo * dsa::kLatent);
      sub[i].lse = a.lse ? a.lse + qo : nullptr;
    }
    DSA_TRY(launch_attend(L, sub, g, scale, n_rows, seq_row_start, B, q_seq, q_pos, idx, count, T, k, ws,
                          ws_bytes, stream, allow_partials, q_early));
  }
  return DSA_OK;
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
  DSA_REQUIRE(q_group == 1 || q_group == 4 || q_group == 8, "q_group must be 1, 4 or 8");
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

// One layer's arguments (q_nope, q_pe, qmul, cache, ld_c, d_rope, out, lse).
dsa_status_t check_layer_args(const dsa_layer_args& a, int64_t n_rows) {
  DSA_REQUIRE(a.d_rope == 0 || a.d_rope == 64, "d_rope must be 0 or 64 (got %d)", a.d_rope);
  DSA_REQUIRE(a.q_nope && a.qmul && a.cache && a.out, "null pointer argument");
  DSA_REQUIRE(a.out_f32 == 0 || a.out_f32 == 1, "out_f32 must be 0 or 1");
  DSA_REQUIRE((a.q_pe != nullptr) == (a.d_rope == 64), "q_pe must be given iff d_rope == 64");
  DSA_REQUIRE(aligned(a.q_nope, 16) && aligned(a.cache, 16) && aligned(a.out, 16) &&
                  (a.q_pe == nullptr || aligned(a.q_pe, 16)),
              "q_nope, q_pe, cache and out must be 16-byte aligned");
  DSA_REQUIRE(aligned(a.qmul, 4) && (a.lse == nullptr || aligned(a.lse, 4)), "misaligned qmul / lse");
  DSA_REQUIRE(a.cache_fp8 == 0 || a.cache_fp8 == 1, "cache_fp8 must be 0 or 1");
  if (a.cache_fp8) {
    const int32_t need = dsa::kLatent + a.d_rope + 4 * (dsa::kLatent / 128 + (a.d_rope ? 1 : 0));
    DSA_REQUIRE(a.ld_c >= need && a.ld_c % 16 == 0,
                "FP8 cache rows: ld_c (bytes) must be >= %d and a multiple of 16 (got %d)", need, a.ld_c);
  } else {
    DSA_REQUIRE(a.ld_c >= dsa::kLatent + a.d_rope && a.ld_c % 8 == 0,
                "ld_c must be >= 512 + d_rope and a multiple of 8");
  }
  DSA_REQUIRE(n_rows * (int64_t)a.ld_c < (int64_t(1) << 62), "cache too large");
  return DSA_OK;
}

dsa_status_t check_attend_common(int64_t n_rows, const int64_t* seq_row_start, int32_t B, const int32_t* q_seq,
                                 const int32_t* q_pos, const int32_t* idx, const int32_t* count, int32_t T,
                                 int32_t k) {
  DSA_REQUIRE(T >= 0, "T must be >= 0");
  DSA_REQUIRE(seq_row_start && q_seq && idx && count, "null pointer argument");
  DSA_REQUIRE(aligned(idx, 4) && aligned(count, 4) && aligned(q_seq, 4) && aligned(seq_row_start, 8) &&
                  (q_pos == nullptr || aligned(q_pos, 4)),
              "misaligned idx/count/q_seq/q_pos/seq_row_start");
  DSA_REQUIRE(n_rows >= 1 && n_rows < (int64_t(1) << 31), "n_rows must be in [1, 2^31)");
  DSA_REQUIRE(B >= 1, "B must be >= 1");
  DSA_REQUIRE(k >= 1 && k <= kMaxK, "k must be in [1, %d]", kMaxK);
  DSA_REQUIRE((int64_t)T * dsa::kHeads < (int64_t(1) << 31), "T too large");
  return DSA_OK;
}

dsa_layer_args one_layer(const void* q_nope, const void* q_pe, const float* qmul, const void* cache, int32_t ld_c,
                         int32_t d_rope, void* out, float* lse) {
  dsa_layer_args a;
  a.q_nope = q_nope;
  a.q_pe = q_pe;
  a.qmul = qmul;
  a.cache = cache;
  a.ld_c = ld_c;
  a.d_rope = d_rope;
  a.out = out;
  a.lse = lse;
  a.out_f32 = 0;
  a.cache_fp8 = 0;
  return a;
}

void fill_attend_plan(const dsa::DevProps& d, int64_t units, int32_t k, bool allow_partials,
                      dsa_attend_plan* out) {
  const dsa::SplitPlan sp = dsa::attend_plan(d, units, k, allow_partials);
  out->n_split = sp.n_split;
  out->rows_per_split = sp.rows_per_split;
  out->merge = sp.merge ? 1 : 0;
  out->reserved = 0;
  out->workspace_bytes = (sp.n_split > 1 && !sp.merge) ? dsa::partial_bytes(units, sp.n_split) : 0;
}

}  // namespace

// =================================================================== no-allocation variant
// Scratch for sparse_mla_attend_noalloc: the split partials (numerators, then
// four statistics per head) of at most kNoAllocMaxPartials (query, split) work
// units, in the layout launch_attend expects of a workspace.  Every GPU that
// loads this library holds the array until the process exits.
constexpr int kNoAllocMaxPartials = DSA_NOALLOC_MAX_PARTIALS;
constexpr size_t kNoAllocBytes = (size_t)kNoAllocMaxPartials * 64 * (512 + 4) * 4;
static __device__ __align__(256) float g_noalloc_scratch[(size_t)kNoAllocMaxPartials * 64 * (512 + 4)];
static_assert(dsa::kPlanHeads == 64 && dsa::kPlanLatent == 512, "scratch layout");

namespace {

// Device address of the scratch array in the current context, looked up once
// per device and context (host code cannot use the array's name as a device
// pointer: there it is a host-side stand-in).
dsa_status_t noalloc_scratch(DevLock& L, void** out) {
  if (L.s->noalloc_ptr == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(DSA_ERR_CUDA, "cudaGetSymbolAddress(scratch) failed: %s", cudaGetErrorString(e));
    L.s->noalloc_ptr = p;
  }
  *out = L.s->noalloc_ptr;
  return DSA_OK;
}

}  // namespace

// =================================================================== C ABI
extern "C" {

dsa_status_t dsa_index_scores(const void* q_idx, const float* w, const void* k_idx, int64_t n_rows,
                              const int64_t* seq_row_start, int32_t B, const int32_t* q_seq,
                              const int32_t* q_pos, int32_t T, int32_t q_group, float* scores,
                              int64_t ld, uint32_t* hist, void* stream) {
  NvtxRange nvtx_range("dsa_index_scores");
  DSA_TRY(check_index_args(q_idx, w, k_idx, n_rows, seq_row_start, B, q_seq, q_pos, T, q_group, ld));
  DSA_REQUIRE(scores && aligned(scores, 16), "scores must be non-null and 16-byte aligned");
  DSA_REQUIRE(hist == nullptr || (q_group == 1 && aligned(hist, 16)), "hist needs q_group 1 and 16-byte alignment");
  if (T == 0) return DSA_OK;
  DevLock L;
  DSA_TRY(lock_device(L));
  return indexer_impl(L, q_idx, w, k_idx, n_rows, seq_row_start, B, q_seq, q_pos, T, q_group, scores, ld, hist,
                      static_cast<cudaStream_t>(stream));
}

dsa_status_t dsa_index_scores_fp8(const void* q8, const float* q_scale, const float* w, const void* k8,
                                  const float* k_scale, int64_t n_rows, const int64_t* seq_row_start,
                                  int32_t B, const int32_t* q_seq, const int32_t* q_pos, int32_t T,
                                  int32_t q_group, float* scores, int64_t ld, uint32_t* hist, void* stream) {
  NvtxRange nvtx_range("dsa_index_scores_fp8");
  DSA_TRY(check_index_args(q8, w, k8, n_rows, seq_row_start, B, q_seq, q_pos, T, q_group, ld));
  DSA_REQUIRE(q_scale && k_scale && aligned(q_scale, 4) && aligned(k_scale, 4),
              "q_scale and k_scale must be non-null and 4-byte aligned");
  DSA_REQUIRE(scores && aligned(scores, 16), "scores must be non-null and 16-byte aligned");
  DSA_REQUIRE(hist == nullptr || (q_group == 1 && aligned(hist, 16)), "hist needs q_group 1 and 16-byte alignment");
  if (T == 0) return DSA_OK;
  DevLock L;
  DSA_TRY(lock_device(L));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (q_group == 8)
    return launch_indexer<8, true>(L, q8, q_scale, w, k8, k_scale, n_rows, seq_row_start, B, q_seq, q_pos, T,
                                   scores, ld, nullptr, s);
  if (q_group == 4)
    return launch_indexer<4, true>(L, q8, q_scale, w, k8, k_scale, n_rows, seq_row_start, B, q_seq, q_pos, T,
                                   scores, ld, nullptr, s);
  return launch_indexer<1, true>(L, q8, q_scale, w, k8, k_scale, n_rows, seq_row_start, B, q_seq, q_pos, T, scores,
                                 ld, hist, s);
}

size_t dsa_topk_workspace_size(int32_t T, int64_t ld, int32_t k) {
  if (T <= 0 || ld <= 0 || k <= 0) return 0;
  dsa::DevProps d;
  if (props_for_query(nullptr, &d) != DSA_OK) return 0;
  return dsa::topk_hist_ws_bytes(d.sms, T, ld);
}

dsa_status_t dsa_topk(const float* scores, int64_t ld, const int32_t* q_pos, int32_t T, int32_t k,
                      int32_t* idx, int32_t* count, const uint32_t* hist, void* workspace, size_t ws_bytes,
                      void* stream) {
  NvtxRange nvtx_range("dsa_topk");
  DSA_TRY(check_topk_args(scores, ld, q_pos, T, k, idx, count));
  DSA_REQUIRE(hist == nullptr || aligned(hist, 16), "hist must be 16-byte aligned");
  if (T == 0) return DSA_OK;
  DevLock L;
  DSA_TRY(lock_device(L));
  return topk_impl(L, scores, ld, q_pos, T, k, idx, count, hist, workspace, ws_bytes,
                   static_cast<cudaStream_t>(stream));
}

size_t sparse_mla_workspace_size(int32_t T, int32_t k) {
  if (T <= 0 || k <= 0) return 0;
  dsa::DevProps d;
  if (props_for_query(nullptr, &d) != DSA_OK) return 0;
  return dsa::attend_ws_bytes(d, T, k);
}

dsa_status_t sparse_mla_attend(const void* q_nope, const void* q_pe, const float* qmul,
                               float softmax_scale, const void* cache, int64_t n_rows, int32_t ld_c,
                               int32_t d_rope, const int64_t* seq_row_start, int32_t B,
                               const int32_t* q_seq, const int32_t* q_pos, const int32_t* idx,
                               const int32_t* count, int32_t T, int32_t k, void* out, float* lse,
                               void* workspace, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("sparse_mla_attend");
  const dsa_layer_args a = one_layer(q_nope, q_pe, qmul, cache, ld_c, d_rope, out, lse);
  DSA_TRY(check_attend_common(n_rows, seq_row_start, B, q_seq, q_pos, idx, count, T, k));
  DSA_TRY(check_layer_args(a, n_rows));
  if (T == 0) return DSA_OK;
  DevLock L;
  DSA_TRY(lock_device(L));
  return launch_attend(L, &a, 1, softmax_scale, n_rows, seq_row_start, B, q_seq, q_pos, idx, count, T, k,
                       workspace, ws_bytes, static_cast<cudaStream_t>(stream));
}

// Same computation as sparse_mla_attend, for callers that may not allocate:
// the split partials go to the library's fixed scratch array instead of a
// caller workspace.  Launches exactly the kernels sparse_mla_attend launches.
dsa_status_t sparse_mla_attend_noalloc(const void* q_nope, const void* q_pe, const float* qmul,
                                       float softmax_scale, const void* cache, int64_t n_rows,
                                       int32_t ld_c, int32_t d_rope, const int64_t* seq_row_start,
                                       int32_t B, const int32_t* q_seq, const int32_t* q_pos,
                                       const int32_t* idx, const int32_t* count, int32_t T, int32_t k,
                                       void* out, float* lse, void* stream) {
  NvtxRange nvtx_range("sparse_mla_attend_noalloc");
  const dsa_layer_args a = one_layer(q_nope, q_pe, qmul, cache, ld_c, d_rope, out, lse);
  DSA_TRY(check_attend_common(n_rows, seq_row_start, B, q_seq, q_pos, idx, count, T, k));
  DSA_TRY(check_layer_args(a, n_rows));
  if (T == 0) return DSA_OK;
  DevLock L;
  DSA_TRY(lock_device(L));
  dsa::DevProps props;
  DSA_TRY(device_props(L, &props));
  const dsa::SplitPlan sp = dsa::attend_plan(props, T, k);
  void* scratch = nullptr;
  size_t scratch_bytes = 0;
  if (sp.n_split > 1 && !sp.merge) {
    const int64_t partials = (int64_t)T * sp.n_split;
    if (partials > kNoAllocMaxPartials)
      return fail(DSA_ERR_WORKSPACE,
                  "sparse_mla_attend_noalloc: %d queries split %d ways need %lld partials; its fixed "
                  "scratch holds %d (use sparse_mla_attend with a workspace, or another batch size: "
                  "dsa_plan_attend predicts the split)",
                  T, sp.n_split, (long long)partials, kNoAllocMaxPartials);
    DSA_TRY(noalloc_scratch(L, &scratch));
    scratch_bytes = kNoAllocBytes;
  }
  return launch_attend(L, &a, 1, softmax_scale, n_rows, seq_row_start, B, q_seq, q_pos, idx, count, T, k,
                       scratch, scratch_bytes, static_cast<cudaStream_t>(stream));
}

size_t sparse_mla_layers_workspace_size(int32_t T, int32_t n_layers, int32_t k) {
  if (T <= 0 || n_layers <= 0 || k <= 0) return 0;
  dsa::DevProps d;
  if (props_for_query(nullptr, &d) != DSA_OK) return 0;
  return dsa::attend_ws_layers(d, T, n_layers, k);
}

dsa_status_t sparse_mla_attend_layers(int32_t n_layers, const dsa_layer_args* layers, float softmax_scale,
                                      int64_t n_rows, const int64_t* seq_row_start, int32_t B,
                                      const int32_t* q_seq, const int32_t* q_pos, const int32_t* idx,
                                      const int32_t* count, int32_t T, int32_t k, void* workspace,
                                      size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("sparse_mla_attend_layers");
  DSA_REQUIRE(n_layers >= 0 && (n_layers == 0 || layers != nullptr), "bad layer list");
  DSA_TRY(check_attend_common(n_rows, seq_row_start, B, q_seq, q_pos, idx, count, T, k));
  for (int l = 0; l < n_layers; ++l) {
    const dsa_status_t st = check_layer_args(layers[l], n_rows);
    if (st != DSA_OK) return fail(st, "layer %d: %s", l, g_last_error.c_str());
    DSA_REQUIRE(layers[l].cache_fp8 == layers[0].cache_fp8, "every layer of a call must use the same cache format");
  }
  if (T == 0 || n_layers == 0) return DSA_OK;
  DevLock L;
  DSA_TRY(lock_device(L));
  return attend_layers_impl(L, layers, n_layers, softmax_scale, n_rows, seq_row_start, B, q_seq, q_pos, idx,
                            count, T, k, 0, workspace, ws_bytes, static_cast<cudaStream_t>(stream));
}

size_t dsa_forward_workspace_size(int32_t T, int64_t ld, int32_t k, int32_t q_group, int32_t n_layers) {
  (void)q_group;
  if (T <= 0 || ld <= 0 || k <= 0) return 0;
  dsa::DevProps d;
  if (props_for_query(nullptr, &d) != DSA_OK) return 0;
  return dsa::forward_layout_for(d, T, ld, k, std::max(0, n_layers), true, true, T, true, q_group == 1).end;
}

}  // extern "C"

namespace {

// Index keys of the fused call: bf16 (q_idx, k_idx) or E4M3 codes with scales.
struct IndexKeys {
  const void* q;
  const float* q_scale;   // FP8 only
  const void* k;
  const float* k_scale;   // FP8 only
  bool fp8;
};

dsa_status_t forward_impl(const IndexKeys& ik, const float* w, int64_t n_rows, const int64_t* seq_row_start,
                          int32_t B, const int32_t* q_seq, const int32_t* q_pos, int32_t T, int32_t q_group,
                          int64_t ld, int32_t n_layers, const dsa_layer_args* layers, float softmax_scale, int32_t k,
                          int32_t* idx_out, int32_t* count_out, void* workspace, size_t ws_bytes, void* stream) {
  DSA_TRY(check_index_args(ik.q, w, ik.k, n_rows, seq_row_start, B, q_seq, q_pos, T, q_group, ld));
  if (ik.fp8)
    DSA_REQUIRE(ik.q_scale && ik.k_scale && aligned(ik.q_scale, 4) && aligned(ik.k_scale, 4),
                "q_scale and k_scale must be non-null and 4-byte aligned");
  DSA_REQUIRE(k >= 1 && k <= kMaxK, "k must be in [1, %d]", kMaxK);
  DSA_REQUIRE(n_layers >= 0 && (n_layers == 0 || layers != nullptr), "bad layer list");
  DSA_REQUIRE(idx_out == nullptr || aligned(idx_out, 4), "misaligned idx_out");
  DSA_REQUIRE(count_out == nullptr || aligned(count_out, 4), "misaligned count_out");
  for (int l = 0; l < n_layers; ++l) {
    const dsa_status_t st = check_layer_args(layers[l], n_rows);
    if (st != DSA_OK) return fail(st, "layer %d: %s", l, g_last_error.c_str());
    DSA_REQUIRE(layers[l].cache_fp8 == layers[0].cache_fp8, "every layer of a call must use the same cache format");
  }
  if (T == 0) return DSA_OK;
  DSA_REQUIRE(workspace != nullptr && aligned(workspace, 256), "workspace must be non-null and 256-byte aligned");
  DevLock L;
  DSA_TRY(lock_device(L));
  dsa::DevProps props;
  DSA_TRY(device_props(L, &props));
  const bool own_idx = idx_out == nullptr, own_count = count_out == nullptr;
  const dsa::ForwardLayout f =
      dsa::forward_layout(props, T, ld, k, q_group, n_layers, own_idx, own_count, ws_bytes);
  if (f.chunk == 0)
    return fail(DSA_ERR_WORKSPACE, "workspace of %zu bytes is too small (need %zu for %d queries)", ws_bytes,
                f.end, std::min(T, q_group));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* idx_ws = own_idx ? reinterpret_cast<int32_t*>(ws + f.idx_off) : nullptr;
  int32_t* cnt_ws = own_count ? reinterpret_cast<int32_t*>(ws + f.cnt_off) : nullptr;
  void* att_ws = ws + f.att_off;
  uint32_t* hist = (f.hist_off != SIZE_MAX) ? reinterpret_cast<uint32_t*>(ws + f.hist_off) : nullptr;
  void* topk_ws = (f.topk_off != SIZE_MAX) ? ws + f.topk_off : nullptr;
  float* scores = reinterpret_cast<float*>(ws + f.scores_off);
  const int64_t q_row = (int64_t)dsa::kIdxHeads * dsa::kIdxDim;   // values (bytes for FP8, elements for bf16)

  for (int32_t t0 = 0; t0 < T; t0 += f.chunk) {
    const int32_t n = std::min(f.chunk, T - t0);
    int32_t* idx_c = own_idx ? idx_ws : idx_out + (int64_t)t0 * k;
    int32_t* cnt_c = own_count ? cnt_ws : count_out + t0;
    const float* w_c = w + (int64_t)t0 * dsa::kIdxHeads;
    if (ik.fp8) {
      const uint8_t* q8 = static_cast<const uint8_t*>(ik.q) + (int64_t)t0 * q_row;
      const float* qs = ik.q_scale + (int64_t)t0 * dsa::kIdxHeads;
      if (q_group == 8)
        DSA_TRY(launch_indexer<8, true>(L, q8, qs, w_c, ik.k, ik.k_scale, n_rows, seq_row_start, B, q_seq + t0,
                                        q_pos + t0, n, scores, ld, nullptr, s));
      else if (q_group == 4)
        DSA_TRY(launch_indexer<4, true>(L, q8, qs, w_c, ik.k, ik.k_scale, n_rows, seq_row_start, B, q_seq + t0,
                                        q_pos + t0, n, scores, ld, nullptr, s));
      else
        DSA_TRY(launch_indexer<1, true>(L, q8, qs, w_c, ik.k, ik.k_scale, n_rows, seq_row_start, B, q_seq + t0,
                                        q_pos + t0, n, scores, ld, hist, s));
    } else {
      DSA_TRY(indexer_impl(L, static_cast<const __nv_bfloat16*>(ik.q) + (int64_t)t0 * q_row, w_c, ik.k, n_rows,
                           seq_row_start, B, q_seq + t0, q_pos + t0, n, q_group, scores, ld, hist, s));
    }
    DSA_TRY(topk_impl(L, scores, ld, q_pos + t0, n, k, idx_c, cnt_c, hist, topk_ws, f.topk_bytes, s));
    // The kernels before the attention in this call (indexer, top-k, earlier
    // attention groups) do not write the queries, so the attention may start
    // copying them while the top-k finishes.
    DSA_TRY(attend_layers_impl(L, layers, n_layers, softmax_scale, n_rows, seq_row_start, B, q_seq + t0,
                               q_pos + t0, idx_c, cnt_c, n, k, t0, att_ws, f.att_bytes, s, f.partials, true));
  }
  return DSA_OK;
}

}  // namespace

extern "C" {

dsa_status_t dsa_sparse_mla_forward(const void* q_idx, const float* w, const void* k_idx, int64_t n_rows,
                                    const int64_t* seq_row_start, int32_t B, const int32_t* q_seq,
                                    const int32_t* q_pos, int32_t T, int32_t q_group, int64_t ld,
                                    int32_t n_layers, const dsa_layer_args* layers,
                                    float softmax_scale, int32_t k, int32_t* idx_out,
                                    int32_t* count_out, void* workspace, size_t ws_bytes,
                                    void* stream) {
  NvtxRange nvtx_range("dsa_sparse_mla_forward");
  return forward_impl(IndexKeys{q_idx, nullptr, k_idx, nullptr, false}, w, n_rows, seq_row_start, B, q_seq, q_pos, T,
                      q_group, ld, n_layers, layers, softmax_scale, k, idx_out, count_out, workspace, ws_bytes,
                      stream);
}

dsa_status_t dsa_sparse_mla_forward_fp8(const void* q8, const float* q_scale, const float* w, const void* k8,
                                        const float* k_scale, int64_t n_rows, const int64_t* seq_row_start,
                                        int32_t B, const int32_t* q_seq, const int32_t* q_pos, int32_t T,
                                        int32_t q_group, int64_t ld, int32_t n_layers,
                                        const dsa_layer_args* layers, float softmax_scale, int32_t k,
                                        int32_t* idx_out, int32_t* count_out, void* workspace, size_t ws_bytes,
                                        void* stream) {
  NvtxRange nvtx_range("dsa_sparse_mla_forward_fp8");
  return forward_impl(IndexKeys{q8, q_scale, k8, k_scale, true}, w, n_rows, seq_row_start, B, q_seq, q_pos, T,
                      q_group, ld, n_layers, layers, softmax_scale, k, idx_out, count_out, workspace, ws_bytes,
                      stream);
}

dsa_status_t dsa_topk_export(const float* scores, int64_t ld, const int32_t* idx, const int32_t* count, int32_t T,
                             int32_t k, int64_t pos_offset, float* out_score, int32_t* out_pos, void* stream) {
  NvtxRange nvtx_range("dsa_topk_export");
  DSA_REQUIRE(T >= 0 && k >= 1 && k <= kMaxK && ld >= 1, "bad sizes");
  DSA_REQUIRE(scores && idx && count && out_score && out_pos, "null pointer argument");
  DSA_REQUIRE(aligned(scores, 4) && aligned(idx, 4) && aligned(count, 4) && aligned(out_score, 4) &&
                  aligned(out_pos, 4), "misaligned argument");
  DSA_REQUIRE(pos_offset >= 0 && pos_offset + ld < (int64_t(1) << 31), "global positions must fit int32");
  if (T == 0) return DSA_OK;
  DevLock L;
  DSA_TRY(lock_device(L));
  return launch(dsa::topk_export_kernel, (unsigned)T, 256, 0, static_cast<cudaStream_t>(stream), 1, scores, ld, idx,
                count, T, k, pos_offset, out_score, out_pos);
}

dsa_status_t dsa_topk_merge(const float* cand_score, const int32_t* cand_pos, int32_t R, int32_t T, int32_t kr,
                            int32_t k, int64_t shard_lo, int64_t shard_hi, int32_t* idx_global, int32_t* idx_local,
                            int32_t* count_local, int32_t* count, void* stream) {
  NvtxRange nvtx_range("dsa_topk_merge");
  DSA_REQUIRE(R >= 1 && T >= 0 && kr >= 1 && k >= 1 && k <= kMaxK, "bad sizes");
  DSA_REQUIRE((int64_t)R * kr <= dsa::kMergeCap, "R x kr must be <= %d candidates per query", dsa::kMergeCap);
  DSA_REQUIRE(cand_score && cand_pos && count, "null pointer argument");
  DSA_REQUIRE((idx_local == nullptr) == (count_local == nullptr), "idx_local and count_local go together");
  DSA_REQUIRE(count_local == nullptr || aligned(count_local, 4), "misaligned count_local");
  DSA_REQUIRE(aligned(cand_score, 4) && aligned(cand_pos, 4) && aligned(count, 4) &&
                  (idx_global == nullptr || aligned(idx_global, 4)) && (idx_local == nullptr || aligned(idx_local, 4)),
              "misaligned argument");
  DSA_REQUIRE(0 <= shard_lo && shard_lo <= shard_hi, "bad shard range");
  if (T == 0) return DSA_OK;
  DevLock L;
  DSA_TRY(lock_device(L));
  dsa::MergeParams mp;
  mp.cand_score = cand_score;
  mp.cand_pos = cand_pos;
  mp.shard_lo = shard_lo;
  mp.shard_hi = shard_hi;
  mp.idx_global = idx_global;
  mp.idx_local = idx_local;
  mp.count_local = count_local;
  mp.count = count;
  mp.R = R;
  mp.T = T;
  mp.kr = kr;
  mp.k = k;
  DSA_TRY(set_smem(*L.s, kKTopkMerge, dsa::topk_merge_kernel, dsa::kTopkSmemBytes));
  return launch(dsa::topk_merge_kernel, (unsigned)T, dsa::kTopkThreads, dsa::kTopkSmemBytes,
                static_cast<cudaStream_t>(stream), 1, mp);
}

dsa_status_t dsa_lse_combine(const float* o_parts, const float* lse_parts, int32_t R, int32_t T, void* out,
                             float* lse, void* stream) {
  NvtxRange nvtx_range("dsa_lse_combine");
  DSA_REQUIRE(R >= 1 && R <= 64 && T >= 0, "1 <= R <= 64 and T >= 0 required");
  DSA_REQUIRE(o_parts && lse_parts && out, "null pointer argument");
  DSA_REQUIRE(aligned(o_parts, 16) && aligned(out, 16) && aligned(lse_parts, 4) && (lse == nullptr || aligned(lse, 4)),
              "misaligned argument");
  DSA_REQUIRE((int64_t)T * dsa::kHeads < (int64_t(1) << 31), "T too large");
  if (T == 0) return DSA_OK;
  DevLock L;
  DSA_TRY(lock_device(L));
  dsa::LseCombineParams cp;
  cp.o_parts = o_parts;
  cp.lse_parts = lse_parts;
  cp.out = static_cast<__nv_bfloat16*>(out);
  cp.lse = lse;
  cp.R = R;
  cp.T = T;
  return launch(dsa::lse_combine_kernel, (unsigned)(T * dsa::kHeads), 128, 0, static_cast<cudaStream_t>(stream), 1,
                cp);
}

dsa_status_t dsa_get_device_props(dsa_device_props* out) {
  DSA_REQUIRE(out != nullptr, "null pointer argument");
  dsa::DevProps d;
  DSA_TRY(props_for_query(nullptr, &d));
  out->sms = d.sms;
  for (int c = 0; c < 9; ++c) out->max_clusters[c] = d.max_clusters[c];
  return DSA_OK;
}

dsa_status_t dsa_plan_attend(int32_t T, int32_t n_layers, int32_t k, int32_t allow_partials,
                             const dsa_device_props* props, dsa_attend_plan* out) {
  DSA_REQUIRE(out != nullptr, "null pointer argument");
  DSA_REQUIRE(T >= 1 && n_layers >= 1 && n_layers <= dsa::kMaxAttLayers && k >= 1 && k <= kMaxK,
              "T >= 1, 1 <= n_layers <= %d and 1 <= k <= %d required", dsa::kMaxAttLayers, kMaxK);
  dsa::DevProps d;
  DSA_TRY(props_for_query(props, &d));
  fill_attend_plan(d, (int64_t)T * n_layers, k, allow_partials != 0, out);
  return DSA_OK;
}

dsa_status_t dsa_plan_forward(int32_t T, int64_t ld, int32_t k, int32_t q_group, int32_t n_layers,
                              int32_t has_idx_out, int32_t has_count_out, size_t ws_bytes,
                              const dsa_device_props* props, dsa_forward_plan* out) {
  DSA_REQUIRE(out != nullptr, "null pointer argument");
  DSA_REQUIRE(T >= 1 && ld >= 4 && k >= 1 && k <= kMaxK && (q_group == 1 || q_group == 4 || q_group == 8) &&
                  n_layers >= 0,
              "bad sizes");
  dsa::DevProps d;
  DSA_TRY(props_for_query(props, &d));
  const dsa::ForwardLayout f = dsa::forward_layout(d, T, ld, k, q_group, n_layers, !has_idx_out, !has_count_out,
                                                   ws_bytes);
  out->chunk = f.chunk;
  out->n_chunks = f.chunk ? f.n_chunks : 0;
  out->last_chunk = f.chunk ? f.last_chunk : 0;
  out->attend_partials = f.partials ? 1 : 0;
  out->idx_offset = f.idx_off;
  out->count_offset = f.cnt_off;
  out->attend_offset = f.att_off;
  out->attend_bytes = f.att_bytes;
  out->hist_offset = f.hist_off;
  out->topk_offset = f.topk_off;
  out->topk_bytes = f.topk_bytes;
  out->scores_offset = f.scores_off;
  out->end = f.end;
  if (f.chunk == 0) return fail(DSA_ERR_WORKSPACE, "workspace of %zu bytes is too small (need %zu)", ws_bytes, f.end);
  return DSA_OK;
}

dsa_status_t dsa_set_fault_test(uint64_t wait_limit_ns, int32_t stall_tile) {
  g_wait_limit_ns.store(wait_limit_ns, std::memory_order_relaxed);
  g_stall_tile.store(stall_tile < 0 ? -1 : stall_tile, std::memory_order_relaxed);
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

int32_t dsa_version(void) { return 201; }

}  // extern "C"
