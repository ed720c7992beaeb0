// C ABI of the MoE feed-forward block (declared in include/moe_block.h):
// host-side validation, workspace layout, TMA descriptors and the launch
// sequence router -> top-k -> scan -> scatter -> gather -> gate|up GEMM ->
// down GEMM -> combine, all on the caller's stream with no host sync.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "moe_block.h"
#include "grouped_gemm.cuh"
#include "grouped_gemm_pair.cuh"
#include "norm.cuh"
#include "permute.cuh"
#include "router.cuh"
#include "nvfp4.cuh"
#include "wq_gemm.cuh"

namespace moe {

__device__ uint32_t g_device_error;

namespace {

constexpr int kMaxDevices = 64;
constexpr int kSmCountHint = 148;  // B200: sizes the router's split of the reduction
constexpr size_t kAlign = 256;

thread_local int t_launches = 0;

struct Dims {
  int T, k, D, E, F, S;
  int e0 = 0, el = 0;  // expert shard: experts [e0, e0 + el) of the E the router scores (el = E: all)
};

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct Layout {
  size_t total;
  size_t partial, idx, w, masks, base, cnt, off, row_of, token_of, tiles_gu, tiles_dn, counts;
  size_t x_perm, h, y, hs, s, x_norm;
  size_t guard;  // 256 bytes of guard words after the data (written and checked only on request)
  int nsplit, nchunks, max_tiles_gu, max_tiles_dn;
};

// Small batches (experts average at most half a 128-row block) read every
// expert weight tile from one row block: the GEMMs then stream the weights
// with an L2 evict-first policy. (Measured: decode T=64 0.288 -> 0.281 ms; at
// T=4096, where an expert's row blocks share its weight tiles through L2, the
// same policy cost 0.707 -> 0.725 ms.)
bool stream_weights(const Dims& d) { return static_cast<long long>(d.T) * d.k * 2 <= static_cast<long long>(kBM) * d.E; }

// Large batches (experts average >= 160 routed rows) use the paired gate|up GEMM.
bool paired_gateup(const Dims& d) { return static_cast<long long>(d.T) * d.k >= 160LL * d.E; }
// The paired down GEMM pays off later (measured: at ~256 rows per expert it is
// slower, at ~1024 faster): its K = expert_dim is short, so a tile's single-
// buffered accumulators drain often.
bool paired_down(const Dims& d) { return static_cast<long long>(d.T) * d.k >= 512LL * d.E; }

// Splits of the router's reduction: enough (token tile, split) CTAs for one
// wave at one CTA per SM, at least two 64-wide slices per split.
int router_splits(const Dims& d) {
  const int tiles = std::max(1, (d.T + kRouterTokens - 1) / kRouterTokens);
  int ns = kSmCountHint / tiles;
  ns = std::min(ns, kMaxRouterSplits);
  ns = std::min(ns, d.D / (2 * kRouterBK));
  return std::max(ns, 1);
}

Layout make_layout(const Dims& d) {
  Layout L{};
  const size_t T = d.T, k = d.k, E = d.E, R = T * k;
  L.nsplit = router_splits(d);
  L.nchunks = static_cast<int>((T + kMaskTokens - 1) / kMaskTokens);
  const int mt_sh = static_cast<int>((T + kBM - 1) / kBM);
  const long long mt_max = static_cast<long long>(R / kBM) + std::min<long long>(E, R) + 1;
  L.max_tiles_gu = static_cast<int>(((d.S + 127) / 128) * mt_sh + mt_max * ((d.F + 127) / 128));
  L.max_tiles_dn = static_cast<int>(((d.D + 255) / 256) * mt_sh + mt_max * ((d.D + 255) / 256));
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes, kAlign);
    return at;
  };
  L.partial = take(static_cast<size_t>(L.nsplit) * T * E * 4);
  L.idx = take(R * 4);
  L.w = take(R * 4);
  L.masks = take(static_cast<size_t>(L.nchunks) * E * 4);
  L.base = take(static_cast<size_t>(L.nchunks) * E * 4);
  L.cnt = take(E * 4);
  L.off = take((E + 1) * 4);
  L.row_of = take(R * 4);
  L.token_of = take(R * 4);
  L.tiles_gu = take(static_cast<size_t>(L.max_tiles_gu) * sizeof(Tile));
  L.tiles_dn = take(static_cast<size_t>(L.max_tiles_dn) * sizeof(Tile));
  L.counts = take(sizeof(TileCounts));
  L.x_perm = take(R * d.D * 2);
  L.h = take(R * d.F * 2);
  L.y = take(R * d.D * 2);
  L.hs = take(T * d.S * 2);
  L.s = take(T * d.D * 4);
  L.x_norm = take(T * d.D * 2);
  L.guard = take(kGuardWords * 4);
  L.total = o;
  return L;
}

Dims dims_of(const moe_params* p) {
  Dims d;
  d.T = p->T;
  d.k = p->top_k_experts;
  d.D = p->embed_dim ? p->embed_dim : MOE_EMBED_DIM;
  d.E = p->num_experts ? p->num_experts : MOE_NUM_EXPERTS;
  d.F = p->expert_dim ? p->expert_dim : MOE_EXPERT_DIM;
  d.S = p->hidden_dim ? p->hidden_dim : MOE_HIDDEN_DIM;
  d.e0 = p->expert_begin;
  d.el = p->expert_count ? p->expert_count : d.E - d.e0;
  return d;
}

bool dims_ok(const Dims& d) {
  if (d.e0 < 0 || d.el < 1 || d.e0 > d.E - d.el) return false;
  if (d.T < 0) return false;
  if (d.D <= 0 || d.F <= 0 || d.S <= 0 || d.D % 64 || d.F % 64 || d.S % 64) return false;
  if (d.E < 8 || d.E > 128 || d.E % 8) return false;
  if (d.k < 1 || d.k > d.E) return false;
  if (static_cast<long long>(d.T) * d.k > (1LL << 30)) return false;
  return true;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
inline bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3) == 0; }

// ---------------------------------------------------------- per-device state

std::mutex g_mutex;
struct DeviceState {
  bool init = false;
  bool arch_ok = false;
  int sm_count = 0;
  uint32_t* err = nullptr;
  void* ws = nullptr;
  size_t ws_bytes = 0;
  int pair_clusters_dn = 0;  // SM-pair clusters of the pair down GEMM that fit on the device at once
};
DeviceState g_dev[kMaxDevices];

// Large batches run the down GEMM on SM pairs (tcgen05 cta_group::2) when its
// column tiles split into whole 64-column chunks per CTA. (The gate|up GEMM
// stays on single SMs: measured slower on pairs, whose M = 256 MMA runs in
// full for an expert's odd last row block over the long K = embed_dim.)
bool pair_sm(const Dims& d, const DeviceState* s) {
  return static_cast<long long>(d.T) * d.k >= 160LL * d.E && d.D % 128 == 0 && s->pair_clusters_dn > 0;
}


moe_status device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceState& s = g_dev[dev];
  if (!s.init) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MOE_ERR_CUDA;
    s.arch_ok = prop.major == 10 && prop.minor == 0;
    s.sm_count = prop.multiProcessorCount;
    if (s.arch_ok) {
      if (cudaGetSymbolAddress(reinterpret_cast<void**>(&s.err), g_device_error) != cudaSuccess) return MOE_ERR_CUDA;
      if (cudaFuncSetAttribute(router_logits_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kRouterSmemBytes) != cudaSuccess)
        return MOE_ERR_CUDA;
      if (cudaFuncSetAttribute(grouped_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kGemmSmemBytes) != cudaSuccess)
        return MOE_ERR_CUDA;
      if (cudaFuncSetAttribute(grouped_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kGemmSmemBytes) != cudaSuccess)
        return MOE_ERR_CUDA;
      if (cudaFuncSetAttribute(grouped_gemm_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kGemmSmemBytes) != cudaSuccess)
        return MOE_ERR_CUDA;
      if (cudaFuncSetAttribute(grouped_gemm_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kGemmSmemBytes) != cudaSuccess)
        return MOE_ERR_CUDA;
      if (cudaFuncSetAttribute(grouped_gemm_pair_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kP2SmemBytes) != cudaSuccess)
        return MOE_ERR_CUDA;
      {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (s.sm_count / 2));
        cfg.blockDim = dim3(kGemmThreads);
        cfg.dynamicSmemBytes = kP2SmemBytes;
        if (cudaOccupancyMaxActiveClusters(&s.pair_clusters_dn, grouped_gemm_pair_kernel<false>, &cfg) != cudaSuccess)
          return MOE_ERR_CUDA;
      }
      if (cudaFuncSetAttribute(fp4_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kF4SmemBytes) !=
          cudaSuccess)
        return MOE_ERR_CUDA;
      if (cudaFuncSetAttribute(wq_gemm_kernel<kWfSfp8, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kWqSmemBytes) != cudaSuccess ||
          cudaFuncSetAttribute(wq_gemm_kernel<kWfSfp8, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kWqSmemBytes) != cudaSuccess ||
          cudaFuncSetAttribute(wq_gemm_kernel<kWfQ4, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kWqSmemBytes) != cudaSuccess ||
          cudaFuncSetAttribute(wq_gemm_kernel<kWfQ4, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kWqSmemBytes) != cudaSuccess)
        return MOE_ERR_CUDA;
      if (cudaFuncSetAttribute(fp4_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kF4SmemBytes) !=
          cudaSuccess)
        return MOE_ERR_CUDA;
    }
    s.init = true;
  }
  if (!s.arch_ok) return MOE_ERR_ARCH;
  *out = &s;
  return MOE_OK;
}

// Library-owned workspace, grown on demand (one per device).
moe_status library_workspace(DeviceState* s, size_t bytes, void** out) {
  std::lock_guard<std::mutex> lock(g_mutex);
  if (s->ws_bytes < bytes) {
    if (s->ws) {
      cudaDeviceSynchronize();
      cudaFree(s->ws);
      s->ws = nullptr;
      s->ws_bytes = 0;
    }
    if (cudaMalloc(&s->ws, bytes) != cudaSuccess) {
      s->ws = nullptr;
      return MOE_ERR_CUDA;
    }
    s->ws_bytes = bytes;
  }
  *out = s->ws;
  return MOE_OK;
}

// ------------------------------------------------------------ tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [rows, cols] bf16 row-major; box = 64 columns x box_rows rows; 128-byte swizzle.
bool map_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [groups, K, N] bf16 with N contiguous; box = 64 (N) x 64 (K) x 1; 128-byte swizzle.
bool map_3d(CUtensorMap* m, const void* base, uint64_t groups, uint64_t K, uint64_t N) {
  const cuuint64_t dims[3] = {N, K, groups};
  const cuuint64_t strides[2] = {N * 2, K * N * 2};
  const cuuint32_t box[3] = {64, 64, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [groups, K, N] bf16 viewed as [groups][N / 64][K][64]: 64-column chunks as a
// dimension of their own, so one box of 64 x 64 x chunks x 1 brings `chunks`
// adjacent chunks, each landing as the 64 x 64 box of map_3d would (8 KB
// apart). Requires N % 64 == 0.
bool map_4d_chunks(CUtensorMap* m, const void* base, uint64_t groups, uint64_t K, uint64_t N, uint32_t chunks) {
  const cuuint64_t dims[4] = {64, K, N / 64, groups};
  const cuuint64_t strides[3] = {N * 2, 128, K * N * 2};
  const cuuint32_t box[4] = {64, 64, chunks, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The wide boxes of a GEMM (GemmParams::tmA2 / tmBw*): A pairs of 128-row
// blocks when a_wide, B chunks of `chunks` when nonzero. A map that cannot be
// encoded leaves the per-block / per-chunk copies in use.
void set_wide_maps(GemmParams* g, int p, const void* a, uint64_t a_rows, uint64_t K, bool a_wide, const void* b0,
                   const void* b1, uint64_t groups, uint64_t N, uint32_t chunks) {
  if (a_wide && !map_2d(&g->tmA2[p], a, a_rows, K, 2 * kBM)) g->a_wide = 0;
  if (g->a_small && !map_2d(&g->tmAs[p], a, a_rows, K, kASmallRows)) g->a_small = 0;
  if (chunks && (!map_4d_chunks(&g->tmBw0[p], b0, groups, K, N, chunks) ||
                 (b1 && !map_4d_chunks(&g->tmBw1[p], b1, groups, K, N, chunks))))
    g->bw_chunks = 0;
}

// Kernel ids of the per-kernel timing records.
enum KernelId : int {
  kKRouterLogits = 0,
  kKRouterTopk,
  kKBuildMasks,
  kKRouteScan,
  kKRouteScatter,
  kKGemmGateUp,
  kKGemmDown,
  kKCombine,
  kKTimeoutProbe,
  kKWeightAmax,
  kKTensorScale,
  kKWeightQuant,
  kKActQuant,
  kKScatterFp4,
  kKFp4GateUp,
  kKFp4Down,
  kKCombineNorm,
  kKAmax,
  kKPreNorm,
  kKGuard,
  kKCount
};
const char* const kKernelNames[kKCount] = {"router_logits", "router_topk", "build_masks", "route_scan",
                                           "route_scatter", "grouped_gemm_gateup",
                                           "grouped_gemm_down", "combine", "timeout_probe",
                                           "nvfp4_weight_amax", "nvfp4_tensor_scale", "nvfp4_weight_quant",
                                           "nvfp4_act_quant", "route_scatter_fp4", "fp4_gemm_gateup",
                                           "fp4_gemm_down", "combine_norm", "amax", "rms_norm_pre",
                                           "workspace_guard"};

struct ProfRecord {
  int id;
  cudaEvent_t start, stop;
};
thread_local bool t_profiling = false;
thread_local uint32_t t_profile_mask = 0;
thread_local std::vector<ProfRecord> t_records;
thread_local std::vector<cudaEvent_t> t_event_pool;

cudaEvent_t pooled_event() {
  if (!t_event_pool.empty()) {
    cudaEvent_t e = t_event_pool.back();
    t_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Brackets one kernel launch with timing events when profiling is on.
// Also an NVTX range named after the kernel around its launch (a profiler's
// timeline shows which library kernel each launch is; no cost without one).
struct LaunchScope {
  cudaStream_t st;
  int id;
  cudaEvent_t a = nullptr;
  LaunchScope(int id_, cudaStream_t st_) : st(st_), id(id_) {
    nvtxRangePushA(kKernelNames[id]);
    if (t_profiling && ((t_profile_mask >> id) & 1u)) {
      a = pooled_event();
      cudaEventRecord(a, st);
    }
  }
  ~LaunchScope() { nvtxRangePop(); }
  LaunchScope(const LaunchScope&) = delete;
  LaunchScope& operator=(const LaunchScope&) = delete;
  moe_status done(cudaError_t launch_err) {
    ++t_launches;
    if (t_profiling && a) {
      cudaEvent_t b = pooled_event();
      cudaEventRecord(b, st);
      t_records.push_back(ProfRecord{id, a, b});
    }
    return launch_err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }
};

// Every kernel is launched with programmatic stream serialization: it may
// start while its predecessor drains, and waits (griddepcontrol.wait) before
// touching memory, so launch latency and prologues overlap the previous
// kernel's tail.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// An NVTX range around a public entry point.
struct ApiRange {
  explicit ApiRange(const char* name) { nvtxRangePushA(name); }
  ~ApiRange() { nvtxRangePop(); }
  ApiRange(const ApiRange&) = delete;
  ApiRange& operator=(const ApiRange&) = delete;
};

#define MOE_TRY(expr)                   \
  do {                                  \
    const moe_status st_ = (expr);      \
    if (st_ != MOE_OK) return st_;      \
  } while (0)

// ------------------------------------------------------------- validation

moe_status check_block_args(const moe_params* p, Dims* d) {
  if (!p) return MOE_ERR_INVALID_ARG;
  *d = dims_of(p);
  if (!dims_ok(*d)) return MOE_ERR_INVALID_ARG;
  if (d->T == 0) return MOE_OK;
  const void* req[] = {p->x, p->w_router, p->wg, p->wu, p->wd, p->sg, p->su, p->sd};
  for (const void* q : req)
    if (!q) return MOE_ERR_INVALID_ARG;
  for (const void* q : req)
    if (!aligned16(q)) return MOE_ERR_ALIGNMENT;
  if (!p->out && !p->out_f32) return MOE_ERR_INVALID_ARG;  // an output is needed
  if ((p->out && !aligned16(p->out)) || (p->out_f32 && !aligned16(p->out_f32))) return MOE_ERR_ALIGNMENT;
  // a shard's output is a partial sum: the post-norm and residual act on the full sum
  if (d->el != d->E && (p->norm_post || p->residual)) return MOE_ERR_INVALID_ARG;
  if (!p->out && (p->norm_post || p->residual)) return MOE_ERR_INVALID_ARG;
  const void* opt4[] = {p->router_bias, p->idx_out, p->w_out, p->cnt_out, p->logits_out};
  for (const void* q : opt4)
    if (q && !aligned4(q)) return MOE_ERR_ALIGNMENT;
  const uintptr_t xb = reinterpret_cast<uintptr_t>(p->x), ob = reinterpret_cast<uintptr_t>(p->out);
  const uintptr_t bytes = static_cast<uintptr_t>(d->T) * d->D * 2;
  if (p->out && xb < ob + bytes && ob < xb + bytes) return MOE_ERR_INVALID_ARG;
  if ((p->norm_pre && !aligned16(p->norm_pre)) || (p->norm_post && !aligned16(p->norm_post))) return MOE_ERR_ALIGNMENT;
  if ((p->norm_pre || p->norm_post || p->residual) && d->D > kCombThreads * kCombVec * 8) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

moe_status resolve_workspace(const moe_params* p, DeviceState* s, const Layout& L, uint8_t** ws) {
  if (p->workspace) {
    if ((reinterpret_cast<uintptr_t>(p->workspace) & (kAlign - 1)) != 0) return MOE_ERR_ALIGNMENT;
    if (p->workspace_bytes < L.total) return MOE_ERR_WORKSPACE;
    *ws = static_cast<uint8_t*>(p->workspace);
    return MOE_OK;
  }
  void* w = nullptr;
  MOE_TRY(library_workspace(s, L.total, &w));
  *ws = static_cast<uint8_t*>(w);
  return MOE_OK;
}

// ---------------------------------------------------------------- stages

moe_status enqueue_route(const Dims& d, const Layout& L, uint8_t* ws, const void* x, const void* wr,
                         const float* bias, int32_t* idx, float* w, cudaStream_t st, float* logits_out = nullptr) {
  float* partial = reinterpret_cast<float*>(ws + L.partial);
  uint32_t* masks = reinterpret_cast<uint32_t*>(ws + L.masks);
  DeviceState* s = nullptr;
  MOE_TRY(device_state(&s));
  RouterParams rp{};
  if (!map_2d(&rp.tmX, x, d.T, d.D, kRouterTokens) || !map_3d(&rp.tmW, wr, 1, d.D, d.E)) return MOE_ERR_CUDA;
  rp.partial = partial;
  rp.masks = masks;
  rp.err = s->err;
  rp.T = d.T;
  rp.D = d.D;
  rp.E = d.E;
  rp.nsplit = L.nsplit;
  const dim3 g1((d.T + kRouterTokens - 1) / kRouterTokens, L.nsplit);
  {
    LaunchScope ls_(kKRouterLogits, st);
    const cudaError_t le_ = launch_k(router_logits_kernel, g1, kRouterThreads, kRouterSmemBytes, st, rp);
    MOE_TRY(ls_.done(le_));
  }
  LaunchScope ls_(kKRouterTopk, st);
  const int tk_blocks = (d.T + kTopkWarps - 1) / kTopkWarps;
  // large batches: two tokens per warp (E <= 128, k <= 16)
  const bool tk_pair = d.E <= 128 && d.k <= 16 && d.T >= 1024;
  const cudaError_t le_ =
      tk_pair ? launch_k(router_topk_pair_kernel, (d.T + 2 * kTopkWarps - 1) / (2 * kTopkWarps), kTopkWarps * 32, 0,
                         st, partial, bias, d.T, d.E, L.nsplit, d.k, idx, w, masks, logits_out)
      : L.nsplit > 8 ? launch_k(router_topk_kernel<true>, tk_blocks, kTopkWarps * 32, 0, st, partial, bias, d.T, d.E,
                                L.nsplit, d.k, idx, w, masks, logits_out)
                     : launch_k(router_topk_kernel<false>, tk_blocks, kTopkWarps * 32, 0, st, partial, bias, d.T, d.E,
                                L.nsplit, d.k, idx, w, masks, logits_out);
  return ls_.done(le_);
}

// Scan of the bitmasks, then the scatter (and, with x, the copy into x_perm).
// allow_pairs = false: tiles of one 128-row block only (the weight-only GEMMs).
moe_status enqueue_permute(const Dims& d, const Layout& L, uint8_t* ws, const int32_t* idx, const void* x,
                           int32_t* cnt, int32_t* off, int32_t* row_of, int32_t* token_of, cudaStream_t st,
                           bool allow_pairs = true) {
  const uint32_t* masks = reinterpret_cast<const uint32_t*>(ws + L.masks);
  int32_t* base = reinterpret_cast<int32_t*>(ws + L.base);
  DeviceState* s = nullptr;
  MOE_TRY(device_state(&s));
  const bool pairs = allow_pairs && pair_sm(d, s);
  {
    LaunchScope ls_(kKRouteScan, st);
    const cudaError_t le_ = launch_k(route_scan_kernel, kScanCtas, kScanThreads, 0, st, masks, L.nchunks, d.T, d.E, d.F, d.S,
                                     d.D, base, cnt, off, reinterpret_cast<Tile*>(ws + L.tiles_gu),
                                     reinterpret_cast<Tile*>(ws + L.tiles_dn),
                                     reinterpret_cast<TileCounts*>(ws + L.counts), 0, 256, 128,
                                     (allow_pairs && paired_gateup(d)) ? 1 : 0,
                                     (pairs || (allow_pairs && paired_down(d))) ? 1 : 0, d.e0, d.el);
    MOE_TRY(ls_.done(le_));
  }
  const long long R = static_cast<long long>(d.T) * d.k;
  const int blocks = static_cast<int>(std::min<long long>((R + 7) / 8, 148LL * 64));
  LaunchScope ls_(kKRouteScatter, st);
  const cudaError_t le_ = launch_k(route_scatter_kernel, blocks, 256, 0, st, idx, masks, base, d.T, d.k, d.E, d.D,
                                   static_cast<const __nv_bfloat16*>(x), row_of, token_of,
                                   reinterpret_cast<__nv_bfloat16*>(ws + L.x_perm), R, s->err, d.e0, d.el);
  return ls_.done(le_);
}

moe_status enqueue_block(const moe_params* p, const Dims& d, const Layout& L, uint8_t* ws, DeviceState* s,
                         cudaStream_t st) {
  const size_t R = static_cast<size_t>(d.T) * d.k;
  int32_t* idx = reinterpret_cast<int32_t*>(ws + L.idx);
  float* w = reinterpret_cast<float*>(ws + L.w);
  int32_t* cnt = reinterpret_cast<int32_t*>(ws + L.cnt);
  int32_t* off = reinterpret_cast<int32_t*>(ws + L.off);
  int32_t* row_of = reinterpret_cast<int32_t*>(ws + L.row_of);
  int32_t* token_of = reinterpret_cast<int32_t*>(ws + L.token_of);
  __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(ws + L.h);
  __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(ws + L.y);
  __nv_bfloat16* hs = reinterpret_cast<__nv_bfloat16*>(ws + L.hs);
  float* sbuf = reinterpret_cast<float*>(ws + L.s);
  __nv_bfloat16* x_perm = reinterpret_cast<__nv_bfloat16*>(ws + L.x_perm);
  TileCounts* counts = reinterpret_cast<TileCounts*>(ws + L.counts);

  uint32_t* guard = reinterpret_cast<uint32_t*>(ws + L.guard);
  if (p->check_guards) {
    LaunchScope ls_(kKGuard, st);
    MOE_TRY(ls_.done(launch_k(guard_fill_kernel, 1, kGuardWords, 0, st, guard)));
  }
  // the block's input: x, or its pre-FFN RMSNorm (bf16, in the workspace)
  const void* xin = p->x;
  if (p->norm_pre) {
    __nv_bfloat16* xn = reinterpret_cast<__nv_bfloat16*>(ws + L.x_norm);
    LaunchScope ls_(kKPreNorm, st);
    MOE_TRY(ls_.done(launch_k(rms_norm_rows_kernel, d.T, kNormThreads, 0, st,
                              static_cast<const __nv_bfloat16*>(p->x),
                              static_cast<const __nv_bfloat16*>(p->norm_pre), d.T, d.D, xn)));
    xin = xn;
  }
  MOE_TRY(enqueue_route(d, L, ws, xin, p->w_router, p->router_bias, idx, w, st, p->logits_out));
  MOE_TRY(enqueue_permute(d, L, ws, idx, xin, cnt, off, row_of, token_of, st));

  // gate|up: experts (problem 0) and shared MLP (problem 1)
  GemmParams gu;
  std::memset(&gu, 0, sizeof(gu));
  bool ok = map_2d(&gu.tmA[0], x_perm, R, d.D, kBM) && map_3d(&gu.tmB0[0], p->wg, d.el, d.D, d.F) &&
            map_3d(&gu.tmB1[0], p->wu, d.el, d.D, d.F) && map_2d(&gu.tmA[1], xin, d.T, d.D, kBM) &&
            map_3d(&gu.tmB0[1], p->sg, 1, d.D, d.S) && map_3d(&gu.tmB1[1], p->su, 1, d.D, d.S);
  if (!ok) return MOE_ERR_CUDA;
  gu.prob[0] = GemmProblem{d.D, d.F, d.el, static_cast<int>(R), h, d.F, 0, 0};
  gu.prob[1] = GemmProblem{d.D, d.S, 1, d.T, hs, d.S, 0, 0};
  gu.nprob = 2;
  gu.stream_weights = stream_weights(d) ? 1 : 0;
  gu.a_wide = paired_gateup(d) ? 1 : 0;
  gu.a_small = paired_gateup(d) ? 0 : 1;
  gu.bw_chunks = 2;  // 128 output columns of each projection
  set_wide_maps(&gu, 0, x_perm, R, d.D, gu.a_wide, p->wg, p->wu, d.el, d.F, 2);
  set_wide_maps(&gu, 1, xin, d.T, d.D, gu.a_wide, p->sg, p->su, 1, d.S, 2);
  gu.tiles = reinterpret_cast<const Tile*>(ws + L.tiles_gu);
  gu.num_tiles = &counts->gateup;
  gu.next_tile = &counts->next_gateup;
  gu.err = s->err;
  const int grid_gu = std::min(s->sm_count, L.max_tiles_gu);
  {
  LaunchScope ls_(kKGemmGateUp, st);
  const cudaError_t le_ =
      paired_gateup(d) ? launch_k(grouped_gemm_kernel<true, true>, grid_gu, kGemmThreadsSm, kGemmSmemBytes, st, gu)
                       : launch_k(grouped_gemm_kernel<true>, grid_gu, kGemmThreadsSm, kGemmSmemBytes, st, gu);
  MOE_TRY(ls_.done(le_));
  }

  // down: experts -> y (bf16), shared -> s (fp32)
  GemmParams dn;
  std::memset(&dn, 0, sizeof(dn));
  ok = map_2d(&dn.tmA[0], h, R, d.F, kBM) && map_3d(&dn.tmB0[0], p->wd, d.el, d.F, d.D) &&
       map_2d(&dn.tmA[1], hs, d.T, d.S, kBM) && map_3d(&dn.tmB0[1], p->sd, 1, d.S, d.D);
  if (!ok) return MOE_ERR_CUDA;
  dn.tmB1[0] = dn.tmB0[0];
  dn.tmB1[1] = dn.tmB0[1];
  dn.prob[0] = GemmProblem{d.F, d.D, d.el, static_cast<int>(R), y, d.D, 0, 0};
  dn.prob[1] = GemmProblem{d.S, d.D, 1, d.T, sbuf, d.D, 1, 0};
  dn.nprob = 2;
  dn.stream_weights = gu.stream_weights;
  // 256-column tiles: 4 chunks per copy on one SM, 2 per CTA on SM pairs
  dn.bw_chunks = pair_sm(d, s) ? 2 : 4;
  dn.a_wide = paired_down(d) && !pair_sm(d, s) ? 1 : 0;
  dn.a_small = (pair_sm(d, s) || paired_down(d)) ? 0 : 1;
  set_wide_maps(&dn, 0, h, R, d.F, dn.a_wide, p->wd, nullptr, d.el, d.D, dn.bw_chunks);
  set_wide_maps(&dn, 1, hs, d.T, d.S, dn.a_wide, p->sd, nullptr, 1, d.D, dn.bw_chunks);
  dn.tiles = reinterpret_cast<const Tile*>(ws + L.tiles_dn);
  dn.num_tiles = &counts->down;
  dn.next_tile = &counts->next_down;
  dn.err = s->err;
  const int grid_dn = std::min(s->sm_count, L.max_tiles_dn);
  {
  LaunchScope ls_(kKGemmDown, st);
  const cudaError_t le_ =
      pair_sm(d, s) ? launch_k(grouped_gemm_pair_kernel<false>, 2 * s->pair_clusters_dn, kGemmThreads, kP2SmemBytes, st, dn)
      : paired_down(d) ? launch_k(grouped_gemm_kernel<false, true>, grid_dn, kGemmThreadsSm, kGemmSmemBytes, st, dn)
                       : launch_k(grouped_gemm_kernel<false>, grid_dn, kGemmThreadsSm, kGemmSmemBytes, st, dn);
  MOE_TRY(ls_.done(le_));
  }

  if (p->norm_post || p->residual) {
    // the post-FFN norm and / or the residual need a token's whole row: one CTA per token
    LaunchScope ls_(kKCombineNorm, st);
    MOE_TRY(ls_.done(launch_k(combine_norm_kernel, d.T, kCombThreads, 0, st, sbuf, y, row_of, w, d.T, d.k, d.D,
                              static_cast<int>(R), p->norm_post ? 1 : 0,
                              static_cast<const __nv_bfloat16*>(p->norm_post),
                              p->residual ? static_cast<const __nv_bfloat16*>(p->x) : nullptr,
                              static_cast<__nv_bfloat16*>(p->out), p->out_f32, s->err)));
  } else {
  LaunchScope ls_(kKCombine, st);
  const int dsplit = std::max(1, std::min(4, (2 * s->sm_count) / std::max(1, d.T)));
  const cudaError_t le_ = launch_k(combine_kernel, dim3(d.T, dsplit), 128, 0, st, sbuf, y, row_of, w, d.T, d.k, d.D,
                                   static_cast<int>(R), static_cast<__nv_bfloat16*>(p->out), p->out_f32, s->err);
  MOE_TRY(ls_.done(le_));
  }

  if (p->check_guards) {
    LaunchScope ls_(kKGuard, st);
    MOE_TRY(ls_.done(launch_k(guard_check_kernel, 1, kGuardWords, 0, st, static_cast<const uint32_t*>(guard), s->err)));
  }
  if (p->idx_out && cudaMemcpyAsync(p->idx_out, idx, R * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (p->w_out && cudaMemcpyAsync(p->w_out, w, R * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (p->cnt_out && cudaMemcpyAsync(p->cnt_out, cnt, d.E * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

// ------------------------------------------------------------- NVFP4 host

// [rows, cols] bytes; box 128 bytes x 128 rows; 128-byte swizzle.
bool map_2d_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols};
  const cuuint32_t box[2] = {128, 128};
  const cuuint32_t estr[2] = {1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [groups, rows, cols] bytes; box 128 bytes x box_rows x 1; 128-byte swizzle.
bool map_3d_u8(CUtensorMap* m, const void* base, uint64_t groups, uint64_t rows, uint64_t cols,
               uint32_t box_rows = 128) {
  const cuuint64_t dims[3] = {cols, rows, groups};
  const cuuint64_t strides[2] = {cols, rows * cols};
  const cuuint32_t box[3] = {128, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t fp4_q_bytes(size_t groups, size_t K, size_t N) { return groups * N * (K / 2); }
size_t fp4_sf_bytes(size_t groups, size_t K, size_t N) { return groups * ((N + 127) / 128) * (K / 64) * 512; }

// The NVFP4 workspace: the routing part (same fields as the bf16 layout) and
// the quantised activations in a 128-padded expert-major row space.
struct Fp4Layout {
  Layout r;  // routing offsets (partial, idx, w, masks, base, cnt, off, row_of, tiles, counts)
  size_t xq_perm, xsf_perm, xq_tok, xsf_tok, hq, hsf, hsq, hssf, y, s;
  size_t total;
  long long r_pad, t_pad;
};

Fp4Layout make_fp4_layout(const Dims& d) {
  Fp4Layout F{};
  Layout& L = F.r;
  const size_t T = d.T, k = d.k, E = d.E, R = T * k;
  L.nsplit = router_splits(d);
  L.nchunks = static_cast<int>((T + kMaskTokens - 1) / kMaskTokens);
  const int mt_sh = static_cast<int>((T + kBM - 1) / kBM);
  const long long mt_max = static_cast<long long>(R / kBM) + std::min<long long>(E, R) + 1;
  L.max_tiles_gu = static_cast<int>(((d.S + 127) / 128) * mt_sh + mt_max * ((d.F + 127) / 128));
  L.max_tiles_dn = static_cast<int>(((d.D + 255) / 256) * mt_sh + mt_max * ((d.D + 255) / 256));
  F.r_pad = mt_max * kBM;
  F.t_pad = static_cast<long long>(mt_sh) * kBM;
  const size_t rp = F.r_pad, tp = F.t_pad;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes, kAlign);
    return at;
  };
  L.partial = take(static_cast<size_t>(L.nsplit) * T * E * 4);
  L.idx = take(R * 4);
  L.w = take(R * 4);
  L.masks = take(static_cast<size_t>(L.nchunks) * E * 4);
  L.base = take(static_cast<size_t>(L.nchunks) * E * 4);
  L.cnt = take(E * 4);
  L.off = take((E + 1) * 4);
  L.row_of = take(R * 4);
  L.tiles_gu = take(static_cast<size_t>(L.max_tiles_gu) * sizeof(Tile));
  L.tiles_dn = take(static_cast<size_t>(L.max_tiles_dn) * sizeof(Tile));
  L.counts = take(sizeof(TileCounts));
  F.xq_perm = take(rp * d.D / 2);
  F.xsf_perm = take(rp * d.D / 16);
  F.xq_tok = take(tp * d.D / 2);
  F.xsf_tok = take(tp * d.D / 16);
  F.hq = take(rp * d.F / 2);
  F.hsf = take(rp * d.F / 16);
  F.hsq = take(tp * d.S / 2);
  F.hssf = take(tp * d.S / 16);
  F.y = take(rp * d.D * 2);
  F.s = take(T * d.D * 4);
  F.total = o;
  L.total = o;
  return F;
}

Dims fp4_dims_of(const moe_nvfp4_params* p) {
  Dims d;
  d.T = p->T;
  d.k = p->top_k_experts;
  d.D = p->embed_dim ? p->embed_dim : MOE_EMBED_DIM;
  d.E = p->num_experts ? p->num_experts : MOE_NUM_EXPERTS;
  d.F = p->expert_dim ? p->expert_dim : MOE_EXPERT_DIM;
  d.S = p->hidden_dim ? p->hidden_dim : MOE_HIDDEN_DIM;
  d.e0 = 0;
  d.el = d.E;
  return d;
}

bool linear_ok(const moe_nvfp4_linear& l) {
  return l.q && l.sf && l.g && aligned16(l.q) && aligned16(l.sf) && aligned4(l.g);
}

moe_status check_fp4_args(const moe_nvfp4_params* p, Dims* d) {
  if (!p) return MOE_ERR_INVALID_ARG;
  *d = fp4_dims_of(p);
  if (!dims_ok(*d) || d->D > 4096) return MOE_ERR_INVALID_ARG;
  if (d->T == 0) return MOE_OK;
  if (!p->x || !p->w_router || !p->out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(p->x) || !aligned16(p->w_router) || !aligned16(p->out)) return MOE_ERR_ALIGNMENT;
  const moe_nvfp4_linear* ls[] = {&p->wg, &p->wu, &p->wd, &p->sg, &p->su, &p->sd};
  for (const moe_nvfp4_linear* l : ls)
    if (!linear_ok(*l)) return (l->q && l->sf && l->g) ? MOE_ERR_ALIGNMENT : MOE_ERR_INVALID_ARG;
  if (!(p->g_x > 0.f) || !(p->g_h > 0.f) || !(p->g_hs > 0.f)) return MOE_ERR_INVALID_ARG;
  if (p->out_f32 && !aligned16(p->out_f32)) return MOE_ERR_ALIGNMENT;
  const void* opt4[] = {p->router_bias, p->idx_out, p->w_out, p->cnt_out};
  for (const void* q : opt4)
    if (q && !aligned4(q)) return MOE_ERR_ALIGNMENT;
  const uintptr_t xb = reinterpret_cast<uintptr_t>(p->x), ob = reinterpret_cast<uintptr_t>(p->out);
  const uintptr_t bytes = static_cast<uintptr_t>(d->T) * d->D * 2;
  if (xb < ob + bytes && ob < xb + bytes) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

moe_status enqueue_block_fp4(const moe_nvfp4_params* p, const Dims& d, const Fp4Layout& F, uint8_t* ws,
                             DeviceState* s, cudaStream_t st) {
  const Layout& L = F.r;
  int32_t* idx = reinterpret_cast<int32_t*>(ws + L.idx);
  float* w = reinterpret_cast<float*>(ws + L.w);
  int32_t* cnt = reinterpret_cast<int32_t*>(ws + L.cnt);
  int32_t* off = reinterpret_cast<int32_t*>(ws + L.off);
  int32_t* row_of = reinterpret_cast<int32_t*>(ws + L.row_of);
  const uint32_t* masks = reinterpret_cast<const uint32_t*>(ws + L.masks);
  int32_t* base = reinterpret_cast<int32_t*>(ws + L.base);
  TileCounts* counts = reinterpret_cast<TileCounts*>(ws + L.counts);

  MOE_TRY(enqueue_route(d, L, ws, p->x, p->w_router, p->router_bias, idx, w, st));
  {
    LaunchScope ls_(kKRouteScan, st);
    const cudaError_t le_ = launch_k(route_scan_kernel, kScanCtas, kScanThreads, 0, st, masks, L.nchunks, d.T, d.E, d.F, d.S,
                                     d.D, base, cnt, off, reinterpret_cast<Tile*>(ws + L.tiles_gu),
                                     reinterpret_cast<Tile*>(ws + L.tiles_dn),
                                     reinterpret_cast<TileCounts*>(ws + L.counts), 1, 256, 128, 0, 0, 0, d.E);
    MOE_TRY(ls_.done(le_));
  }
  {
    const int blocks = static_cast<int>(std::min<long long>((d.T + 7) / 8, 148LL * 64));  // a warp per token
    LaunchScope ls_(kKScatterFp4, st);
    const cudaError_t le_ = launch_k(route_scatter_fp4_kernel, blocks, 256, 0, st, idx, masks, base, d.T, d.k, d.E,
                                     d.D, static_cast<const __nv_bfloat16*>(p->x), p->g_x, row_of,
                                     ws + F.xq_perm, ws + F.xsf_perm, ws + F.xq_tok, ws + F.xsf_tok,
                                     static_cast<int>(F.r_pad), s->err);
    MOE_TRY(ls_.done(le_));
  }
  const long long rp = F.r_pad, tp = F.t_pad;

  Fp4Params gu;
  std::memset(&gu, 0, sizeof(gu));
  bool ok = map_2d_u8(&gu.tmA[0], ws + F.xq_perm, rp, d.D / 2) &&
            map_3d_u8(&gu.tmB0[0], p->wg.q, d.E, d.F, d.D / 2) && map_3d_u8(&gu.tmB1[0], p->wu.q, d.E, d.F, d.D / 2) &&
            map_2d_u8(&gu.tmA[1], ws + F.xq_tok, tp, d.D / 2) && map_3d_u8(&gu.tmB0[1], p->sg.q, 1, d.S, d.D / 2) &&
            map_3d_u8(&gu.tmB1[1], p->su.q, 1, d.S, d.D / 2);
  if (!ok) return MOE_ERR_CUDA;
  gu.prob[0] = Fp4Problem{d.D,      d.F,      d.E,    static_cast<int>(rp), ws + F.xsf_perm, p->wg.sf, p->wu.sf,
                          p->wg.g,  p->wu.g,  p->g_x, ws + F.hq,            ws + F.hsf,      p->g_h,   d.F / 2, 0};
  gu.prob[1] = Fp4Problem{d.D,     d.S,     1,      static_cast<int>(tp), ws + F.xsf_tok, p->sg.sf, p->su.sf,
                          p->sg.g, p->su.g, p->g_x, ws + F.hsq,           ws + F.hssf,    p->g_hs,  d.S / 2, 0};
  gu.nprob = 2;
  gu.tiles = reinterpret_cast<const Tile*>(ws + L.tiles_gu);
  gu.num_tiles = &counts->gateup;
  gu.next_tile = &counts->next_gateup;
  gu.err = s->err;
  {
    LaunchScope ls_(kKFp4GateUp, st);
    const cudaError_t le_ =
        launch_k(fp4_gemm_kernel<true>, std::min(s->sm_count, L.max_tiles_gu), f4_threads<true>(), kF4SmemBytes, st, gu);
    MOE_TRY(ls_.done(le_));
  }

  Fp4Params dn;
  std::memset(&dn, 0, sizeof(dn));
  ok = map_2d_u8(&dn.tmA[0], ws + F.hq, rp, d.F / 2) && map_3d_u8(&dn.tmB0[0], p->wd.q, d.E, d.D, d.F / 2) &&
       map_2d_u8(&dn.tmA[1], ws + F.hsq, tp, d.S / 2) && map_3d_u8(&dn.tmB0[1], p->sd.q, 1, d.D, d.S / 2) &&
       map_3d_u8(&dn.tmBw[0], p->wd.q, d.E, d.D, d.F / 2, 256) && map_3d_u8(&dn.tmBw[1], p->sd.q, 1, d.D, d.S / 2, 256);
  if (!ok) return MOE_ERR_CUDA;
  dn.tmB1[0] = dn.tmB0[0];
  dn.tmB1[1] = dn.tmB0[1];
  float* sbuf = reinterpret_cast<float*>(ws + F.s);
  dn.prob[0] = Fp4Problem{d.F,     d.D,     d.E,    static_cast<int>(rp), ws + F.hsf, p->wd.sf, p->wd.sf,
                          p->wd.g, p->wd.g, p->g_h, ws + F.y,             nullptr,    0.f,      d.D,     0};
  dn.prob[1] = Fp4Problem{d.S,     d.D,     1,       static_cast<int>(tp), ws + F.hssf, p->sd.sf, p->sd.sf,
                          p->sd.g, p->sd.g, p->g_hs, sbuf,                 nullptr,     0.f,      d.D,     1};
  dn.nprob = 2;
  dn.tiles = reinterpret_cast<const Tile*>(ws + L.tiles_dn);
  dn.num_tiles = &counts->down;
  dn.next_tile = &counts->next_down;
  dn.err = s->err;
  {
    LaunchScope ls_(kKFp4Down, st);
    const cudaError_t le_ =
        launch_k(fp4_gemm_kernel<false>, std::min(s->sm_count, L.max_tiles_dn), f4_threads<false>(), kF4SmemBytes, st, dn);
    MOE_TRY(ls_.done(le_));
  }
  {
    LaunchScope ls_(kKCombineNorm, st);
    const cudaError_t le_ = launch_k(combine_norm_kernel, d.T, kCombThreads, 0, st, sbuf,
                                     reinterpret_cast<const __nv_bfloat16*>(ws + F.y), row_of, w, d.T, d.k, d.D,
                                     static_cast<int>(F.r_pad), p->rms_norm_out, nullptr, nullptr,
                                     static_cast<__nv_bfloat16*>(p->out), p->out_f32, s->err);
    MOE_TRY(ls_.done(le_));
  }
  const size_t R = static_cast<size_t>(d.T) * d.k;
  if (p->idx_out && cudaMemcpyAsync(p->idx_out, idx, R * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (p->w_out && cudaMemcpyAsync(p->w_out, w, R * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (p->cnt_out && cudaMemcpyAsync(p->cnt_out, cnt, d.E * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

// -------------------------------------------------- weight-only formats

size_t wq_bytes(int fmt, size_t groups, size_t K, size_t N) {
  const size_t blk = fmt == MOE_WFMT_SFP8 ? wq_block_bytes<kWfSfp8>() : wq_block_bytes<kWfQ4>();
  return groups * ((N + 127) / 128) * (K / kBK) * blk;
}

bool wq_linear_ok(int fmt, const moe_wq_linear& l) {
  return l.q && aligned16(l.q) && (fmt != MOE_WFMT_SFP8 || (l.scale && aligned4(l.scale)));
}

moe_status check_wq_args(const moe_wq_params* p, Dims* d) {
  if (!p) return MOE_ERR_INVALID_ARG;
  if (p->format != MOE_WFMT_SFP8 && p->format != MOE_WFMT_Q4_0) return MOE_ERR_INVALID_ARG;
  d->T = p->T;
  d->k = p->top_k_experts;
  d->D = p->embed_dim ? p->embed_dim : MOE_EMBED_DIM;
  d->E = p->num_experts ? p->num_experts : MOE_NUM_EXPERTS;
  d->F = p->expert_dim ? p->expert_dim : MOE_EXPERT_DIM;
  d->S = p->hidden_dim ? p->hidden_dim : MOE_HIDDEN_DIM;
  d->e0 = 0;
  d->el = d->E;
  if (!dims_ok(*d)) return MOE_ERR_INVALID_ARG;
  if (d->T == 0) return MOE_OK;
  if (!p->x || !p->w_router || !p->out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(p->x) || !aligned16(p->w_router) || !aligned16(p->out)) return MOE_ERR_ALIGNMENT;
  const moe_wq_linear* ls[] = {&p->wg, &p->wu, &p->wd, &p->sg, &p->su, &p->sd};
  for (const moe_wq_linear* l : ls)
    if (!wq_linear_ok(p->format, *l)) return (l->q && (p->format != MOE_WFMT_SFP8 || l->scale)) ? MOE_ERR_ALIGNMENT
                                                                                                 : MOE_ERR_INVALID_ARG;
  if (p->out_f32 && !aligned16(p->out_f32)) return MOE_ERR_ALIGNMENT;
  const void* opt4[] = {p->router_bias, p->idx_out, p->w_out, p->cnt_out};
  for (const void* q : opt4)
    if (q && !aligned4(q)) return MOE_ERR_ALIGNMENT;
  const uintptr_t xb = reinterpret_cast<uintptr_t>(p->x), ob = reinterpret_cast<uintptr_t>(p->out);
  const uintptr_t bytes = static_cast<uintptr_t>(d->T) * d->D * 2;
  if (xb < ob + bytes && ob < xb + bytes) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

template <int FMT, bool GATEUP>
cudaError_t launch_wq(int grid, cudaStream_t st, const WqParams& P) {
  return launch_k(wq_gemm_kernel<FMT, GATEUP>, grid, kWqThreads, kWqSmemBytes, st, P);
}

moe_status enqueue_block_wq(const moe_wq_params* p, const Dims& d, const Layout& L, uint8_t* ws, DeviceState* s,
                            cudaStream_t st) {
  const size_t R = static_cast<size_t>(d.T) * d.k;
  int32_t* idx = reinterpret_cast<int32_t*>(ws + L.idx);
  float* w = reinterpret_cast<float*>(ws + L.w);
  int32_t* cnt = reinterpret_cast<int32_t*>(ws + L.cnt);
  int32_t* off = reinterpret_cast<int32_t*>(ws + L.off);
  int32_t* row_of = reinterpret_cast<int32_t*>(ws + L.row_of);
  int32_t* token_of = reinterpret_cast<int32_t*>(ws + L.token_of);
  __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(ws + L.h);
  __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(ws + L.y);
  __nv_bfloat16* hs = reinterpret_cast<__nv_bfloat16*>(ws + L.hs);
  float* sbuf = reinterpret_cast<float*>(ws + L.s);
  __nv_bfloat16* x_perm = reinterpret_cast<__nv_bfloat16*>(ws + L.x_perm);
  TileCounts* counts = reinterpret_cast<TileCounts*>(ws + L.counts);
  const bool sfp = p->format == MOE_WFMT_SFP8;

  MOE_TRY(enqueue_route(d, L, ws, p->x, p->w_router, p->router_bias, idx, w, st));
  MOE_TRY(enqueue_permute(d, L, ws, idx, p->x, cnt, off, row_of, token_of, st, false));

  auto sc = [&](const moe_wq_linear& l) { return sfp ? l.scale : static_cast<const float*>(nullptr); };
  WqParams gu;
  std::memset(&gu, 0, sizeof(gu));
  if (!map_2d(&gu.tmA[0], x_perm, R, d.D, kBM) || !map_2d(&gu.tmA[1], p->x, d.T, d.D, kBM) ||
      !map_2d(&gu.tmAs[0], x_perm, R, d.D, kASmallRows) || !map_2d(&gu.tmAs[1], p->x, d.T, d.D, kASmallRows))
    return MOE_ERR_CUDA;
  gu.prob[0] = WqProblem{d.D, d.F, d.E, static_cast<int>(R), p->wg.q, p->wu.q, sc(p->wg), sc(p->wu), h, d.F, 0};
  gu.prob[1] = WqProblem{d.D, d.S, 1, d.T, p->sg.q, p->su.q, sc(p->sg), sc(p->su), hs, d.S, 0};
  gu.nprob = 2;
  gu.a_small = 1;
  gu.tiles = reinterpret_cast<const Tile*>(ws + L.tiles_gu);
  gu.num_tiles = &counts->gateup;
  gu.next_tile = &counts->next_gateup;
  gu.err = s->err;
  {
    LaunchScope ls_(kKGemmGateUp, st);
    const int grid = std::min(s->sm_count, L.max_tiles_gu);
    MOE_TRY(ls_.done(sfp ? launch_wq<kWfSfp8, true>(grid, st, gu) : launch_wq<kWfQ4, true>(grid, st, gu)));
  }
  WqParams dn;
  std::memset(&dn, 0, sizeof(dn));
  if (!map_2d(&dn.tmA[0], h, R, d.F, kBM) || !map_2d(&dn.tmA[1], hs, d.T, d.S, kBM) ||
      !map_2d(&dn.tmAs[0], h, R, d.F, kASmallRows) || !map_2d(&dn.tmAs[1], hs, d.T, d.S, kASmallRows))
    return MOE_ERR_CUDA;
  dn.prob[0] = WqProblem{d.F, d.D, d.E, static_cast<int>(R), p->wd.q, nullptr, sc(p->wd), nullptr, y, d.D, 0};
  dn.prob[1] = WqProblem{d.S, d.D, 1, d.T, p->sd.q, nullptr, sc(p->sd), nullptr, sbuf, d.D, 1};
  dn.nprob = 2;
  dn.a_small = 1;
  dn.tiles = reinterpret_cast<const Tile*>(ws + L.tiles_dn);
  dn.num_tiles = &counts->down;
  dn.next_tile = &counts->next_down;
  dn.err = s->err;
  {
    LaunchScope ls_(kKGemmDown, st);
    const int grid = std::min(s->sm_count, L.max_tiles_dn);
    MOE_TRY(ls_.done(sfp ? launch_wq<kWfSfp8, false>(grid, st, dn) : launch_wq<kWfQ4, false>(grid, st, dn)));
  }
  {
    LaunchScope ls_(kKCombine, st);
    const int dsplit = std::max(1, std::min(4, (2 * s->sm_count) / std::max(1, d.T)));
    MOE_TRY(ls_.done(launch_k(combine_kernel, dim3(d.T, dsplit), 128, 0, st, sbuf, y, row_of, w, d.T, d.k, d.D,
                              static_cast<int>(R), static_cast<__nv_bfloat16*>(p->out), p->out_f32, s->err)));
  }
  if (p->idx_out && cudaMemcpyAsync(p->idx_out, idx, R * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (p->w_out && cudaMemcpyAsync(p->w_out, w, R * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (p->cnt_out && cudaMemcpyAsync(p->cnt_out, cnt, d.E * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // namespace
}  // namespace moe

namespace moe {
namespace {

// Scratch of moe_route_noalloc: one fixed array per device that loads this
// library, held until the process exits. It carries the router's split-K
// partial logits and the 32-token expert bitmasks of a single call.
// Sized for moe_route's own split of the reduction at every T <= 4096: the
// router runs at most kSmCountHint (token tile, split) CTAs, so splits x T <=
// 148 x 128 and the partials take <= 148 * 128 * 128 * 4 B = 9.25 MiB, plus
// <= 64 KiB of bitmasks.
constexpr size_t kNoAllocScratchBytes = size_t(10) << 20;  // 10 MiB
constexpr int kNoAllocMaxTokens = 4096;
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];
uint8_t* g_noalloc_base[kMaxDevices] = {};
std::mutex g_noalloc_mutex;

// Device address of this device's scratch array, looked up once per device
// (the host-side symbol is only a stand-in and must never reach a kernel).
moe_status noalloc_base(uint8_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_base[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return MOE_ERR_CUDA;
    g_noalloc_base[dev] = static_cast<uint8_t*>(ptr);
  }
  *out = g_noalloc_base[dev];
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

namespace moe {
namespace {

// ------------------------------------------------------- dense GeGLU FFN

struct DenseDims {
  int T, D, S;
};

struct DenseLayout {
  size_t hs, tiles_gu, tiles_dn, counts, part, total;
  int max_gu, max_dn;
  int dn_ksplit;  // K splits of the down GEMM (1: none)
};

DenseDims dense_dims(const moe_dense_params* p) {
  return DenseDims{p->T, p->embed_dim ? p->embed_dim : MOE_E4B_EMBED_DIM,
                   p->hidden_dim ? p->hidden_dim : MOE_E4B_HIDDEN_DIM};
}

bool dense_dims_ok(const DenseDims& d) {
  return d.T >= 0 && d.D > 0 && d.S > 0 && d.D % 64 == 0 && d.S % 64 == 0 && d.D <= (1 << 20) && d.S <= (1 << 20);
}

// Small batches leave most SMs without a down tile (one 128-row block gives
// embed_dim / 256 tiles, 10 at embed_dim 2560, each streaming hidden_dim x 256
// weights): cut the reduction so that about one wave of (tile, K range) work
// items covers the device, at least 4 K blocks each. Large batches (paired
// GEMMs) never split.
int dense_down_ksplit(const DenseDims& d) {
  if (d.T >= 2 * kBM) return 1;
  const long long tiles = ((d.T + kBM - 1) / kBM) * static_cast<long long>((d.D + 255) / 256);
  const long long by_sm = kSmCountHint / std::max(1LL, tiles);
  const long long by_k = (d.S / 64) / 4;
  return static_cast<int>(std::max(1LL, std::min(by_sm, by_k)));
}

DenseLayout dense_layout(const DenseDims& d) {
  DenseLayout L{};
  const size_t mt = (static_cast<size_t>(d.T) + kBM - 1) / kBM;
  L.dn_ksplit = dense_down_ksplit(d);
  L.max_gu = static_cast<int>(std::max<size_t>(1, mt * ((d.S + 127) / 128)));
  L.max_dn = static_cast<int>(std::max<size_t>(1, mt * ((d.D + 255) / 256) * L.dn_ksplit));
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes, kAlign);
    return at;
  };
  L.hs = take(static_cast<size_t>(d.T) * d.S * 2);
  L.tiles_gu = take(static_cast<size_t>(L.max_gu) * sizeof(Tile));
  L.tiles_dn = take(static_cast<size_t>(L.max_dn) * sizeof(Tile));
  L.counts = take(sizeof(TileCounts));
  L.part = take(L.dn_ksplit > 1 ? static_cast<size_t>(L.dn_ksplit) * d.T * d.D * 4 : 0);
  L.total = o;
  return L;
}

moe_status enqueue_dense(const moe_dense_params* p, const DenseDims& d, const DenseLayout& L, uint8_t* ws,
                         DeviceState* s, cudaStream_t st) {
  __nv_bfloat16* hs = reinterpret_cast<__nv_bfloat16*>(ws + L.hs);
  TileCounts* counts = reinterpret_cast<TileCounts*>(ws + L.counts);
  // large batches: paired gate|up (two row blocks per weight stage), down on SM pairs
  const bool pairs = d.T >= 2 * kBM;
  const bool pair_dn = pairs && d.D % 128 == 0 && s->pair_clusters_dn > 0;
  {
    LaunchScope ls_(kKRouteScan, st);
    MOE_TRY(ls_.done(launch_k(dense_tiles_kernel, 1, 256, 0, st, d.T, d.S, d.D, pairs ? 1 : 0, pair_dn ? 1 : 0, 256,
                              L.dn_ksplit, reinterpret_cast<Tile*>(ws + L.tiles_gu),
                              reinterpret_cast<Tile*>(ws + L.tiles_dn), counts)));
  }
  GemmParams gu;
  std::memset(&gu, 0, sizeof(gu));
  if (!map_2d(&gu.tmA[0], p->x, d.T, d.D, kBM) || !map_3d(&gu.tmB0[0], p->wg, 1, d.D, d.S) ||
      !map_3d(&gu.tmB1[0], p->wu, 1, d.D, d.S))
    return MOE_ERR_CUDA;
  gu.prob[0] = GemmProblem{d.D, d.S, 1, d.T, hs, d.S, 0, 0};
  gu.nprob = 1;
  gu.stream_weights = d.T <= kBM ? 1 : 0;  // one row block reads each weight tile once
  gu.a_wide = pairs ? 1 : 0;
  gu.a_small = pairs ? 0 : 1;
  gu.bw_chunks = 2;
  set_wide_maps(&gu, 0, p->x, d.T, d.D, gu.a_wide, p->wg, p->wu, 1, d.S, 2);
  gu.tiles = reinterpret_cast<const Tile*>(ws + L.tiles_gu);
  gu.num_tiles = &counts->gateup;
  gu.next_tile = &counts->next_gateup;
  gu.err = s->err;
  {
    LaunchScope ls_(kKGemmGateUp, st);
    const int grid = std::min(s->sm_count, L.max_gu);
    MOE_TRY(ls_.done(pairs ? launch_k(grouped_gemm_kernel<true, true>, grid, kGemmThreadsSm, kGemmSmemBytes, st, gu)
                           : launch_k(grouped_gemm_kernel<true>, grid, kGemmThreadsSm, kGemmSmemBytes, st, gu)));
  }
  GemmParams dn;
  std::memset(&dn, 0, sizeof(dn));
  if (!map_2d(&dn.tmA[0], hs, d.T, d.S, kBM) || !map_3d(&dn.tmB0[0], p->wd, 1, d.S, d.D)) return MOE_ERR_CUDA;
  dn.tmB1[0] = dn.tmB0[0];
  // split K: the down GEMM writes fp32 partial sums per K range and a pass adds
  // them up in order and rounds; otherwise, with out_f32, it writes fp32 and a
  // pass rounds it into out; else it writes the bf16 out itself
  const bool split = L.dn_ksplit > 1;
  float* part = reinterpret_cast<float*>(ws + L.part);
  dn.prob[0] = GemmProblem{d.S, d.D, 1, d.T,
                           split ? static_cast<void*>(part)
                                 : (p->out_f32 ? static_cast<void*>(p->out_f32) : p->out),
                           d.D, (split || p->out_f32) ? 1 : 0, static_cast<long long>(d.T) * d.D};
  dn.nprob = 1;
  dn.stream_weights = gu.stream_weights;
  dn.bw_chunks = pair_dn ? 2 : 4;
  dn.a_small = pair_dn ? 0 : 1;
  set_wide_maps(&dn, 0, hs, d.T, d.S, 0, p->wd, nullptr, 1, d.D, dn.bw_chunks);
  dn.tiles = reinterpret_cast<const Tile*>(ws + L.tiles_dn);
  dn.num_tiles = &counts->down;
  dn.next_tile = &counts->next_down;
  dn.err = s->err;
  {
    LaunchScope ls_(kKGemmDown, st);
    const int grid = std::min(s->sm_count, L.max_dn);
    MOE_TRY(ls_.done(pair_dn ? launch_k(grouped_gemm_pair_kernel<false>, 2 * s->pair_clusters_dn, kGemmThreads,
                                        kP2SmemBytes, st, dn)
                             : launch_k(grouped_gemm_kernel<false>, grid, kGemmThreadsSm, kGemmSmemBytes, st, dn)));
  }
  if (split) {
    const size_t n4 = static_cast<size_t>(d.T) * d.D / 4;
    LaunchScope ls_(kKCombine, st);
    const int blocks = static_cast<int>(std::min<size_t>((n4 + 255) / 256, static_cast<size_t>(s->sm_count) * 8));
    MOE_TRY(ls_.done(launch_k(reduce_splits_kernel, blocks, 256, 0, st, static_cast<const float*>(part), L.dn_ksplit,
                              n4, p->out_f32, static_cast<__nv_bfloat16*>(p->out))));
  } else if (p->out_f32) {
    const size_t n8 = static_cast<size_t>(d.T) * d.D / 8;
    LaunchScope ls_(kKCombine, st);
    const int blocks = static_cast<int>(std::min<size_t>((n8 + 255) / 256, static_cast<size_t>(s->sm_count) * 8));
    MOE_TRY(ls_.done(launch_k(round_bf16_kernel, blocks, 256, 0, st, static_cast<const float*>(p->out_f32), n8,
                              static_cast<__nv_bfloat16*>(p->out))));
  }
  return MOE_OK;
}

}  // namespace
}  // namespace moe

extern "C" {

size_t moe_workspace_bytes_ex(const moe_params* p) {
  if (!p) return 0;
  const Dims d = dims_of(p);
  if (!dims_ok(d)) return 0;
  return make_layout(d).total;
}

size_t moe_workspace_bytes(int T, int top_k) {
  moe_params p;
  std::memset(&p, 0, sizeof(p));
  p.T = T;
  p.top_k_experts = top_k;
  return moe_workspace_bytes_ex(&p);
}

moe_status moe_workspace_layout(const moe_params* p, moe_ws_layout* out) {
  if (!p || !out) return MOE_ERR_INVALID_ARG;
  const Dims d = dims_of(p);
  if (!dims_ok(d)) return MOE_ERR_INVALID_ARG;
  const Layout L = make_layout(d);
  out->total_bytes = L.total;
  out->x_perm = L.x_perm;
  out->h = L.h;
  out->y = L.y;
  out->hs = L.hs;
  out->s = L.s;
  out->idx = L.idx;
  out->w = L.w;
  out->cnt = L.cnt;
  out->off = L.off;
  out->row_of = L.row_of;
  out->token_of = L.token_of;
  out->x_norm = L.x_norm;
  out->guard = L.guard;
  return MOE_OK;
}

moe_status moe_block_forward_ex(const moe_params* p, void* stream) {
  ApiRange nvtx_range_("moe_block_forward_ex");
  t_launches = 0;
  Dims d;
  MOE_TRY(check_block_args(p, &d));
  if (d.T == 0) return MOE_OK;
  DeviceState* s = nullptr;
  MOE_TRY(device_state(&s));
  if (!encode_fn()) return MOE_ERR_CUDA;
  const Layout L = make_layout(d);
  uint8_t* ws = nullptr;
  MOE_TRY(resolve_workspace(p, s, L, &ws));
  return enqueue_block(p, d, L, ws, s, static_cast<cudaStream_t>(stream));
}

moe_status moe_block_forward(const void* x, const void* w_router, const void* wg, const void* wu, const void* wd,
                             const void* sg, const void* su, const void* sd, int T, void* out, void* stream) {
  moe_params p;
  std::memset(&p, 0, sizeof(p));
  p.T = T;
  p.top_k_experts = MOE_TOP_K;
  p.x = x;
  p.w_router = w_router;
  p.wg = wg;
  p.wu = wu;
  p.wd = wd;
  p.sg = sg;
  p.su = su;
  p.sd = sd;
  p.out = out;
  return moe_block_forward_ex(&p, stream);
}

moe_status moe_route(const moe_params* p, int32_t* idx, float* w, void* stream) {
  ApiRange nvtx_range_("moe_route");
  t_launches = 0;
  if (!p) return MOE_ERR_INVALID_ARG;
  const Dims d = dims_of(p);
  if (!dims_ok(d)) return MOE_ERR_INVALID_ARG;
  if (d.T == 0) return MOE_OK;
  if (!p->x || !p->w_router || !idx || !w) return MOE_ERR_INVALID_ARG;
  if (!aligned16(p->x) || !aligned16(p->w_router) || !aligned4(idx) || !aligned4(w)) return MOE_ERR_ALIGNMENT;
  if ((p->router_bias && !aligned4(p->router_bias)) || (p->logits_out && !aligned4(p->logits_out)))
    return MOE_ERR_ALIGNMENT;
  DeviceState* s = nullptr;
  MOE_TRY(device_state(&s));
  if (!encode_fn()) return MOE_ERR_CUDA;
  const Layout L = make_layout(d);
  uint8_t* ws = nullptr;
  MOE_TRY(resolve_workspace(p, s, L, &ws));
  return enqueue_route(d, L, ws, p->x, p->w_router, p->router_bias, idx, w, static_cast<cudaStream_t>(stream),
                       p->logits_out);
}

moe_status moe_permute(const moe_params* p, const int32_t* idx, int32_t* cnt, int32_t* off, int32_t* row_of,
                       int32_t* token_of, void* stream) {
  ApiRange nvtx_range_("moe_permute");
  t_launches = 0;
  if (!p) return MOE_ERR_INVALID_ARG;
  const Dims d = dims_of(p);
  if (!dims_ok(d)) return MOE_ERR_INVALID_ARG;
  if (d.T == 0) return MOE_OK;
  if (!idx || !cnt || !off || !row_of || !token_of) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {idx, cnt, off, row_of, token_of};
  for (const void* q : ptrs)
    if (!aligned4(q)) return MOE_ERR_ALIGNMENT;
  DeviceState* s = nullptr;
  MOE_TRY(device_state(&s));
  const Layout L = make_layout(d);
  uint8_t* ws = nullptr;
  MOE_TRY(resolve_workspace(p, s, L, &ws));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t mask_bytes = static_cast<size_t>(L.nchunks) * d.E * 4;
  if (cudaMemsetAsync(ws + L.masks, 0, mask_bytes, st) != cudaSuccess) return MOE_ERR_CUDA;
  {
    LaunchScope ls_(kKBuildMasks, st);
    const long long R = static_cast<long long>(d.T) * d.k;
    const int blocks = static_cast<int>(std::min<long long>((R + 255) / 256, 148LL * 16));
    const cudaError_t le_ = launch_k(build_masks_kernel, blocks, 256, 0, st, idx, d.T, d.k, d.E, reinterpret_cast<uint32_t*>(ws + L.masks), s->err);
    MOE_TRY(ls_.done(le_));
  }
  return enqueue_permute(d, L, ws, idx, nullptr, cnt, off, row_of, token_of, st);
}

moe_status moe_get_device_status(void* stream) {
  DeviceState* s = nullptr;
  MOE_TRY(device_state(&s));
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, s->err, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (word) {
    if (cudaMemset(s->err, 0, sizeof(word)) != cudaSuccess) return MOE_ERR_CUDA;
    if (word & kErrWaitTimeout) return MOE_ERR_DEVICE_TIMEOUT;
    return (word & kErrGuard) ? MOE_ERR_GUARD : MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

moe_status moe_debug_timeout_probe(int timeout_us, void* stream) {
  t_launches = 0;
  if (timeout_us <= 0 || timeout_us > 10000000) return MOE_ERR_INVALID_ARG;
  DeviceState* s = nullptr;
  MOE_TRY(device_state(&s));
  {
  LaunchScope ls_(kKTimeoutProbe, static_cast<cudaStream_t>(stream));
  const cudaError_t le_ = launch_k(timeout_probe_kernel, 1, 32, 0, static_cast<cudaStream_t>(stream), 
      s->err, static_cast<unsigned long long>(timeout_us) * 1000ull);
  return ls_.done(le_);
  }
}

const char* moe_status_string(moe_status st) {
  switch (st) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_ALIGNMENT: return "MOE_ERR_ALIGNMENT";
    case MOE_ERR_ARCH: return "MOE_ERR_ARCH";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT";
    case MOE_ERR_GUARD: return "MOE_ERR_GUARD";
  }
  return "MOE_ERR_UNKNOWN";
}

int moe_last_launch_count(void) { return t_launches; }

moe_status moe_workspace_guard_check(const moe_params* p, void* stream) {
  t_launches = 0;
  ApiRange nvtx_range_("moe_workspace_guard_check");
  if (!p || !p->workspace) return MOE_ERR_INVALID_ARG;
  const Dims d = dims_of(p);
  if (!dims_ok(d)) return MOE_ERR_INVALID_ARG;
  const Layout L = make_layout(d);
  if ((reinterpret_cast<uintptr_t>(p->workspace) & (kAlign - 1)) != 0) return MOE_ERR_ALIGNMENT;
  if (p->workspace_bytes < L.total) return MOE_ERR_WORKSPACE;
  DeviceState* s = nullptr;
  MOE_TRY(device_state(&s));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  LaunchScope ls_(kKGuard, st);
  return ls_.done(launch_k(guard_check_kernel, 1, kGuardWords, 0, st,
                           reinterpret_cast<const uint32_t*>(static_cast<uint8_t*>(p->workspace) + L.guard), s->err));
}

moe_status moe_round_bf16(const float* in, void* out, size_t n, void* stream) {
  ApiRange nvtx_range_("moe_round_bf16");
  t_launches = 0;
  if (n == 0) return MOE_OK;
  if (!in || !out || n % 8) return MOE_ERR_INVALID_ARG;
  if (!aligned16(in) || !aligned16(out)) return MOE_ERR_ALIGNMENT;
  const uintptr_t ib = reinterpret_cast<uintptr_t>(in), ob = reinterpret_cast<uintptr_t>(out);
  if (ib < ob + n * 2 && ob < ib + n * 4) return MOE_ERR_INVALID_ARG;
  DeviceState* s = nullptr;
  MOE_TRY(device_state(&s));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t n8 = n / 8;
  const int blocks = static_cast<int>(std::min<size_t>((n8 + 255) / 256, static_cast<size_t>(s->sm_count) * 8));
  LaunchScope ls_(kKCombine, st);
  return ls_.done(launch_k(round_bf16_kernel, blocks, 256, 0, st, in, n8, static_cast<__nv_bfloat16*>(out)));
}

moe_status moe_block_forward_hostio(const moe_params* p, const void* x_host, void* out_host, void* stream) {
  ApiRange nvtx_range_("moe_block_forward_hostio");
  t_launches = 0;
  Dims d;
  MOE_TRY(check_block_args(p, &d));
  if (d.T == 0) return MOE_OK;
  if (!x_host || !out_host || !p->out) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t bytes = static_cast<size_t>(d.T) * d.D * 2;
  if (cudaMemcpyAsync(const_cast<void*>(p->x), x_host, bytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  DeviceState* s = nullptr;
  MOE_TRY(device_state(&s));
  if (!encode_fn()) return MOE_ERR_CUDA;
  const Layout L = make_layout(d);
  uint8_t* ws = nullptr;
  MOE_TRY(resolve_workspace(p, s, L, &ws));
  MOE_TRY(enqueue_block(p, d, L, ws, s, st));
  if (cudaMemcpyAsync(out_host, p->out, bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status moe_profile_begin(uint32_t kernel_mask) {
  t_profile_mask = kernel_mask;
  for (const ProfRecord& r : t_records) {
    t_event_pool.push_back(r.start);
    t_event_pool.push_back(r.stop);
  }
  t_records.clear();
  t_profiling = true;
  return MOE_OK;
}

int moe_profile_end(float* total_ms, int* launches, int n) {
  t_profiling = false;
  for (int i = 0; i < n; ++i) {
    if (total_ms) total_ms[i] = 0.f;
    if (launches) launches[i] = 0;
  }
  for (const ProfRecord& r : t_records) {
    float ms = 0.f;
    cudaEventSynchronize(r.stop);
    cudaEventElapsedTime(&ms, r.start, r.stop);
    if (r.id < n) {
      if (total_ms) total_ms[r.id] += ms;
      if (launches) launches[r.id] += 1;
    }
    t_event_pool.push_back(r.start);
    t_event_pool.push_back(r.stop);
  }
  t_records.clear();
  return kKCount;
}

const char* moe_kernel_name(int id) { return (id >= 0 && id < kKCount) ? kKernelNames[id] : nullptr; }

moe_status moe_route_noalloc(const moe_params* p, int32_t* idx, float* w, void* stream) {
  ApiRange nvtx_range_("moe_route_noalloc");
  t_launches = 0;
  if (!p) return MOE_ERR_INVALID_ARG;
  const Dims d = dims_of(p);
  if (!dims_ok(d)) return MOE_ERR_INVALID_ARG;
  if (d.T == 0) return MOE_OK;
  if (d.T > kNoAllocMaxTokens) return MOE_ERR_WORKSPACE;
  if (!p->x || !p->w_router || !idx || !w) return MOE_ERR_INVALID_ARG;
  if (!aligned16(p->x) || !aligned16(p->w_router) || !aligned4(idx) || !aligned4(w)) return MOE_ERR_ALIGNMENT;
  if ((p->router_bias && !aligned4(p->router_bias)) || (p->logits_out && !aligned4(p->logits_out)))
    return MOE_ERR_ALIGNMENT;
  DeviceState* s = nullptr;
  MOE_TRY(device_state(&s));
  if (!encode_fn()) return MOE_ERR_CUDA;
  uint8_t* scratch = nullptr;
  MOE_TRY(noalloc_base(&scratch));
  // Same kernels and the same split of the reduction as moe_route (so the same
  // summation order and results), with the partial logits and bitmasks placed
  // in the fixed array (the bitmasks are cleared by the router kernel).
  Layout L = make_layout(d);
  const size_t mask_bytes = align_up(static_cast<size_t>(L.nchunks) * d.E * 4, kAlign);
  const size_t partial_bytes = align_up(static_cast<size_t>(L.nsplit) * d.T * d.E * 4, kAlign);
  if (partial_bytes + mask_bytes > kNoAllocScratchBytes) return MOE_ERR_WORKSPACE;
  L.partial = 0;
  L.masks = partial_bytes;
  return enqueue_route(d, L, scratch, p->x, p->w_router, p->router_bias, idx, w, static_cast<cudaStream_t>(stream),
                       p->logits_out);
}

moe_status moe_wq_weight_bytes(int format, int groups, int K, int N, size_t* bytes) {
  if (format != MOE_WFMT_SFP8 && format != MOE_WFMT_Q4_0) return MOE_ERR_INVALID_ARG;
  if (groups <= 0 || K <= 0 || N <= 0 || K % 64 || N % 64) return MOE_ERR_INVALID_ARG;
  if (bytes) *bytes = wq_bytes(format, groups, K, N);
  return MOE_OK;
}

moe_status moe_wq_quantize_weight(int format, const void* w, int groups, int K, int N, uint8_t* q, float* scale,
                                  void* stream) {
  ApiRange nvtx_range_("moe_wq_quantize_weight");
  t_launches = 0;
  if (format != MOE_WFMT_SFP8 && format != MOE_WFMT_Q4_0) return MOE_ERR_INVALID_ARG;
  if (groups <= 0 || K <= 0 || N <= 0 || K % 64 || N % 64 || groups > 65535) return MOE_ERR_INVALID_ARG;
  const bool sfp = format == MOE_WFMT_SFP8;
  if (!w || !q || (sfp && !scale)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(q) || (sfp && !aligned4(scale))) return MOE_ERR_ALIGNMENT;
  DeviceState* s = nullptr;
  MOE_TRY(device_state(&s));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(q, 0, wq_bytes(format, groups, K, N), st) != cudaSuccess) return MOE_ERR_CUDA;
  if (sfp) {
    if (cudaMemsetAsync(scale, 0, sizeof(float) * groups, st) != cudaSuccess) return MOE_ERR_CUDA;
    const size_t per_group = static_cast<size_t>(K) * N;
    uint32_t* amax_bits = reinterpret_cast<uint32_t*>(scale);  // amax first, then the scale in place
    {
      const int bpg = static_cast<int>(std::min<size_t>((per_group / 8 + 255) / 256, 64));
      LaunchScope ls_(kKWeightAmax, st);
      MOE_TRY(ls_.done(launch_k(weight_amax_kernel, dim3(bpg, groups), 256, 0, st,
                                static_cast<const __nv_bfloat16*>(w), per_group, amax_bits)));
    }
    LaunchScope ls_(kKTensorScale, st);
    MOE_TRY(ls_.done(launch_k(sfp8_scale_kernel, (groups + 127) / 128, 128, 0, st,
                              static_cast<const uint32_t*>(amax_bits), scale, groups)));
  }
  const long long items = static_cast<long long>(N) * (K / 64);
  const dim3 grid(static_cast<unsigned>((items + 127) / 128), groups);
  LaunchScope ls_(kKWeightQuant, st);
  return ls_.done(sfp ? launch_k(wq_quant_kernel<kWfSfp8>, grid, 128, 0, st, static_cast<const __nv_bfloat16*>(w), K,
                                 N, static_cast<const float*>(scale), q)
                      : launch_k(wq_quant_kernel<kWfQ4>, grid, 128, 0, st, static_cast<const __nv_bfloat16*>(w), K,
                                 N, static_cast<const float*>(nullptr), q));
}

size_t moe_wq_workspace_bytes(const moe_wq_params* p) {
  if (!p) return 0;
  Dims d;
  d.T = p->T;
  d.k = p->top_k_experts;
  d.D = p->embed_dim ? p->embed_dim : MOE_EMBED_DIM;
  d.E = p->num_experts ? p->num_experts : MOE_NUM_EXPERTS;
  d.F = p->expert_dim ? p->expert_dim : MOE_EXPERT_DIM;
  d.S = p->hidden_dim ? p->hidden_dim : MOE_HIDDEN_DIM;
  d.e0 = 0;
  d.el = d.E;
  if (!dims_ok(d)) return 0;
  return make_layout(d).total;
}

moe_status moe_block_forward_wq(const moe_wq_params* p, void* stream) {
  ApiRange nvtx_range_("moe_block_forward_wq");
  t_launches = 0;
  Dims d;
  MOE_TRY(check_wq_args(p, &d));
  if (d.T == 0) return MOE_OK;
  DeviceState* s = nullptr;
  MOE_TRY(device_state(&s));
  if (!encode_fn()) return MOE_ERR_CUDA;
  const Layout L = make_layout(d);
  uint8_t* ws = nullptr;
  if (p->workspace) {
    if ((reinterpret_cast<uintptr_t>(p->workspace) & (kAlign - 1)) != 0) return MOE_ERR_ALIGNMENT;
    if (p->workspace_bytes < L.total) return MOE_ERR_WORKSPACE;
    ws = static_cast<uint8_t*>(p->workspace);
  } else {
    void* wsv = nullptr;
    MOE_TRY(library_workspace(s, L.total, &wsv));
    ws = static_cast<uint8_t*>(wsv);
  }
  return enqueue_block_wq(p, d, L, ws, s, static_cast<cudaStream_t>(stream));
}

moe_status moe_nvfp4_weight_bytes(int groups, int K, int N, size_t* q_bytes, size_t* sf_bytes) {
  if (groups <= 0 || K <= 0 || N <= 0 || K % 64 || N % 64) return MOE_ERR_INVALID_ARG;
  if (q_bytes) *q_bytes = fp4_q_bytes(groups, K, N);
  if (sf_bytes) *sf_bytes = fp4_sf_bytes(groups, K, N);
  return MOE_OK;
}

moe_status moe_nvfp4_quantize_weight(const void* w, int groups, int K, int N, uint8_t* q, uint8_t* sf, float* g,
                                     void* stream) {
  ApiRange nvtx_range_("moe_nvfp4_quantize_weight");
  t_launches = 0;
  if (groups <= 0 || K <= 0 || N <= 0 || K % 64 || N % 64 || groups > 65535) return MOE_ERR_INVALID_ARG;
  if (!w || !q || !sf || !g) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(q) || !aligned16(sf) || !aligned4(g)) return MOE_ERR_ALIGNMENT;
  DeviceState* s = nullptr;
  MOE_TRY(device_state(&s));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(g, 0, sizeof(float) * groups, st) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemsetAsync(sf, 0, fp4_sf_bytes(groups, K, N), st) != cudaSuccess) return MOE_ERR_CUDA;
  const size_t per_group = static_cast<size_t>(K) * N;
  uint32_t* amax_bits = reinterpret_cast<uint32_t*>(g);  // amax first, then G in place
  {
    const int bpg = static_cast<int>(std::min<size_t>((per_group / 8 + 255) / 256, 64));
    LaunchScope ls_(kKWeightAmax, st);
    const cudaError_t le_ = launch_k(weight_amax_kernel, dim3(bpg, groups), 256, 0, st,
                                     static_cast<const __nv_bfloat16*>(w), per_group, amax_bits);
    MOE_TRY(ls_.done(le_));
  }
  {
    LaunchScope ls_(kKTensorScale, st);
    const cudaError_t le_ = launch_k(tensor_scale_kernel, (groups + 127) / 128, 128, 0, st,
                                     static_cast<const uint32_t*>(amax_bits), g, groups);
    MOE_TRY(ls_.done(le_));
  }
  const long long items = static_cast<long long>(N) * (K / 16);
  LaunchScope ls_(kKWeightQuant, st);
  const cudaError_t le_ = launch_k(weight_quant_kernel, dim3(static_cast<unsigned>((items + 255) / 256), groups), 256, 0,
                                   st, static_cast<const __nv_bfloat16*>(w), K, N, static_cast<const float*>(g), q, sf);
  return ls_.done(le_);
}

moe_status moe_nvfp4_quantize_act(const void* x, int rows, int K, float g, uint8_t* q, uint8_t* sf, void* stream) {
  ApiRange nvtx_range_("moe_nvfp4_quantize_act");
  t_launches = 0;
  if (rows < 0 || K <= 0 || K % 64 || !(g > 0.f)) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (!x || !q || !sf) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(q)) return MOE_ERR_ALIGNMENT;
  DeviceState* s = nullptr;
  MOE_TRY(device_state(&s));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int blocks = std::min((rows + 7) / 8, s->sm_count * 16);
  LaunchScope ls_(kKActQuant, st);
  const cudaError_t le_ =
      launch_k(act_quant_kernel, blocks, 256, 0, st, static_cast<const __nv_bfloat16*>(x), rows, K, g, q, sf);
  return ls_.done(le_);
}

size_t moe_nvfp4_workspace_bytes(const moe_nvfp4_params* p) {
  if (!p) return 0;
  const Dims d = fp4_dims_of(p);
  if (!dims_ok(d)) return 0;
  return make_fp4_layout(d).total;
}

moe_status moe_nvfp4_workspace_layout(const moe_nvfp4_params* p, moe_nvfp4_ws_layout* out) {
  if (!p || !out) return MOE_ERR_INVALID_ARG;
  const Dims d = fp4_dims_of(p);
  if (!dims_ok(d)) return MOE_ERR_INVALID_ARG;
  const Fp4Layout F = make_fp4_layout(d);
  out->total_bytes = F.total;
  out->xq_perm = F.xq_perm;
  out->xsf_perm = F.xsf_perm;
  out->xq_tok = F.xq_tok;
  out->xsf_tok = F.xsf_tok;
  out->hq = F.hq;
  out->hsf = F.hsf;
  out->hsq = F.hsq;
  out->hssf = F.hssf;
  out->y = F.y;
  out->s = F.s;
  out->idx = F.r.idx;
  out->w = F.r.w;
  out->cnt = F.r.cnt;
  out->off = F.r.off;
  out->row_of = F.r.row_of;
  out->routed_rows = F.r_pad;
  out->token_rows = F.t_pad;
  return MOE_OK;
}

moe_status moe_block_forward_nvfp4(const moe_nvfp4_params* p, void* stream) {
  ApiRange nvtx_range_("moe_block_forward_nvfp4");
  t_launches = 0;
  Dims d;
  MOE_TRY(check_fp4_args(p, &d));
  if (d.T == 0) return MOE_OK;
  DeviceState* s = nullptr;
  MOE_TRY(device_state(&s));
  if (!encode_fn()) return MOE_ERR_CUDA;
  const Fp4Layout F = make_fp4_layout(d);
  uint8_t* ws = nullptr;
  if (p->workspace) {
    if ((reinterpret_cast<uintptr_t>(p->workspace) & (kAlign - 1)) != 0) return MOE_ERR_ALIGNMENT;
    if (p->workspace_bytes < F.total) return MOE_ERR_WORKSPACE;
    ws = static_cast<uint8_t*>(p->workspace);
  } else {
    void* wsv = nullptr;
    MOE_TRY(library_workspace(s, F.total, &wsv));
    ws = static_cast<uint8_t*>(wsv);
  }
  return enqueue_block_fp4(p, d, F, ws, s, static_cast<cudaStream_t>(stream));
}

moe_status moe_nvfp4_calibrate(const moe_params* p, float* amax, float* scales, void* stream) {
  ApiRange nvtx_range_("moe_nvfp4_calibrate");
  t_launches = 0;
  Dims d;
  MOE_TRY(check_block_args(p, &d));
  if (!amax || !scales || !p->workspace) return MOE_ERR_INVALID_ARG;
  if (!aligned4(amax) || !aligned4(scales)) return MOE_ERR_ALIGNMENT;
  if (amax < scales + 3 && scales < amax + 3) return MOE_ERR_INVALID_ARG;
  DeviceState* s = nullptr;
  MOE_TRY(device_state(&s));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(amax, 0, 3 * sizeof(float), st) != cudaSuccess) return MOE_ERR_CUDA;
  if (d.T == 0) {
    LaunchScope ls_(kKTensorScale, st);
    return ls_.done(launch_k(tensor_scale_kernel, 1, 32, 0, st, reinterpret_cast<const uint32_t*>(amax), scales, 3));
  }
  if (!encode_fn()) return MOE_ERR_CUDA;
  const Layout L = make_layout(d);
  uint8_t* ws = nullptr;
  MOE_TRY(resolve_workspace(p, s, L, &ws));
  MOE_TRY(enqueue_block(p, d, L, ws, s, st));
  const size_t R = static_cast<size_t>(d.T) * d.k;
  const void* srcs[3] = {p->norm_pre ? ws + L.x_norm : p->x, ws + L.h, ws + L.hs};
  const size_t ns[3] = {static_cast<size_t>(d.T) * d.D, R * d.F, static_cast<size_t>(d.T) * d.S};
  for (int i = 0; i < 3; ++i) {
    const int blocks = static_cast<int>(std::min<size_t>((ns[i] / 8 + 255) / 256, static_cast<size_t>(s->sm_count) * 8));
    LaunchScope ls_(kKAmax, st);
    const cudaError_t le_ = launch_k(amax_bf16_kernel, blocks, 256, 0, st, static_cast<const __nv_bfloat16*>(srcs[i]),
                                     ns[i], reinterpret_cast<uint32_t*>(amax) + i);
    MOE_TRY(ls_.done(le_));
  }
  // the three tensor scales G = 448 * 6 / amax (1 for an all-zero tensor)
  LaunchScope ls_(kKTensorScale, st);
  return ls_.done(launch_k(tensor_scale_kernel, 1, 32, 0, st, reinterpret_cast<const uint32_t*>(amax), scales, 3));
}

size_t moe_dense_workspace_bytes(const moe_dense_params* p) {
  if (!p) return 0;
  const DenseDims d = dense_dims(p);
  if (!dense_dims_ok(d)) return 0;
  return dense_layout(d).total;
}

moe_status moe_dense_ffn_forward(const moe_dense_params* p, void* stream) {
  ApiRange nvtx_range_("moe_dense_ffn_forward");
  t_launches = 0;
  if (!p) return MOE_ERR_INVALID_ARG;
  const DenseDims d = dense_dims(p);
  if (!dense_dims_ok(d)) return MOE_ERR_INVALID_ARG;
  if (d.T == 0) return MOE_OK;
  const void* req[] = {p->x, p->wg, p->wu, p->wd, p->out};
  for (const void* q : req)
    if (!q) return MOE_ERR_INVALID_ARG;
  for (const void* q : req)
    if (!aligned16(q)) return MOE_ERR_ALIGNMENT;
  if (p->out_f32 && !aligned16(p->out_f32)) return MOE_ERR_ALIGNMENT;
  const uintptr_t xb = reinterpret_cast<uintptr_t>(p->x), ob = reinterpret_cast<uintptr_t>(p->out);
  const uintptr_t bytes = static_cast<uintptr_t>(d.T) * d.D * 2;
  if (xb < ob + bytes && ob < xb + bytes) return MOE_ERR_INVALID_ARG;
  DeviceState* s = nullptr;
  MOE_TRY(device_state(&s));
  if (!encode_fn()) return MOE_ERR_CUDA;
  const DenseLayout L = dense_layout(d);
  uint8_t* ws = nullptr;
  if (p->workspace) {
    if ((reinterpret_cast<uintptr_t>(p->workspace) & (kAlign - 1)) != 0) return MOE_ERR_ALIGNMENT;
    if (p->workspace_bytes < L.total) return MOE_ERR_WORKSPACE;
    ws = static_cast<uint8_t*>(p->workspace);
  } else {
    void* w = nullptr;
    MOE_TRY(library_workspace(s, L.total, &w));
    ws = static_cast<uint8_t*>(w);
  }
  return enqueue_dense(p, d, L, ws, s, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
