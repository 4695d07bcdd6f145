// lt_api.cu -- the device entry points of the C ABI declared in include/lt.h:
// argument checks, TMA descriptors and kernel launches.  Nothing here
// allocates device memory or synchronises (except lt_device_status).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include <atomic>
#include <algorithm>
#include <climits>
#include <cmath>
#include <cstring>
#include <mutex>
#include <queue>
#include <utility>
#include <vector>

#include "attn_fwd.cuh"
#include "attn_fwd64.cuh"
#include "compact_kv.cuh"
#include "dqueue.cuh"
#include "lazy_ratio.cuh"
#include "selftest.cuh"
#include "decode.cuh"
#include "lt.h"

namespace {

// One NVTX range per library call, named after the entry point, so that a
// profiler's timeline and `ncu --nvtx` filters show which call enqueued which
// kernels.  Host side only (a graph replay runs none of it); with no tool
// attached each push/pop is a call through a no-op pointer.
struct CallRange {
  explicit CallRange(const char* name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
  CallRange(const CallRange&) = delete;
  CallRange& operator=(const CallRange&) = delete;
};
#define LT_RANGE() const CallRange lt_call_range_(__func__)

// Device status word: bit lt::kErrTimeout is set by a kernel that gave up a
// bounded wait.  One copy per device; read and cleared by lt_device_status.
__device__ unsigned g_status_word;

// Workspace of lt_decode_attn_splitk_noalloc: a fixed array in the library's
// own device memory, for callers that cannot allocate.  Every device that
// loads the library holds it until the process exits; every call on a device
// shares it.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;   // 4 MiB
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int sm_count = 0;
  unsigned* status = nullptr;  // device address of g_status_word
  int max_decode_splits = 8;   // largest cluster the decode kernels launch with
  int max_ratio_cluster = 8;   // largest cluster the separate ratio pass launches with
  // The head_dim-128 attention kernels move registers between warpgroups with
  // setmaxnreg, which is only safe when the compiled kernels launch with the
  // per-thread count the split was computed from (else a raise could wait
  // forever); checked once per device.
  bool attn128_regs_ok = false;
  // Device address of g_noalloc_scratch (host code may not use the symbol
  // itself: on the host it names a stand-in, not device memory).
  float* noalloc_scratch = nullptr;
};

std::mutex g_mutex;
DeviceInfo g_devices[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Per-device set-up, once, with the device current.
lt_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LT_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& info = g_devices[dev];
  if (!info.ready) {
    if (cudaDeviceGetAttribute(&info.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return LT_ERR_CUDA;
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_status_word) != cudaSuccess) return LT_ERR_CUDA;
    info.status = static_cast<unsigned*>(addr);
    void* scratch = nullptr;
    if (cudaGetSymbolAddress(&scratch, g_noalloc_scratch) != cudaSuccess || !scratch) return LT_ERR_CUDA;
    info.noalloc_scratch = static_cast<float*>(scratch);
    if (cudaFuncSetAttribute(lt::attn_fwd64_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             lt::Attn64Layout::kAlloc) != cudaSuccess ||
        cudaFuncSetAttribute(lt::attn_fwd_kernel<128, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             lt::AttnLayout<128>::kAlloc) != cudaSuccess ||
        cudaFuncSetAttribute(lt::attn_fwd64_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             lt::Attn64Layout::kAlloc) != cudaSuccess ||
        cudaFuncSetAttribute(lt::attn_fwd_kernel<128, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             lt::AttnLayout<128>::kAlloc) != cudaSuccess ||
        cudaFuncSetAttribute(lt::lazy_ratio_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             lt::RatioLayout<64>::kBytes) != cudaSuccess ||
        cudaFuncSetAttribute(lt::lazy_ratio_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             lt::RatioLayout<128>::kBytes) != cudaSuccess)
      return LT_ERR_CUDA;
    {
      cudaFuncAttributes fa0{}, fa1{};
      info.attn128_regs_ok =
          cudaFuncGetAttributes(&fa0, lt::attn_fwd_kernel<128, false>) == cudaSuccess &&
          cudaFuncGetAttributes(&fa1, lt::attn_fwd_kernel<128, true>) == cudaSuccess &&
          fa0.numRegs == lt::AttnLayout<128>::kLaunchRegs && fa1.numRegs == lt::AttnLayout<128>::kLaunchRegs &&
          2 * lt::AttnLayout<128>::kRegsSoftmax + lt::AttnLayout<128>::kRegsOther ==
              3 * lt::AttnLayout<128>::kLaunchRegs;
    }
    // Clusters of 16 CTAs are beyond the portable size: use them for the decode
    // split only where the device reports that one fits.
    info.max_decode_splits = 8;
    if (cudaFuncSetAttribute(lt::decode_kernel<64>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
            cudaSuccess &&
        cudaFuncSetAttribute(lt::decode_kernel<128>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
            cudaSuccess) {
      int fits64 = 0, fits128 = 0;
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = lt::kDecodeMaxSplits;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(lt::kDecodeMaxSplits, 1, 1);
      cfg.blockDim = dim3(lt::kDecodeThreads, 1, 1);
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&fits64, lt::decode_kernel<64>, &cfg) == cudaSuccess &&
          cudaOccupancyMaxActiveClusters(&fits128, lt::decode_kernel<128>, &cfg) == cudaSuccess && fits64 > 0 &&
          fits128 > 0)
        info.max_decode_splits = lt::kDecodeMaxSplits;
    }
    // The same for the separate ratio pass: one cluster per (sequence, query
    // head), up to 16 CTAs where the device fits such clusters.
    info.max_ratio_cluster = 8;
    if (lt::kRatioMaxCluster > 8 &&
        cudaFuncSetAttribute(lt::lazy_ratio_kernel<64>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
            cudaSuccess &&
        cudaFuncSetAttribute(lt::lazy_ratio_kernel<128>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
            cudaSuccess) {
      int fits64 = 0, fits128 = 0;
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = lt::kRatioMaxCluster;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(lt::kRatioMaxCluster, 1, 1);
      cfg.blockDim = dim3(32 * lt::kRatioWarps, 1, 1);
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      cfg.dynamicSmemBytes = lt::RatioLayout<64>::kBytes;
      const bool q64 = cudaOccupancyMaxActiveClusters(&fits64, lt::lazy_ratio_kernel<64>, &cfg) == cudaSuccess;
      cfg.dynamicSmemBytes = lt::RatioLayout<128>::kBytes;
      const bool q128 = cudaOccupancyMaxActiveClusters(&fits128, lt::lazy_ratio_kernel<128>, &cfg) == cudaSuccess;
      if (q64 && q128 && fits64 > 0 && fits128 > 0) info.max_ratio_cluster = lt::kRatioMaxCluster;
    }
    cudaGetLastError();   // a refused query above is not an error of a later call
    info.ready = true;
  }
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return LT_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  *out = &info;
  return LT_OK;
}

bool aligned(const void* p, uintptr_t a) { return p && (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Common checks of a packed-batch shape.
lt_status check_shape(const lt_shape* s) {
  if (!s) return LT_ERR_INVALID_ARG;
  if (s->batch < 1 || s->total_tokens < 0 || s->max_seqlen < 0 || s->hq < 1 || s->hkv < 1) return LT_ERR_INVALID_ARG;
  if (s->hq % s->hkv != 0) return LT_ERR_INVALID_ARG;
  if (!s->cu_seqlens && s->batch != 1) return LT_ERR_INVALID_ARG;
  if (s->cu_seqlens && !aligned(s->cu_seqlens, 4)) return LT_ERR_INVALID_ARG;
  if (s->head_dim != 64 && s->head_dim != 128) return LT_ERR_UNSUPPORTED;
  // Element offsets are computed in 64 bits, but token indices are int.
  if ((long long)s->total_tokens * s->hq * s->head_dim > (1LL << 40)) return LT_ERR_INVALID_ARG;
  return LT_OK;
}

// 3-D tensor map over a [T, heads, d] bf16 tensor: box of 128 rows x 64 columns
// of one head, 128-byte swizzle (the layout the MMA descriptors expect).
lt_status make_map(CUtensorMap* map, const void* base, int d, int heads, int T) {
  cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(heads), cuuint64_t(T)};
  cuuint64_t strides[2] = {cuuint64_t(d) * 2, cuuint64_t(heads) * d * 2};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t estride[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                        estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LT_OK : LT_ERR_CUDA;
}

// Launch with programmatic stream serialization: the kernel may be launched
// while the previous kernel in the stream is finishing; it waits (pdl_wait)
// before touching memory the previous kernel may use.  Used for the kernels of
// the prefill loop, whose launch gaps are otherwise a few microseconds each.
template <typename... ExpTypes, typename... ActTypes>
cudaError_t launch_pdl(void (*kernel)(ExpTypes...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       ActTypes&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<ActTypes>(args)...);
}

float resolve_scale(float softmax_scale, int d) {
  return softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(float(d));
}

constexpr float kLog2e = 1.4426950408889634f;

// Long prefills: the attention's work items in q-tile bands, KV head by KV head.
constexpr bool kBandedOrder = true;
// Packed batches: the attention's work items sequence by sequence, KV head by KV head.
constexpr bool kSeqMajorOrder = true;
// Split-K decode: caches longer than this take the two-CTAs-a-SM kernel
// (measured faster from 32 768 rows on, slower at 4096).
constexpr int kDecodeSplitKDense = 8192;
// Short single-sequence prefills: the static longest-first item schedule below.
constexpr bool kStaticSchedule = true;

// Static longest-first schedule of the attention's work items (one sequence,
// a few items per CTA).  The cost model counts quarter key-tile times: both
// tiles of an item run side by side (one per softmax warpgroup), so a pair of
// heads on q-tile qt costs its qt + 1 key tiles, and two q-tiles of one head
// the mean of theirs; every item adds one tile's worth of fixed work (Q load,
// epilogue).  With the fused ratio, each key tile that holds a sink or the
// first window key of an observed row counts two tiles more: its masked pass
// over the scores plus the ratio steps of the other tiles of that item.  The
// weight was measured (fused launch per layer, one process, alternating
// builds): 1/2, 1, 2 and 4 extra tiles gave 111.1, 111.0, 109.2 and 111.1 us
// on a gqa1p2b layer (head_dim 64); 1/4, 1/2, 1 and 2 gave 148.0, 146.1, 144.1
// and 142.5 us on a 4096-token head_dim-128 layer.
struct ScheduleKey {
  int d, fused, n_qtiles, len, hq, pair, S, W, n_obs, grid, num_items;
  bool operator==(const ScheduleKey& o) const {
    return d == o.d && fused == o.fused && n_qtiles == o.n_qtiles && len == o.len && hq == o.hq &&
           pair == o.pair && S == o.S && W == o.W && n_obs == o.n_obs && grid == o.grid &&
           num_items == o.num_items;
  }
};

// Key tiles of q-tile qt (rows qt*128 .. min(len, qt*128+128) - 1) whose
// scores the fused ratio sums by a per-key mask: those below S (the sinks)
// and, for each observed row i, the tile holding key i - W + 1 when that key
// is not the tile's first.
int masked_tiles(int qt, int len, int S, int W, int n_obs) {
  const int obs_lo = len - std::min(n_obs, len);
  const int r0 = std::max(qt * 128, obs_lo), r1 = std::min(len, qt * 128 + 128) - 1;
  if (r0 > r1) return 0;
  int count = std::min((S + 127) / 128, qt + 1);
  int last = -1;
  for (int i = r0; i <= r1; ++i) {
    const int w = i - W + 1;
    if (w <= 0 || (w & 127) == 0) continue;
    const int j = w / 128;
    if (j == last || j * 128 < S) continue;
    count += 1;
    last = j;
  }
  return count;
}

int64_t item_cost(const ScheduleKey& k, int t) {
  const int mw = k.fused ? 8 : 0;
  if (k.pair) {
    const int qt = k.n_qtiles - 1 - t / (k.hq / 2);
    if (qt * 128 >= k.len) return 0;
    return 4LL * (qt + 1) + 4 + (mw ? mw * masked_tiles(qt, k.len, k.S, k.W, k.n_obs) : 0);
  }
  const int npairs = (k.n_qtiles + 1) / 2;
  const int qp = npairs - 1 - t / k.hq;
  const int t1 = 2 * qp + 1, t0 = 2 * qp;
  if (t0 * 128 >= k.len) return 0;
  int64_t c = 4 + (t1 * 128 < k.len ? 2LL * (t1 + 1 + t0 + 1) : 4LL * (t0 + 1));
  if (mw) {
    c += mw * masked_tiles(t0, k.len, k.S, k.W, k.n_obs);
    if (t1 * 128 < k.len) c += mw * masked_tiles(t1, k.len, k.S, k.W, k.n_obs);
  }
  return c;
}

// Fills `out` with the longest-first assignment when its slowest CTA is
// cheaper than the snake order's; otherwise out.used = 0.
void build_schedule(const ScheduleKey& k, lt::AttnSchedule& out) {
  out.used = 0;
  const int n = k.num_items, G = k.grid;
  std::vector<int64_t> cost(n);
  for (int t = 0; t < n; ++t) cost[t] = item_cost(k, t);
  int64_t snake_max = 0;
  for (int c = 0; c < G; ++c) {
    int64_t load = 0;
    for (int r = 0; r * G < n; ++r) {
      const int t = r * G + ((r & 1) ? (G - 1 - c) : c);
      if (t < n) load += cost[t];
    }
    snake_max = std::max(snake_max, load);
  }
  std::vector<int> order(n);
  for (int t = 0; t < n; ++t) order[t] = t;
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return cost[a] > cost[b]; });
  // Least-loaded CTA first, the lower index on ties.
  using Slot = std::pair<int64_t, int>;
  std::priority_queue<Slot, std::vector<Slot>, std::greater<Slot>> heap;
  for (int c = 0; c < G; ++c) heap.push({0, c});
  std::vector<std::vector<int>> per(G);
  int64_t lpt_max = 0;
  for (int t : order) {
    Slot sl = heap.top();
    heap.pop();
    per[sl.second].push_back(t);
    sl.first += cost[t];
    lpt_max = std::max(lpt_max, sl.first);
    heap.push(sl);
  }
  if (lpt_max >= snake_max) return;
  int pos = 0;
  for (int c = 0; c < G; ++c) {
    out.off[c] = uint16_t(pos);
    for (int t : per[c]) out.item[pos++] = uint16_t(t);
  }
  out.off[G] = uint16_t(pos);
  out.used = 1;
}

// The schedule for a launch: the snake order (used = 0) unless the launch is
// one sequence of known length with at most kSchedMaxItems items; the last
// shape's schedule is kept per host thread.
// The attention launch's work items: q-tile bands (see attn_decode) and the
// item count.  A single sequence with at least two bands of q-tiles takes bands
// of about one wave of the grid on one KV head (6.9% faster on a 131 072-token
// sequence); shorter single sequences keep the plain heaviest-first order,
// which balances their tail.  A packed batch (even group) takes one band per
// sequence: sequence by sequence, KV head by KV head (9.5% faster on the
// batched workload; bands of one wave with the sequences interleaved measured
// 5.6% slower, their waves partly empty with sequences of different lengths).
struct AttnPlan {
  bool pair_heads;
  long long n_qtiles, qt_band, num_items;
};
AttnPlan attn_plan(int batch, int hq, int hkv, int max_len, int sm_count) {
  AttnPlan pl;
  const int group = hq / hkv;
  pl.n_qtiles = (max_len + 127) / 128;
  pl.pair_heads = (group % 2) == 0;
  pl.qt_band = 0;
  if (pl.pair_heads && kBandedOrder && batch == 1) {
    const long long band = std::max<long long>(1, sm_count / ((long long)batch * (group / 2)));
    if (pl.n_qtiles >= 2 * band) pl.qt_band = band;
  } else if (pl.pair_heads && kSeqMajorOrder && batch > 1) {
    // Packed batch: one band of all q-tiles per sequence, i.e. sequence by
    // sequence and within one KV head by KV head.
    pl.qt_band = pl.n_qtiles;
  }
  if (pl.qt_band > 0)
    pl.num_items = ((pl.n_qtiles + pl.qt_band - 1) / pl.qt_band) * pl.qt_band * hkv * batch * (group / 2);
  else
    pl.num_items = pl.pair_heads ? pl.n_qtiles * batch * (hq / 2) : ((pl.n_qtiles + 1) / 2) * batch * hq;
  return pl;
}

const lt::AttnSchedule& attn_schedule(const ScheduleKey& k, bool eligible) {
  static thread_local lt::AttnSchedule none = [] {
    lt::AttnSchedule z;
    std::memset(&z, 0, sizeof(z));
    return z;
  }();
  if (!eligible || k.num_items <= k.grid || k.num_items > lt::kSchedMaxItems || k.grid > lt::kSchedMaxCtas)
    return none;
  static thread_local ScheduleKey last{};
  static thread_local bool have = false;
  static thread_local lt::AttnSchedule sched;
  if (!have || !(last == k)) {
    std::memset(&sched, 0, sizeof(sched));
    build_schedule(k, sched);
    last = k;
    have = true;
  }
  return sched;
}

}  // namespace

extern "C" {

// Shared by lt_prefill_attn and lt_prefill_attn_ratio: checks, descriptors,
// launch.  `ratio` null selects the plain attention kernel.
static bool dq_args(const void* state, int L, int batch);
static int dq_blocks(int batch);

static lt_status launch_attention(const lt_shape* shape, const void* Q, const void* K, const void* V, void* O,
                                  float* LSE, float softmax_scale, int S, int W, int n_obs, float* ratio,
                                  lt_stream stream, bool zero_ratio = true, void* dq_state = nullptr,
                                  int dq_L = 0, int dq_layer = 0) {
  lt_status st = check_shape(shape);
  if (st != LT_OK) return st;
  if (!std::isfinite(softmax_scale)) return LT_ERR_INVALID_ARG;
  if (ratio && (!aligned(ratio, 4) || S < 0 || W < 0 || (long long)S + W < 1 || n_obs < 1 || n_obs > 4096))
    return LT_ERR_INVALID_ARG;
  const int T = shape->total_tokens;
  const int max_len = shape->cu_seqlens ? shape->max_seqlen : T;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (T > 0 && (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16) || !aligned(LSE, 4)))
    return LT_ERR_INVALID_ARG;
  if (dq_state && (!ratio || !dq_args(dq_state, dq_L, shape->batch) || dq_layer < 0 || dq_layer >= dq_L))
    return LT_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  if (ratio && zero_ratio) {
    // The kernel adds each tile's share of the mean; sequences without tokens keep 0.
    if ((st = device_info(&dev)) != LT_OK) return st;
    const int n = shape->batch * shape->hq;
    if (launch_pdl(lt::zero_f32_kernel, dim3((n + 255) / 256), dim3(256), 0, s, ratio, n) != cudaSuccess)
      return LT_ERR_CUDA;
  }
  if (T == 0 || max_len == 0) {
    // Nothing to read or write; the queue still takes the layer (all ratios 0).
    if (!dq_state) return LT_OK;
    const cudaError_t e = launch_pdl(lt::dqueue_push_kernel, dim3(dq_blocks(shape->batch)), dim3(128), 0, s,
                                     dq_state, dq_L, shape->batch, dq_layer, static_cast<const float*>(ratio),
                                     shape->hq, 1);
    return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? LT_OK : LT_ERR_CUDA;
  }
  const int group = shape->hq / shape->hkv;
  if (!dev && (st = device_info(&dev)) != LT_OK) return st;
  const AttnPlan plan = attn_plan(shape->batch, shape->hq, shape->hkv, max_len, dev->sm_count);
  const long long n_qtiles = plan.n_qtiles, qt_band = plan.qt_band, num_items = plan.num_items;
  const bool pair_heads = plan.pair_heads;
  if (num_items > INT_MAX) return LT_ERR_INVALID_ARG;

  const int d = shape->head_dim;
  if (d == 128 && !dev->attn128_regs_ok) return LT_ERR_UNSUPPORTED;
  CUtensorMap mq, mk, mv;
  if (make_map(&mq, Q, d, shape->hq, T) != LT_OK || make_map(&mk, K, d, shape->hkv, T) != LT_OK ||
      make_map(&mv, V, d, shape->hkv, T) != LT_OK)
    return LT_ERR_INVALID_ARG;

  lt::AttnParams p;
  p.batch = shape->batch;
  p.total_tokens = T;
  p.hq = shape->hq;
  p.hkv = shape->hkv;
  p.group = group;
  p.n_qtiles = int(n_qtiles);
  p.pair_heads = pair_heads ? 1 : 0;
  p.qt_band = int(qt_band);
  p.num_items = int(num_items);
  p.cu_seqlens = shape->cu_seqlens;
  p.O = static_cast<__nv_bfloat16*>(O);
  p.LSE = LSE;
  p.scale_log2 = resolve_scale(softmax_scale, d) * kLog2e;
  p.status = dev->status;
  p.ratio = ratio;
  p.S = S;
  p.W = W;
  p.n_obs = n_obs;
  p.dq_state = dq_state;
  p.dq_L = dq_L;
  p.dq_layer = dq_layer;
  const int grid = int(num_items < dev->sm_count ? num_items : dev->sm_count);
  // A single sequence whose length the host knows (no cu_seqlens) and whose
  // items are not banded may take the static schedule.
  const ScheduleKey key{d, ratio ? 1 : 0, int(n_qtiles), T, shape->hq, pair_heads ? 1 : 0, S, W, n_obs, grid,
                        int(num_items)};
  const lt::AttnSchedule& sched =
      attn_schedule(key, kStaticSchedule && shape->batch == 1 && !shape->cu_seqlens && qt_band == 0);
  cudaError_t e;
  if (d == 64) {
    constexpr int kThreads = lt::Attn64Layout::kThreads, kSmem = lt::Attn64Layout::kAlloc;
    if (ratio)
      e = launch_pdl(lt::attn_fwd64_kernel<true>, dim3(grid), dim3(kThreads), kSmem, s, mq, mk, mv, p, sched);
    else
      e = launch_pdl(lt::attn_fwd64_kernel<false>, dim3(grid), dim3(kThreads), kSmem, s, mq, mk, mv, p, sched);
  } else {
    constexpr int kThreads = lt::AttnLayout<128>::kThreads, kSmem = lt::AttnLayout<128>::kAlloc;
    if (ratio)
      e = launch_pdl(lt::attn_fwd_kernel<128, true>, dim3(grid), dim3(kThreads), kSmem, s, mq, mk, mv, p, sched);
    else
      e = launch_pdl(lt::attn_fwd_kernel<128, false>, dim3(grid), dim3(kThreads), kSmem, s, mq, mk, mv, p, sched);
  }
  return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? LT_OK : LT_ERR_CUDA;
}

lt_status lt_attn_schedule(int head_dim, int fused, int len, int hq, int hkv, int S, int W, int n_obs, int grid,
                           int* used, int* num_items, int32_t* off, int32_t* item, int capacity) {
  LT_RANGE();
  if (!used || !num_items || (head_dim != 64 && head_dim != 128) || len < 1 || hq < 1 || hkv < 1 ||
      hq % hkv != 0 || grid < 1 || capacity < 0)
    return LT_ERR_INVALID_ARG;
  if (fused && (S < 0 || W < 0 || (long long)S + W < 1 || n_obs < 1 || n_obs > 4096)) return LT_ERR_INVALID_ARG;
  const AttnPlan plan = attn_plan(1, hq, hkv, len, grid);
  if (plan.num_items > INT_MAX) return LT_ERR_INVALID_ARG;
  *num_items = int(plan.num_items);
  *used = 0;
  const int g = int(plan.num_items < grid ? plan.num_items : grid);
  const ScheduleKey key{head_dim, fused ? 1 : 0, int(plan.n_qtiles), len, hq, plan.pair_heads ? 1 : 0,
                        fused ? S : 0, fused ? W : 0, fused ? n_obs : 0, g, int(plan.num_items)};
  const lt::AttnSchedule& sched = attn_schedule(key, kStaticSchedule && plan.qt_band == 0);
  if (!sched.used) return LT_OK;
  *used = 1;
  if (!off || !item || capacity < plan.num_items) return LT_ERR_INVALID_ARG;
  for (int c = 0; c <= g; ++c) off[c] = sched.off[c];
  for (long long t = 0; t < plan.num_items; ++t) item[t] = sched.item[t];
  return LT_OK;
}

lt_status lt_prefill_attn(const lt_shape* shape, const void* Q, const void* K, const void* V, void* O, float* LSE,
                          float softmax_scale, lt_stream stream) {
  LT_RANGE();
  return launch_attention(shape, Q, K, V, O, LSE, softmax_scale, 0, 0, 0, nullptr, stream);
}

lt_status lt_prefill_attn_ratio(const lt_shape* shape, const void* Q, const void* K, const void* V, void* O,
                                float* LSE, float softmax_scale, int S, int W, int n_obs, float* ratio,
                                lt_stream stream) {
  LT_RANGE();
  if (!ratio) return LT_ERR_INVALID_ARG;
  return launch_attention(shape, Q, K, V, O, LSE, softmax_scale, S, W, n_obs, ratio, stream);
}

lt_status lt_prefill_attn_ratio_acc(const lt_shape* shape, const void* Q, const void* K, const void* V, void* O,
                                    float* LSE, float softmax_scale, int S, int W, int n_obs, float* ratio,
                                    lt_stream stream) {
  LT_RANGE();
  if (!ratio) return LT_ERR_INVALID_ARG;
  return launch_attention(shape, Q, K, V, O, LSE, softmax_scale, S, W, n_obs, ratio, stream, false);
}

lt_status lt_prefill_attn_ratio_push(const lt_shape* shape, const void* Q, const void* K, const void* V, void* O,
                                     float* LSE, float softmax_scale, int S, int W, int n_obs, float* ratio,
                                     void* state, int L, int layer, lt_stream stream) {
  LT_RANGE();
  if (!ratio || !state) return LT_ERR_INVALID_ARG;
  return launch_attention(shape, Q, K, V, O, LSE, softmax_scale, S, W, n_obs, ratio, stream, false, state, L, layer);
}

lt_status lt_lazy_ratio(const lt_shape* shape, const void* Q, const void* K, const float* LSE, float softmax_scale,
                        int S, int W, int n_obs, float* ratio, lt_stream stream) {
  LT_RANGE();
  lt_status st = check_shape(shape);
  if (st != LT_OK) return st;
  // With no tokens only `ratio` is written (zeros); the inputs may be null.
  if (!aligned(ratio, 4)) return LT_ERR_INVALID_ARG;
  if (shape->total_tokens > 0 && (!aligned(Q, 16) || !aligned(K, 16) || !aligned(LSE, 4))) return LT_ERR_INVALID_ARG;
  if (S < 0 || W < 0 || (long long)S + W < 1 || n_obs < 1 || n_obs > 4096) return LT_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return LT_ERR_INVALID_ARG;
  const int group = shape->hq / shape->hkv;
  if (shape->hq > 65535 || shape->batch > 65535) return LT_ERR_INVALID_ARG;

  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != LT_OK) return st;
  lt::RatioParams p;
  p.batch = shape->batch;
  p.total_tokens = shape->total_tokens;
  p.hq = shape->hq;
  p.hkv = shape->hkv;
  p.group = group;
  p.S = S;
  p.W = W;
  p.n_obs = n_obs;
  p.cu_seqlens = shape->cu_seqlens;
  p.Q = static_cast<const __nv_bfloat16*>(Q);
  p.K = static_cast<const __nv_bfloat16*>(K);
  p.LSE = LSE;
  p.scale_log2 = resolve_scale(softmax_scale, shape->head_dim) * kLog2e;
  p.ratio = ratio;

  // Cluster size: about kRatioKeysPerCta keys of the longest sequence's band per
  // CTA, but no more CTAs per (sequence, head) than two waves of the grid need:
  // a packed batch already has batch x hq clusters, and splitting each further
  // only adds cluster barriers and DSMEM reads (8 sequences x 32 heads: 91.1 us
  // at 7 CTAs a cluster, 62.2 at 2, 56.4 at 1; one sequence of 32 heads keeps 7-8).
  const long long max_len = shape->cu_seqlens ? shape->max_seqlen : shape->total_tokens;
  const long long band = std::min<long long>(S, max_len) + std::min<long long>(max_len, (long long)n_obs + W - 1);
  const long long pairs = (long long)shape->batch * shape->hq;
  const long long by_grid = std::max<long long>(1, (2LL * dev->sm_count + pairs - 1) / pairs);
  const int cluster = int(std::min<long long>(
      std::min<long long>(dev->max_ratio_cluster, by_grid),
      std::max<long long>(1, (band + lt::kRatioKeysPerCta - 1) / lt::kRatioKeysPerCta)));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cluster, shape->hq, shape->batch);
  cfg.blockDim = dim3(32 * lt::kRatioWarps, 1, 1);
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (shape->head_dim == 64) {
    cfg.dynamicSmemBytes = lt::RatioLayout<64>::kBytes;
    e = cudaLaunchKernelEx(&cfg, lt::lazy_ratio_kernel<64>, p);
  } else {
    cfg.dynamicSmemBytes = lt::RatioLayout<128>::kBytes;
    e = cudaLaunchKernelEx(&cfg, lt::lazy_ratio_kernel<128>, p);
  }
  return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? LT_OK : LT_ERR_CUDA;
}

lt_status lt_compact_kv(const lt_shape* shape, const void* K, const void* V, const uint8_t* mask, int S, int W,
                        void* K_stream, void* V_stream, int32_t* stream_len, lt_stream stream) {
  LT_RANGE();
  lt_status st = check_shape(shape);
  if (st != LT_OK) return st;
  if (!mask || !aligned(K_stream, 16) || !aligned(V_stream, 16) || !aligned(stream_len, 4)) return LT_ERR_INVALID_ARG;
  if (shape->total_tokens > 0 && (!aligned(K, 16) || !aligned(V, 16))) return LT_ERR_INVALID_ARG;
  if (S < 0 || W < 0 || (long long)S + W < 1 || (long long)S + W > (1 << 24)) return LT_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != LT_OK) return st;
  lt::CompactParams p;
  p.batch = shape->batch;
  p.total_tokens = shape->total_tokens;
  p.hkv = shape->hkv;
  p.D = shape->head_dim;
  p.S = S;
  p.W = W;
  p.cu_seqlens = shape->cu_seqlens;
  p.K = static_cast<const uint4*>(K);
  p.V = static_cast<const uint4*>(V);
  p.mask = mask;
  p.Ks = static_cast<uint4*>(K_stream);
  p.Vs = static_cast<uint4*>(V_stream);
  p.len = stream_len;
  const long long work = (long long)shape->batch * (S + W) * shape->hkv * (shape->head_dim / 8);
  long long blocks = (work + 255) / 256;
  const long long cap = (long long)dev->sm_count * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  lt::compact_kv_kernel<<<int(blocks), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(p);
  return cudaGetLastError() == cudaSuccess ? LT_OK : LT_ERR_CUDA;
}

lt_status lt_compact_kv_layers(const lt_shape* shape, const void* const* K_layers, const void* const* V_layers, int L,
                               const int32_t* layers, int n, int S, int W, void* K_pool, void* V_pool,
                               int32_t* pool_len, lt_stream stream) {
  LT_RANGE();
  lt_status st = check_shape(shape);
  if (st != LT_OK) return st;
  if (L < 1 || n < 0 || n > L || !aligned(K_layers, 8) || !aligned(V_layers, 8) ||
      (n > 0 && (!aligned(layers, 4) || !aligned(K_pool, 16) || !aligned(V_pool, 16) || !aligned(pool_len, 4))))
    return LT_ERR_INVALID_ARG;
  if (S < 0 || W < 0 || (long long)S + W < 1 || (long long)S + W > (1 << 24)) return LT_ERR_INVALID_ARG;
  if (n == 0) return LT_OK;
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != LT_OK) return st;
  lt::CompactLayersParams p;
  p.batch = shape->batch;
  p.total_tokens = shape->total_tokens;
  p.hkv = shape->hkv;
  p.D = shape->head_dim;
  p.S = S;
  p.W = W;
  p.L = L;
  p.n = n;
  p.cu_seqlens = shape->cu_seqlens;
  p.K_layers = reinterpret_cast<const uint4* const*>(K_layers);
  p.V_layers = reinterpret_cast<const uint4* const*>(V_layers);
  p.layers = layers;
  p.K_pool = static_cast<uint4*>(K_pool);
  p.V_pool = static_cast<uint4*>(V_pool);
  p.pool_len = pool_len;
  const long long work = (long long)n * shape->batch * (S + W) * shape->hkv * (shape->head_dim / 8);
  long long blocks = (work + 255) / 256;
  const long long cap = (long long)dev->sm_count * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  lt::compact_layers_kernel<<<int(blocks), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(p);
  return cudaGetLastError() == cudaSuccess ? LT_OK : LT_ERR_CUDA;
}

size_t lt_dqueue_state_bytes(int L, int batch) {
  if (L < 1 || batch < 1) return 0;
  return lt::dqueue_bytes(L, batch);
}

static bool dq_args(const void* state, int L, int batch) {
  return aligned(state, 16) && L >= 1 && L <= 4096 && batch >= 1 && batch <= (1 << 20);
}

static int dq_blocks(int batch) { return (batch + 3) / 4; }   // 128 threads: a warp per sequence

lt_status lt_dqueue_init(void* state, int L, int budget, int batch, lt_stream stream) {
  LT_RANGE();
  if (!dq_args(state, L, batch) || budget < 0 || budget > L) return LT_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  lt_status st = device_info(&dev);
  if (st != LT_OK) return st;
  const cudaError_t e = launch_pdl(lt::dqueue_init_kernel, dim3(dq_blocks(batch)), dim3(128), 0,
                                   reinterpret_cast<cudaStream_t>(stream), state, L, budget, batch);
  return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? LT_OK : LT_ERR_CUDA;
}

lt_status lt_dqueue_push_gathered(void* state, int L, int batch, int layer, const float* ratio, int shards,
                                  int hq_shard, lt_stream stream) {
  LT_RANGE();
  if (!dq_args(state, L, batch) || !aligned(ratio, 4) || shards < 1 || hq_shard < 1) return LT_ERR_INVALID_ARG;
  const cudaError_t e = launch_pdl(lt::dqueue_push_kernel, dim3(dq_blocks(batch)), dim3(128), 0,
                                   reinterpret_cast<cudaStream_t>(stream), state, L, batch, layer, ratio, hq_shard,
                                   shards);
  return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? LT_OK : LT_ERR_CUDA;
}

lt_status lt_dqueue_push(void* state, int L, int batch, int layer, const float* ratio, int hq, lt_stream stream) {
  LT_RANGE();
  return lt_dqueue_push_gathered(state, L, batch, layer, ratio, 1, hq, stream);
}

lt_status lt_dqueue_result(const void* state, int L, int batch, int budget, uint8_t* lazy_mask, int32_t* order,
                           lt_stream stream) {
  LT_RANGE();
  if (!dq_args(state, L, batch) || !lazy_mask || budget < 0 || budget > L || (order && !aligned(order, 4)))
    return LT_ERR_INVALID_ARG;
  lt::dqueue_result_kernel<<<dq_blocks(batch), 128, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      state, L, batch, budget, lazy_mask, order);
  return cudaGetLastError() == cudaSuccess ? LT_OK : LT_ERR_CUDA;
}

lt_status lt_dqueue_error(const void* state, int* error_bits) {
  LT_RANGE();
  if (!aligned(state, 16) || !error_bits) return LT_ERR_INVALID_ARG;
  int32_t w = 0;
  if (cudaMemcpy(&w, static_cast<const int32_t*>(state) + 3, sizeof w, cudaMemcpyDeviceToHost) != cudaSuccess)
    return LT_ERR_CUDA;
  *error_bits = w;
  return LT_OK;
}

lt_status lt_compact_kv_pending(const lt_shape* shape, const void* const* K_layers, const void* const* V_layers,
                                const void* state, int L, int budget, int S, int W, void* K_pool, void* V_pool,
                                int32_t* pool_len, lt_stream stream) {
  LT_RANGE();
  lt_status st = check_shape(shape);
  if (st != LT_OK) return st;
  if (!aligned(K_layers, 8) || !aligned(V_layers, 8) || !dq_args(state, L, shape->batch) || budget < 1 ||
      budget > L || !aligned(K_pool, 16) || !aligned(V_pool, 16) || !aligned(pool_len, 4))
    return LT_ERR_INVALID_ARG;
  if (S < 0 || W < 0 || (long long)S + W < 1 || (long long)S + W > (1 << 24)) return LT_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != LT_OK) return st;
  lt::CompactPendingParams p;
  p.batch = shape->batch;
  p.total_tokens = shape->total_tokens;
  p.hkv = shape->hkv;
  p.D = shape->head_dim;
  p.S = S;
  p.W = W;
  p.L = L;
  p.budget = budget;
  p.cu_seqlens = shape->cu_seqlens;
  p.K_layers = reinterpret_cast<const uint4* const*>(K_layers);
  p.V_layers = reinterpret_cast<const uint4* const*>(V_layers);
  p.state = state;
  p.K_pool = static_cast<uint4*>(K_pool);
  p.V_pool = static_cast<uint4*>(V_pool);
  p.pool_len = pool_len;
  const long long work = (long long)shape->batch * (S + W) * shape->hkv * (shape->head_dim / 8);
  long long blocks = (work + 255) / 256;
  const long long cap = (long long)dev->sm_count * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  if (launch_pdl(lt::compact_pending_kernel, dim3(int(blocks)), dim3(256), 0, reinterpret_cast<cudaStream_t>(stream),
                 p) != cudaSuccess)
    return LT_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? LT_OK : LT_ERR_CUDA;
}

lt_status lt_kv_pool_commit(const lt_shape* shape, const void* K_cur, const void* V_cur, const void* state, int L,
                            int budget, int layer, int S, int W, void* K_full, void* V_full, void* K_stream,
                            void* V_stream, int32_t* stream_len, lt_stream stream) {
  LT_RANGE();
  lt_status st = check_shape(shape);
  if (st != LT_OK) return st;
  if (!dq_args(state, L, shape->batch) || budget < 0 || budget > L || layer < 0 || layer >= L) return LT_ERR_INVALID_ARG;
  if (S < 0 || W < 0 || (long long)S + W < 1 || (long long)S + W > (1 << 24)) return LT_ERR_INVALID_ARG;
  if (shape->total_tokens > 0 && (!aligned(K_cur, 16) || !aligned(V_cur, 16))) return LT_ERR_INVALID_ARG;
  if (budget < L && shape->total_tokens > 0 && (!aligned(K_full, 16) || !aligned(V_full, 16)))
    return LT_ERR_INVALID_ARG;
  if (budget > 0 && (!aligned(K_stream, 16) || !aligned(V_stream, 16) || !aligned(stream_len, 4)))
    return LT_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != LT_OK) return st;
  lt::PoolCommitParams p;
  p.batch = shape->batch;
  p.total_tokens = shape->total_tokens;
  p.hkv = shape->hkv;
  p.D = shape->head_dim;
  p.S = S;
  p.W = W;
  p.L = L;
  p.budget = budget;
  p.layer = layer;
  p.cu_seqlens = shape->cu_seqlens;
  p.K_cur = static_cast<const uint4*>(K_cur);
  p.V_cur = static_cast<const uint4*>(V_cur);
  p.K_full = static_cast<uint4*>(K_full);
  p.V_full = static_cast<uint4*>(V_full);
  p.state = state;
  p.K_stream = static_cast<uint4*>(K_stream);
  p.V_stream = static_cast<uint4*>(V_stream);
  p.stream_len = stream_len;
  // Enough CTAs to stream a whole layer's K/V at HBM bandwidth.
  const long long work = std::max<long long>((long long)shape->total_tokens, (long long)shape->batch * (S + W)) *
                         shape->hkv * (shape->head_dim / 8);
  long long blocks = (work + 255) / 256;
  const long long cap = (long long)dev->sm_count * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  if (launch_pdl(lt::kv_pool_commit_kernel, dim3(int(blocks)), dim3(256), 0, reinterpret_cast<cudaStream_t>(stream),
                 p) != cudaSuccess)
    return LT_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? LT_OK : LT_ERR_CUDA;
}

lt_status lt_dqueue_slots(const void* state, int L, int batch, int32_t* slots, lt_stream stream) {
  LT_RANGE();
  if (!dq_args(state, L, batch) || !aligned(slots, 4)) return LT_ERR_INVALID_ARG;
  const long long n = (long long)batch * L;
  const int blocks = int(std::min<long long>((n + 127) / 128, 4096));
  lt::dqueue_slots_kernel<<<blocks, 128, 0, reinterpret_cast<cudaStream_t>(stream)>>>(state, L, batch, slots);
  return cudaGetLastError() == cudaSuccess ? LT_OK : LT_ERR_CUDA;
}

lt_status lt_stream_ring_init(const int32_t* stream_len, int32_t* next_slot, int batch, int S, int W,
                              lt_stream stream) {
  LT_RANGE();
  if (!aligned(stream_len, 4) || !aligned(next_slot, 4) || batch < 1 || S < 0 || W < 1) return LT_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  lt_status st = device_info(&dev);
  if (st != LT_OK) return st;
  lt::stream_ring_init_kernel<<<(batch + 127) / 128, 128, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      stream_len, next_slot, batch, S, W);
  return cudaGetLastError() == cudaSuccess ? LT_OK : LT_ERR_CUDA;
}

lt_status lt_stream_append(void* K_stream, void* V_stream, int32_t* stream_len, int32_t* next_slot, const void* k_new,
                           const void* v_new, int batch, int hkv, int head_dim, int S, int W, lt_stream stream) {
  LT_RANGE();
  if (!aligned(K_stream, 16) || !aligned(V_stream, 16) || !aligned(stream_len, 4) || !aligned(next_slot, 4) ||
      !aligned(k_new, 16) || !aligned(v_new, 16) || batch < 1 || hkv < 1 || S < 0 || W < 1)
    return LT_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return LT_ERR_UNSUPPORTED;
  DeviceInfo* dev = nullptr;
  lt_status st = device_info(&dev);
  if (st != LT_OK) return st;
  lt::stream_append_kernel<<<batch, 128, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<uint4*>(K_stream), static_cast<uint4*>(V_stream), stream_len, next_slot,
      static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), hkv, head_dim, S, W);
  return cudaGetLastError() == cudaSuccess ? LT_OK : LT_ERR_CUDA;
}

namespace {

// CTAs per (sequence, KV head): a power of two up to the device's cluster
// limit, at least 128 rows each, and no more CTAs than two per SM in total.
int decode_splits(const DeviceInfo* dev, int batch, int hkv, int max_len) {
  int splits = 1;
  while (splits < dev->max_decode_splits && (long long)batch * hkv * splits * 2 <= 2LL * dev->sm_count &&
         max_len / (splits * 2) >= 128)
    splits *= 2;
  return splits;
}

lt_status launch_decode(lt::DecodeParams& p, int head_dim, int max_len, float softmax_scale, lt_stream stream) {
  DeviceInfo* dev = nullptr;
  lt_status st = device_info(&dev);
  if (st != LT_OK) return st;
  p.group = p.hq / p.hkv;
  p.max_len = max_len;
  p.splits = decode_splits(dev, p.batch, p.hkv, max_len);
  p.scale_log2 = resolve_scale(softmax_scale, head_dim) * kLog2e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.hkv * p.splits, p.batch, 1);
  cfg.blockDim = dim3(lt::kDecodeThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.splits;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlaps the previous kernel's tail
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = head_dim == 64 ? cudaLaunchKernelEx(&cfg, lt::decode_kernel<64>, p)
                                       : cudaLaunchKernelEx(&cfg, lt::decode_kernel<128>, p);
  return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? LT_OK : LT_ERR_CUDA;
}

}  // namespace

lt_status lt_stream_decode(const void* q, const void* K_stream, const void* V_stream, const int32_t* stream_len,
                           int batch, int hq, int hkv, int head_dim, int slots, void* O, float* LSE,
                           float softmax_scale, lt_stream stream) {
  LT_RANGE();
  if (!aligned(q, 16) || !aligned(K_stream, 16) || !aligned(V_stream, 16) || !aligned(stream_len, 4) ||
      !aligned(O, 16) || !aligned(LSE, 4) || batch < 1 || batch > 65535 || hq < 1 || hkv < 1 || hq % hkv ||
      slots < 1 || !std::isfinite(softmax_scale))
    return LT_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return LT_ERR_UNSUPPORTED;
  if ((long long)hkv * lt::kDecodeMaxSplits > 2147483647LL) return LT_ERR_INVALID_ARG;
  lt::DecodeParams p{};
  p.batch = batch;
  p.hq = hq;
  p.hkv = hkv;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.K = static_cast<const __nv_bfloat16*>(K_stream);
  p.V = static_cast<const __nv_bfloat16*>(V_stream);
  p.seq_start = nullptr;
  p.seq_stride = (long long)hkv * slots * head_dim;
  p.row_stride = head_dim;
  p.head_stride = (long long)slots * head_dim;
  p.len = stream_len;
  p.O = static_cast<__nv_bfloat16*>(O);
  p.LSE = LSE;
  return launch_decode(p, head_dim, slots, softmax_scale, stream);
}

lt_status lt_decode_attn(const void* q, const void* K, const void* V, const int32_t* seq_start, int seq_capacity,
                         const int32_t* len, int batch, int hq, int hkv, int head_dim, int max_len, void* O,
                         float* LSE, float softmax_scale, lt_stream stream) {
  LT_RANGE();
  if (!aligned(q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(len, 4) || !aligned(O, 16) ||
      !aligned(LSE, 4) || (seq_start && !aligned(seq_start, 4)) || batch < 1 || batch > 65535 || hq < 1 ||
      hkv < 1 || hq % hkv || max_len < 1 || (!seq_start && seq_capacity < max_len) ||
      !std::isfinite(softmax_scale))
    return LT_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return LT_ERR_UNSUPPORTED;
  if ((long long)hkv * lt::kDecodeMaxSplits > 2147483647LL) return LT_ERR_INVALID_ARG;
  lt::DecodeParams p{};
  p.batch = batch;
  p.hq = hq;
  p.hkv = hkv;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.K = static_cast<const __nv_bfloat16*>(K);
  p.V = static_cast<const __nv_bfloat16*>(V);
  p.seq_start = seq_start;
  p.row_stride = (long long)hkv * head_dim;
  p.seq_stride = seq_start ? 0 : (long long)seq_capacity * p.row_stride;
  p.head_stride = head_dim;
  p.len = len;
  p.O = static_cast<__nv_bfloat16*>(O);
  p.LSE = LSE;
  return launch_decode(p, head_dim, max_len, softmax_scale, stream);
}

size_t lt_decode_splitk_workspace_bytes(int batch, int hq, int head_dim, int max_len) {
  if (batch < 1 || hq < 1 || (head_dim != 64 && head_dim != 128) || max_len < 1) return 0;
  return lt::decode_splitk_floats(batch, hq, head_dim, max_len) * sizeof(float);
}

namespace {

// Checks and launches of the split-K decode over a full cache; `part` holds
// at least lt_decode_splitk_workspace_bytes of the call's sizes.
lt_status launch_decode_splitk(const void* q, const void* K, const void* V, const int32_t* seq_start,
                               int seq_capacity, const int32_t* len, int batch, int hq, int hkv, int head_dim,
                               int max_len, void* O, float* LSE, float softmax_scale, float* part,
                               lt_stream stream) {
  if (!aligned(q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(len, 4) || !aligned(O, 16) ||
      !aligned(LSE, 4) || !aligned(part, 16) || (seq_start && !aligned(seq_start, 4)) || batch < 1 ||
      batch > 65535 || hq < 1 || hkv < 1 || hq % hkv || max_len < 1 || (!seq_start && seq_capacity < max_len) ||
      !std::isfinite(softmax_scale))
    return LT_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return LT_ERR_UNSUPPORTED;
  const int splits = lt::decode_splitk_splits(max_len);
  if ((long long)hkv * splits > 2147483647LL) return LT_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  lt_status st = device_info(&dev);
  if (st != LT_OK) return st;
  lt::DecodeParams p{};
  p.batch = batch;
  p.hq = hq;
  p.hkv = hkv;
  p.group = hq / hkv;
  p.splits = splits;
  p.max_len = max_len;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.K = static_cast<const __nv_bfloat16*>(K);
  p.V = static_cast<const __nv_bfloat16*>(V);
  p.seq_start = seq_start;
  p.row_stride = (long long)hkv * head_dim;
  p.seq_stride = seq_start ? 0 : (long long)seq_capacity * p.row_stride;
  p.head_stride = head_dim;
  p.len = len;
  p.O = static_cast<__nv_bfloat16*>(O);
  p.LSE = LSE;
  p.scale_log2 = resolve_scale(softmax_scale, head_dim) * kLog2e;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const dim3 grid(hkv * splits, batch, 1), mgrid(hq, batch, 1);
  // Both launches programmatic: each may start while the kernel before it
  // finishes, and waits for it before touching memory.
  cudaError_t e;
  // Caches of more than kDecodeSplitKDense rows: two CTAs a SM.
  const bool dense = max_len > kDecodeSplitKDense;
  if (head_dim == 64) {
    e = dense ? launch_pdl(lt::decode_splitk_kernel<64, 2>, grid, dim3(lt::kDecodeThreads), 0, s, p, part)
              : launch_pdl(lt::decode_splitk_kernel<64, 1>, grid, dim3(lt::kDecodeThreads), 0, s, p, part);
    if (e == cudaSuccess) e = launch_pdl(lt::decode_merge_kernel<64>, mgrid, dim3(64), 0, s, part, hq, splits, p.O, LSE);
  } else {
    e = dense ? launch_pdl(lt::decode_splitk_kernel<128, 2>, grid, dim3(lt::kDecodeThreads), 0, s, p, part)
              : launch_pdl(lt::decode_splitk_kernel<128, 1>, grid, dim3(lt::kDecodeThreads), 0, s, p, part);
    if (e == cudaSuccess)
      e = launch_pdl(lt::decode_merge_kernel<128>, mgrid, dim3(128), 0, s, part, hq, splits, p.O, LSE);
  }
  return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? LT_OK : LT_ERR_CUDA;
}

}  // namespace

lt_status lt_decode_attn_splitk(const void* q, const void* K, const void* V, const int32_t* seq_start,
                                int seq_capacity, const int32_t* len, int batch, int hq, int hkv, int head_dim,
                                int max_len, void* O, float* LSE, float softmax_scale, void* workspace,
                                size_t workspace_bytes, lt_stream stream) {
  LT_RANGE();
  const size_t need = lt_decode_splitk_workspace_bytes(batch, hq, head_dim, max_len);
  if (need == 0 && (head_dim == 64 || head_dim == 128)) return LT_ERR_INVALID_ARG;
  if (need > 0 && (!workspace || workspace_bytes < need)) return LT_ERR_INVALID_ARG;
  return launch_decode_splitk(q, K, V, seq_start, seq_capacity, len, batch, hq, hkv, head_dim, max_len, O, LSE,
                              softmax_scale, static_cast<float*>(workspace), stream);
}

size_t lt_decode_splitk_noalloc_capacity_bytes(void) { return kNoAllocScratchBytes; }

lt_status lt_decode_attn_splitk_noalloc(const void* q, const void* K, const void* V, const int32_t* seq_start,
                                        int seq_capacity, const int32_t* len, int batch, int hq, int hkv,
                                        int head_dim, int max_len, void* O, float* LSE, float softmax_scale,
                                        lt_stream stream) {
  LT_RANGE();
  const size_t need = lt_decode_splitk_workspace_bytes(batch, hq, head_dim, max_len);
  if (need == 0 && (head_dim == 64 || head_dim == 128)) return LT_ERR_INVALID_ARG;
  if (need > kNoAllocScratchBytes) return LT_ERR_INVALID_ARG;   // beyond the fixed workspace
  DeviceInfo* dev = nullptr;
  lt_status st = device_info(&dev);   // the first call on a device takes the array's address
  if (st != LT_OK) return st;
  return launch_decode_splitk(q, K, V, seq_start, seq_capacity, len, batch, hq, hkv, head_dim, max_len, O, LSE,
                              softmax_scale, dev->noalloc_scratch, stream);
}

lt_status lt_selftest_wait_timeout(unsigned limit_us, lt_stream stream) {
  LT_RANGE();
  if (limit_us == 0 || limit_us > 10000000u) return LT_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  lt_status st = device_info(&dev);
  if (st != LT_OK) return st;
  lt::wait_timeout_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      dev->status, (unsigned long long)limit_us * 1000ull);
  return cudaGetLastError() == cudaSuccess ? LT_OK : LT_ERR_CUDA;
}

lt_status lt_device_status(int clear) {
  LT_RANGE();
  unsigned v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return LT_ERR_CUDA;
  if (cudaMemcpyFromSymbol(&v, g_status_word, sizeof v) != cudaSuccess) return LT_ERR_CUDA;
  if (clear) {
    const unsigned zero = 0;
    if (cudaMemcpyToSymbol(g_status_word, &zero, sizeof zero) != cudaSuccess) return LT_ERR_CUDA;
  }
  return (v & lt::kErrTimeout) ? LT_ERR_TIMEOUT : LT_OK;
}

}  // extern "C"
