// dqueue.cuh -- the layer priority queue kept in device memory, and the
// compaction it drives.
//
// LightTransfer project page (Methodology, LightTransfer-Test, Figure 2
// caption) and the LightTransfer write-up (second solution): after each layer
// of the prefill the layer enters a queue keyed by its lazy ratio; once more
// layers are queued than the full-KV capacity C = L - budget allows, the layer
// with the highest ratio is popped and its KV cache is reduced to the
// streaming version.  Keeping the queue on the device lets a whole prefill
// (attention, ratio, queue, compaction for every layer) run as one stream of
// kernels with no host round trip, so it can be captured in a CUDA graph.
//
// State (caller-allocated device memory, lt_dqueue_state_bytes):
//   header   int32[4]            L, budget, batch, error bits
//   size     int32[batch]        layers currently queued
//   ndem     int32[batch]        layers demoted so far
//   last     int32[batch]        layer demoted by the latest push, or -1
//   pushed   int32[batch][L]     1 once the layer has been pushed
//   qlayer   int32[batch][L]     queued layers (unordered)
//   qscore   float[batch][L]     their scores
//   order    int32[batch][L]     demoted layers in demotion order
#pragma once

#include "lt_device.cuh"

namespace lt {

constexpr int kDqErrBadPush = 1;    // layer out of range, pushed twice, or non-finite score
constexpr int kDqErrShape = 2;      // call's L / batch differ from the state's

struct DQueueView {
  int32_t* header;
  int32_t* size;
  int32_t* ndem;
  int32_t* last;
  int32_t* pushed;
  int32_t* qlayer;
  float* qscore;
  int32_t* order;
};

__host__ __device__ inline size_t dqueue_bytes(int L, int batch) {
  return sizeof(int32_t) * (4 + 3 * size_t(batch) + 4 * size_t(batch) * L);
}

__host__ __device__ inline DQueueView dqueue_view(void* state, int L, int batch) {
  DQueueView v;
  int32_t* w = static_cast<int32_t*>(state);
  v.header = w;
  v.size = w + 4;
  v.ndem = v.size + batch;
  v.last = v.ndem + batch;
  v.pushed = v.last + batch;
  v.qlayer = v.pushed + size_t(batch) * L;
  v.qscore = reinterpret_cast<float*>(v.qlayer + size_t(batch) * L);
  v.order = reinterpret_cast<int32_t*>(v.qscore + size_t(batch) * L);
  return v;
}

__global__ void dqueue_init_kernel(void* state, int L, int budget, int batch) {
  pdl_wait();
  pdl_launch_dependents();
  DQueueView v = dqueue_view(state, L, batch);
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
  if (tid == 0) {
    v.header[0] = L;
    v.header[1] = budget;
    v.header[2] = batch;
    v.header[3] = 0;
  }
  for (int b = tid; b < batch; b += gridDim.x * blockDim.x) {
    v.size[b] = 0;
    v.ndem[b] = 0;
    v.last[b] = -1;
    for (int l = 0; l < L; ++l) v.pushed[size_t(b) * L + l] = 0;
  }
}

// Higher score first; on a tie the lower layer index.
__device__ __forceinline__ bool dq_outranks(float sa, int a, float sb, int b) { return sa != sb ? sa > sb : a < b; }

// One thread per sequence: score = mean of the layer's head ratios (summed in
// double in head order, as the host lt_layer_score does), push, pop the
// best-ranked layer while more than C = L - budget are queued.  ratio is
// [shards, batch, hq_shard]: shard n holds heads [n hq_shard, (n+1) hq_shard)
// (the all-gather of head-sharded ratios; shards = 1 is the plain [batch, hq]),
// so the sum runs over the heads in the same order either way.
__global__ void dqueue_push_kernel(void* state, int L, int batch, int layer, const float* ratio, int hq_shard,
                                   int shards) {
  pdl_wait();
  pdl_launch_dependents();
  DQueueView v = dqueue_view(state, L, batch);
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= batch) return;
  if (v.header[0] != L || v.header[2] != batch) {
    atomicOr(&v.header[3], kDqErrShape);
    return;
  }
  v.last[b] = -1;
  double sum = 0.0;
  for (int n = 0; n < shards; ++n)
    for (int h = 0; h < hq_shard; ++h) sum += ratio[(size_t(n) * batch + b) * hq_shard + h];
  const float score = float(sum / (double(hq_shard) * shards));
  int32_t* pushed = v.pushed + size_t(b) * L;
  if (layer < 0 || layer >= L || pushed[layer] || !isfinite(score)) {
    atomicOr(&v.header[3], kDqErrBadPush);
    return;
  }
  pushed[layer] = 1;
  int32_t* ql = v.qlayer + size_t(b) * L;
  float* qs = v.qscore + size_t(b) * L;
  int n = v.size[b];
  ql[n] = layer;
  qs[n] = score;
  ++n;
  const int cap = L - v.header[1];
  if (n > cap) {
    int best = 0;
    for (int k = 1; k < n; ++k)
      if (dq_outranks(qs[k], ql[k], qs[best], ql[best])) best = k;
    const int dem = ql[best];
    ql[best] = ql[n - 1];
    qs[best] = qs[n - 1];
    --n;
    v.order[size_t(b) * L + v.ndem[b]] = dem;
    v.ndem[b] += 1;
    v.last[b] = dem;
  }
  v.size[b] = n;
}

// lazy_mask[b, l] = 1 for the layers demoted so far; order[b, k] for k < budget
// (entries past the number demoted are -1).
__global__ void dqueue_result_kernel(const void* state, int L, int batch, int budget, uint8_t* lazy_mask,
                                     int32_t* order) {
  DQueueView v = dqueue_view(const_cast<void*>(state), L, batch);
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= batch) return;
  const int nd = v.ndem[b];
  for (int l = 0; l < L; ++l) lazy_mask[size_t(b) * L + l] = 0;
  for (int k = 0; k < nd; ++k) lazy_mask[size_t(b) * L + v.order[size_t(b) * L + k]] = 1;
  if (order)
    for (int k = 0; k < budget; ++k) order[size_t(b) * budget + k] = k < nd ? v.order[size_t(b) * L + k] : -1;
}

struct CompactPendingParams {
  int batch, total_tokens, hkv, D, S, W, L, budget;
  const int32_t* cu_seqlens;
  const uint4* const* K_layers;   // device array [L] of the layers' K base pointers
  const uint4* const* V_layers;
  const void* state;
  uint4* K_pool;                  // [budget, batch, hkv, S+W, d]
  uint4* V_pool;
  int32_t* pool_len;              // [budget, batch]
};

// For every sequence whose latest push demoted a layer: gather that layer's
// sink and recent rows (p = [0, min(S,N)) ++ [max(S, N-W), N)) into pool slot
// k = its demotion index; rows past the kept count are zero.  Same data
// movement as compact_kv_kernel, with the layer chosen on the device.
__global__ void __launch_bounds__(256) compact_pending_kernel(const CompactPendingParams p) {
  pdl_wait();
  pdl_launch_dependents();
  DQueueView v = dqueue_view(const_cast<void*>(p.state), p.L, p.batch);
  const int pieces = p.D / 8;
  const int slots = p.S + p.W;
  const long long per_seq = (long long)slots * p.hkv * pieces;
  const long long total = per_seq * p.batch;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long x = (long long)blockIdx.x * blockDim.x + threadIdx.x; x < total; x += stride) {
    const int b = int(x / per_seq);
    const int layer = v.last[b];
    if (layer < 0) continue;
    const int k = v.ndem[b] - 1;
    if (k < 0 || k >= p.budget) continue;
    long long rem = x - (long long)b * per_seq;
    const int r = int(rem / ((long long)p.hkv * pieces));
    rem -= (long long)r * p.hkv * pieces;
    const int kh = int(rem / pieces);
    const int piece = int(rem - (long long)kh * pieces);
    int start = 0, N = p.total_tokens;
    if (p.cu_seqlens) {
      start = p.cu_seqlens[b];
      N = p.cu_seqlens[b + 1] - start;
    }
    const int n_sink = min(p.S, N);
    const int keep = min(N, slots);
    const size_t dst = (((size_t(k) * p.batch + b) * p.hkv + kh) * slots + r) * pieces + piece;
    if (r < keep) {
      const int pos = r < n_sink ? r : max(p.S, N - p.W) + (r - n_sink);
      const size_t src = ((size_t(start) + pos) * p.hkv + kh) * pieces + piece;
      p.K_pool[dst] = p.K_layers[layer][src];
      p.V_pool[dst] = p.V_layers[layer][src];
    } else {
      p.K_pool[dst] = make_uint4(0u, 0u, 0u, 0u);
      p.V_pool[dst] = make_uint4(0u, 0u, 0u, 0u);
    }
    if (r == 0 && kh == 0 && piece == 0) p.pool_len[size_t(k) * p.batch + b] = keep;
  }
}

// Zeroes n floats (the fused ratio's accumulator) as a kernel, so that it can
// be launched programmatically ahead of the attention.
__global__ void zero_f32_kernel(float* x, int n) {
  pdl_wait();
  pdl_launch_dependents();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) x[i] = 0.f;
}

}  // namespace lt
