// dqueue.cuh -- the layer priority queue kept in device memory, and the
// compaction it drives.
//
// LightTransfer project page (Methodology, LightTransfer-Test, Figure 2
// caption) and the LightTransfer write-up (second solution): after each layer
// of the prefill the layer enters a queue keyed by its lazy ratio; once more
// layers are queued than the full-KV capacity C = L - budget allows, the layer
// with the highest ratio is popped and its KV cache is reduced to the
// streaming version, "freeing memory for storing the KV cache of the current
// layer".  Keeping the queue on the device lets a whole prefill (attention,
// ratio, queue, compaction for every layer) run as one stream of kernels with
// no host round trip, so it can be captured in a CUDA graph.
//
// The queue also assigns full-KV slots: a pool of C slots holds the full K/V
// of the queued layers (every queued layer owns one slot).  A pushed layer
// takes a never-used slot while the queue is filling; once it is full, a push
// either demotes the pushed layer itself (it never takes a slot) or demotes an
// older layer, whose slot the pushed layer takes over.  With the current
// layer's own K/V buffer that is at most C + 1 full layers at any time.
//
// State (caller-allocated device memory, lt_dqueue_state_bytes), int32 words:
//   header   int32[8]            L, budget, batch, error bits, CTA-done
//                                counter (the attention kernel's last-CTA
//                                push), 3 reserved
//   size     int32[batch]        layers currently queued
//   ndem     int32[batch]        layers demoted so far
//   last     int32[batch]        layer demoted by the latest push, or -1
//   pushed   int32[batch][L]     1 once the layer has been pushed
//   qlayer   int32[batch][L]     queued layers (unordered)
//   qscore   float[batch][L]     their scores
//   order    int32[batch][L]     demoted layers in demotion order
//   slot     int32[batch][L]     full-KV slot of each layer, -1 if none
#pragma once

#include <climits>

#include "lt_device.cuh"

namespace lt {

constexpr int kDqErrBadPush = 1;    // layer out of range, pushed twice, or non-finite score
constexpr int kDqErrShape = 2;      // call's L / batch differ from the state's
constexpr int kDqErrAborted = 4;    // a fused push was skipped: its attention launch gave up a wait

constexpr int kDqHeader = 8;        // header words
constexpr int kDqCounter = 4;       // header word: CTAs of the current attention launch done
constexpr int kDqAbortUnit = 1 << 16;   // added to the counter by a CTA that gave up a wait

struct DQueueView {
  int32_t* header;
  int32_t* size;
  int32_t* ndem;
  int32_t* last;
  int32_t* pushed;
  int32_t* qlayer;
  float* qscore;
  int32_t* order;
  int32_t* slot;
};

__host__ __device__ inline size_t dqueue_bytes(int L, int batch) {
  return sizeof(int32_t) * (kDqHeader + 3 * size_t(batch) + 5 * size_t(batch) * L);
}

__host__ __device__ inline DQueueView dqueue_view(void* state, int L, int batch) {
  DQueueView v;
  int32_t* w = static_cast<int32_t*>(state);
  v.header = w;
  v.size = w + kDqHeader;
  v.ndem = v.size + batch;
  v.last = v.ndem + batch;
  v.pushed = v.last + batch;
  v.qlayer = v.pushed + size_t(batch) * L;
  v.qscore = reinterpret_cast<float*>(v.qlayer + size_t(batch) * L);
  v.order = reinterpret_cast<int32_t*>(v.qscore + size_t(batch) * L);
  v.slot = v.order + size_t(batch) * L;
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
    for (int i = 3; i < kDqHeader; ++i) v.header[i] = 0;
  }
  for (int b = tid; b < batch; b += gridDim.x * blockDim.x) {
    v.size[b] = 0;
    v.ndem[b] = 0;
    v.last[b] = -1;
    for (int l = 0; l < L; ++l) {
      v.pushed[size_t(b) * L + l] = 0;
      v.slot[size_t(b) * L + l] = -1;
    }
  }
}

// Higher score first; on a tie the lower layer index.
__device__ __forceinline__ bool dq_outranks(float sa, int a, float sb, int b) { return sa != sb ? sa > sb : a < b; }

// Score of sequence b, computed by one whole warp: the mean of its head
// ratios, summed in double in head order as the host lt_layer_score does.
// ratio is [shards, batch, hq_shard]: shard n holds heads [n hq_shard,
// (n+1) hq_shard) (the all-gather of head-sharded ratios; shards = 1 is the
// plain [batch, hq]), so the sum runs over the heads in the same order either
// way.  The lanes load 32 heads at a time in parallel (one memory round trip
// per 32 heads instead of one per head); lane 0 adds them in order.  Loads
// bypass L1 (ld.global.cg): the ratios may have been added by other CTAs of
// the same kernel just before (the attention kernel's last-CTA push).
// Returns the score in every lane.
__device__ __forceinline__ float dq_score_warp(const float* ratio, int batch, int b, int hq_shard, int shards) {
  const int lane = threadIdx.x & 31;
  const int hq = hq_shard * shards;
  double sum = 0.0;
  for (int h0 = 0; h0 < hq; h0 += 32) {
    const int h = h0 + lane;
    float x = 0.f;
    if (h < hq) {
      const int n = h / hq_shard;
      x = __ldcg(ratio + (size_t(n) * batch + b) * hq_shard + (h - n * hq_shard));
    }
    const int cnt = min(32, hq - h0);
    for (int k = 0; k < cnt; ++k) {
      const float y = __shfl_sync(0xffffffffu, x, k);
      if (lane == 0) sum += double(y);
    }
  }
  const float score = float(sum / double(hq));
  return __shfl_sync(0xffffffffu, score, 0);
}

// Push (layer, score) into sequence b's queue, by one whole warp (the same
// score in every lane); while more than C = L - budget layers are queued, pop
// the best-ranked one (it becomes a streaming layer).  The queued entries are
// read in parallel and the best one found by a shuffle reduction: the
// ranking (score, then lower layer) is a strict order over distinct layers,
// so the result does not depend on the reduction order.  Full-KV slots follow
// the queue: the pushed layer takes the popped layer's slot, or a never-used
// one (slot n-1) while no layer has been popped yet, or none when it is
// popped itself.  An invalid push (layer out of range or pushed twice,
// non-finite score) sets an error bit and changes nothing.
__device__ __forceinline__ void dq_push_warp(const DQueueView& v, int L, int b, int layer, float score) {
  const int lane = threadIdx.x & 31;
  int32_t* pushed = v.pushed + size_t(b) * L;
  int32_t* ql = v.qlayer + size_t(b) * L;
  float* qs = v.qscore + size_t(b) * L;
  int32_t* slot = v.slot + size_t(b) * L;
  const bool bad = layer < 0 || layer >= L || !isfinite(score) || __ldcg(pushed + layer) != 0;
  const int n0 = __ldcg(v.size + b);
  const int cap = L - v.header[1];
  __syncwarp();
  if (bad) {
    if (lane == 0) {
      v.last[b] = -1;
      atomicOr(&v.header[3], kDqErrBadPush);
    }
    return;
  }
  const int n = n0 + 1;
  if (n <= cap) {
    if (lane == 0) {
      pushed[layer] = 1;
      ql[n0] = layer;
      qs[n0] = score;
      slot[layer] = n0;          // no layer popped so far: slots 0..n0-1 are held
      v.size[b] = n;
      v.last[b] = -1;
    }
    return;
  }
  // Best-ranked of the n0 queued entries and the pushed one (index n0).
  float bs = -INFINITY;
  int bl = INT_MAX, bk = -1;
  for (int k = lane; k < n; k += 32) {
    const float sk = k < n0 ? __ldcg(qs + k) : score;
    const int lk = k < n0 ? __ldcg(ql + k) : layer;
    if (bk < 0 || dq_outranks(sk, lk, bs, bl)) {
      bs = sk;
      bl = lk;
      bk = k;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float os = __shfl_xor_sync(0xffffffffu, bs, off);
    const int ol = __shfl_xor_sync(0xffffffffu, bl, off);
    const int ok = __shfl_xor_sync(0xffffffffu, bk, off);
    if (ok >= 0 && (bk < 0 || dq_outranks(os, ol, bs, bl))) {
      bs = os;
      bl = ol;
      bk = ok;
    }
  }
  if (lane == 0) {
    const int dem = bl;
    pushed[layer] = 1;
    if (bk != n0) {
      // An older layer is popped: the pushed one takes its queue entry and its slot.
      ql[bk] = layer;
      qs[bk] = score;
      slot[layer] = slot[dem];
      slot[dem] = -1;
    }
    const int nd = v.ndem[b];
    v.order[size_t(b) * L + nd] = dem;
    v.ndem[b] = nd + 1;
    v.last[b] = dem;
    v.size[b] = n0;
  }
}

// One warp per sequence: score, then push.
__global__ void dqueue_push_kernel(void* state, int L, int batch, int layer, const float* ratio, int hq_shard,
                                   int shards) {
  pdl_wait();
  pdl_launch_dependents();
  DQueueView v = dqueue_view(state, L, batch);
  const int b = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (b >= batch) return;
  if (v.header[0] != L || v.header[2] != batch) {
    if ((threadIdx.x & 31) == 0) atomicOr(&v.header[3], kDqErrShape);
    return;
  }
  dq_push_warp(v, L, b, layer, dq_score_warp(ratio, batch, b, hq_shard, shards));
}

// The push done by the last CTA of a kernel to finish (the attention kernel
// fused with the ratio): every CTA calls this once, after all of its own
// ratio additions, with all of its threads (a multiple of 32).  The CTA that
// completes the count pushes every sequence's score (a warp per sequence) and
// resets the counter for the next launch.  A CTA that gave up a bounded wait
// marks the launch; the push is then skipped and the queue's error bit set
// (the ratios are incomplete).
__device__ __forceinline__ void dq_last_cta_push(void* state, int L, int batch, int layer, const float* ratio,
                                                 int hq, bool aborted, int* smem_flag) {
  DQueueView v = dqueue_view(state, L, batch);
  // The caller has passed a CTA barrier after its last ratio addition: thread
  // 0's device-scope fence below orders every thread's additions (ordered
  // before it by that barrier) before the count.
  if (threadIdx.x == 0) {
    __threadfence();
    const int prev = atomicAdd(&v.header[kDqCounter], 1 + (aborted ? kDqAbortUnit : 0));
    const int done = (prev & (kDqAbortUnit - 1)) + 1;
    *smem_flag = done == int(gridDim.x) ? (1 + ((prev >> 16) != 0 || aborted ? 1 : 0)) : 0;
  }
  __syncthreads();
  const int flag = *smem_flag;
  if (flag == 0) return;
  __threadfence();     // every CTA's additions (counted before ours) are visible
  const int warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  if (v.header[0] != L || v.header[2] != batch) {
    if (threadIdx.x == 0) atomicOr(&v.header[3], kDqErrShape);
  } else if (flag == 2) {
    if (threadIdx.x == 0) atomicOr(&v.header[3], kDqErrAborted);
    for (int b = threadIdx.x; b < batch; b += blockDim.x) v.last[b] = -1;   // nothing to compact
  } else {
    for (int b = warp; b < batch; b += nwarps) dq_push_warp(v, L, b, layer, dq_score_warp(ratio, batch, b, hq, 1));
  }
  __syncthreads();
  if (threadIdx.x == 0) v.header[kDqCounter] = 0;
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

struct PoolCommitParams {
  int batch, total_tokens, hkv, D, S, W, L, budget, layer;
  const int32_t* cu_seqlens;
  const uint4* K_cur;      // [T, hkv, d] the current layer's K/V (its own buffer)
  const uint4* V_cur;
  uint4* K_full;           // [L - budget, T, hkv, d] full-KV slots
  uint4* V_full;
  const void* state;
  uint4* K_stream;         // [budget, batch, hkv, S+W, d]
  uint4* V_stream;
  int32_t* stream_len;     // [budget, batch]
};

// After the push of layer `layer`, for every sequence b (whose rows are the
// same token range in every slot):
//   * the layer the push demoted, if any, is reduced to its streaming rows
//     p = [0, min(S,N)) ++ [max(S, N-W), N) in streaming slot k = its demotion
//     index (rows past the kept count zero) -- read from the current layer's
//     buffer when the current layer itself was demoted, else from the
//     demoted layer's full-KV slot;
//   * the current layer, if it stays full, is stored in its full-KV slot: the
//     slot the demotion just freed, or a never-used one.
// When the demoted layer's slot is reused, the thread that copies a kept row
// out of the slot is the thread that then overwrites that row, so the read
// comes first without any barrier.  Sequences whose push demoted nothing and
// that keep no slot (the current layer was demoted) only do the gather.
__global__ void __launch_bounds__(256) kv_pool_commit_kernel(const PoolCommitParams p) {
  pdl_wait();
  pdl_launch_dependents();
  DQueueView v = dqueue_view(const_cast<void*>(p.state), p.L, p.batch);
  const int pieces = p.D / 8;
  const int slots = p.S + p.W;
  const long long row_pieces = (long long)p.hkv * pieces;
  const size_t slot_elems = size_t(p.total_tokens) * size_t(row_pieces);
  const long long stride = (long long)gridDim.x * blockDim.x;
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int cap = p.L - p.budget;
  for (int b = 0; b < p.batch; ++b) {
    int start = 0, N = p.total_tokens;
    if (p.cu_seqlens) {
      start = p.cu_seqlens[b];
      N = p.cu_seqlens[b + 1] - start;
    }
    const int dem = v.last[b];
    const int k = v.ndem[b] - 1;
    const bool gather = dem >= 0 && dem < p.L && k >= 0 && k < p.budget;
    const int s = v.slot[size_t(b) * p.L + p.layer];
    const bool store = s >= 0 && s < cap;
    // The demoted layer's rows: the current buffer, or the slot the current
    // layer takes over (a demoted older layer always held a slot).
    const bool from_cur = dem == p.layer;
    if (gather && !from_cur && !store) continue;   // inconsistent state: touch nothing
    const int n_sink = min(p.S, N);
    const int win0 = max(p.S, N - p.W);
    const int keep = min(N, slots);
    // Rows visited: all N when storing, else only the kept rows.
    const int rows = store ? N : (gather ? keep : 0);
    const long long work = (long long)rows * row_pieces;
    for (long long x = tid; x < work; x += stride) {
      const int i = int(x / row_pieces);
      const int rem = int(x - (long long)i * row_pieces);
      // Position inside the sequence and its index among the kept rows (-1: dropped).
      int r, idx;
      if (store) {
        r = i;
        idx = !gather ? -1 : (r < n_sink ? r : (r >= win0 ? n_sink + (r - win0) : -1));
      } else {
        idx = i;
        r = i < n_sink ? i : win0 + (i - n_sink);
      }
      const size_t src = (size_t(start) + r) * size_t(row_pieces) + rem;
      uint4 kc = make_uint4(0u, 0u, 0u, 0u), vc = kc;
      if (store || from_cur) {
        kc = p.K_cur[src];
        vc = p.V_cur[src];
      }
      if (idx >= 0) {
        const int kh = rem / pieces;
        const int piece = rem - kh * pieces;
        const size_t dst = (((size_t(k) * p.batch + b) * p.hkv + kh) * slots + idx) * pieces + piece;
        if (from_cur) {
          p.K_stream[dst] = kc;
          p.V_stream[dst] = vc;
        } else {
          p.K_stream[dst] = p.K_full[size_t(s) * slot_elems + src];
          p.V_stream[dst] = p.V_full[size_t(s) * slot_elems + src];
        }
      }
      if (store) {
        p.K_full[size_t(s) * slot_elems + src] = kc;
        p.V_full[size_t(s) * slot_elems + src] = vc;
      }
    }
    if (gather) {
      // Rows of the streaming slot past the kept count are zero; its length.
      if (tid == 0) p.stream_len[size_t(k) * p.batch + b] = keep;
      const long long zwork = (long long)(slots - keep) * row_pieces;
      for (long long x = tid; x < zwork; x += stride) {
        const int idx = keep + int(x / row_pieces);
        const int rem = int(x % row_pieces);
        const int kh = rem / pieces;
        const int piece = rem - kh * pieces;
        const size_t dst = (((size_t(k) * p.batch + b) * p.hkv + kh) * slots + idx) * pieces + piece;
        p.K_stream[dst] = make_uint4(0u, 0u, 0u, 0u);
        p.V_stream[dst] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  }
}

// full-KV slot of every layer of every sequence (device int32 [batch, L]; -1:
// the layer holds no slot -- demoted, or not pushed yet).
__global__ void dqueue_slots_kernel(const void* state, int L, int batch, int32_t* out) {
  DQueueView v = dqueue_view(const_cast<void*>(state), L, batch);
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < (long long)batch * L;
       i += (long long)gridDim.x * blockDim.x)
    out[i] = v.slot[i];
}

// Zeroes n floats (the fused ratio's accumulator) as a kernel, so that it can
// be launched programmatically ahead of the attention.
__global__ void zero_f32_kernel(float* x, int n) {
  pdl_wait();
  pdl_launch_dependents();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) x[i] = 0.f;
}

}  // namespace lt
