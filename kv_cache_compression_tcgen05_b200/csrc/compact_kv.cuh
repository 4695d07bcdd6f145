// compact_kv.cuh -- KV-cache compaction of a demoted layer to its streaming form.
//
// LightTransfer write-up (second solution of LightTransfer-Test): the layer
// popped from the priority queue has its KV cache switched to the streaming
// version; LightTransfer project page (Figure 2 caption): its KV cache is
// reduced, freeing memory for the current layer.  The streaming version keeps
// the S initial (sink) rows and the W most recent rows:
//     p = [0, min(S, N)) ++ [max(S, N - W), N)
//     K_stream[b, kh, r] = K[cu[b] + p_r, kh]   (r < len = min(N, S + W)), zero after.
//
// A bit copy bound by HBM bandwidth.  One thread moves one 16-byte piece of a
// K row and the same piece of the V row; consecutive threads take consecutive
// pieces of [row][kv head][d] so both the reads (the [T, hkv, d] source) and the
// writes (128/256-byte rows of the [b, hkv, S+W, d] destination) are full
// coalesced segments.  Grid-stride loop over a grid sized to the SM count.
#pragma once

#include "lt_device.cuh"

namespace lt {

struct CompactParams {
  int batch;
  int total_tokens;
  int hkv;
  int D;
  int S;
  int W;
  const int32_t* cu_seqlens;
  const uint4* K;
  const uint4* V;
  const uint8_t* mask;
  uint4* Ks;
  uint4* Vs;
  int32_t* len;
};

__global__ void __launch_bounds__(256) compact_kv_kernel(const CompactParams p) {
  const int pieces = p.D / 8;                       // 16-byte pieces per row
  const int slots = p.S + p.W;
  const long long per_seq = (long long)slots * p.hkv * pieces;
  const long long total = per_seq * p.batch;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long x = (long long)blockIdx.x * blockDim.x + threadIdx.x; x < total; x += stride) {
    const int b = int(x / per_seq);
    if (!p.mask[b]) continue;
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
    const size_t dst = ((size_t(b) * p.hkv + kh) * slots + r) * pieces + piece;
    if (r < keep) {
      const int pos = r < n_sink ? r : max(p.S, N - p.W) + (r - n_sink);
      const size_t src = ((size_t(start) + pos) * p.hkv + kh) * pieces + piece;
      p.Ks[dst] = p.K[src];
      p.Vs[dst] = p.V[src];
    } else {
      p.Ks[dst] = make_uint4(0u, 0u, 0u, 0u);
      p.Vs[dst] = make_uint4(0u, 0u, 0u, 0u);
    }
    if (r == 0 && kh == 0 && piece == 0) p.len[b] = keep;
  }
  // Sequences that are not demoted get length 0.
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < p.batch; b += int(stride))
    if (!p.mask[b]) p.len[b] = 0;
}

// Compaction of several layers in one launch: pool slot k receives the
// streaming rows of layer layers[k] for every sequence (same gather as
// compact_kv_kernel with all sequences selected); a layer index outside
// [0, L) leaves its slot untouched.  Enough independent 16-byte pieces for the
// whole launch keep HBM busy where one layer alone is bound by latency.
struct CompactLayersParams {
  int batch, total_tokens, hkv, D, S, W, L, n;
  const int32_t* cu_seqlens;
  const uint4* const* K_layers;   // device array [L] of the layers' K base pointers
  const uint4* const* V_layers;
  const int32_t* layers;          // [n]
  uint4* K_pool;                  // [n, batch, hkv, S+W, d]
  uint4* V_pool;
  int32_t* pool_len;              // [n, batch]
};

__global__ void __launch_bounds__(256) compact_layers_kernel(const CompactLayersParams p) {
  const int pieces = p.D / 8;
  const int slots = p.S + p.W;
  const long long per_seq = (long long)slots * p.hkv * pieces;
  const long long per_slot = per_seq * p.batch;
  const long long total = per_slot * p.n;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long x = (long long)blockIdx.x * blockDim.x + threadIdx.x; x < total; x += stride) {
    const int k = int(x / per_slot);
    const int layer = p.layers[k];
    if (layer < 0 || layer >= p.L) continue;
    long long rem = x - (long long)k * per_slot;
    const int b = int(rem / per_seq);
    rem -= (long long)b * per_seq;
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

}  // namespace lt
