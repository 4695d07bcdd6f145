// decode.cuh -- one decode step of attention over a layer's KV cache: the
// streaming cache of a demoted layer, or the full cache of a kept one.
//
// Press-release page ("LLM突破：推理加速，长CoT生成惊艳"): the converted layers
// use streaming attention, which needs only a constant-size KV cache, while the
// other layers keep full attention; the LightTransfer project page: the lazy
// layers pay attention mostly to the initial and the recent tokens.  After
// compaction a lazy layer keeps, per sequence and KV head, S + W rows: the S
// sink positions and the W most recent ones.  At decode the new token's
// key/value enter the window (replacing its oldest row once the cache is full)
// and the token attends to the cached rows:
//     K_p = [0, min(S, p+1)) U [max(S, p-W+1), p]   (p = the token's position)
// -- the same key set the lazy ratio measures.  A kept layer's token attends
// to all of its sequence's rows.
//
// Streaming cache layout: [batch, hkv, S+W, d] bf16 (as lt_compact_kv writes
// it), len[b] valid rows; rows [0, S) are the sinks, rows [S, S+W) the window,
// used as a ring once full: next[b] is the slot the next token goes to.
// Full cache layout: token-major [rows, hkv, d] bf16, the rows of one sequence
// contiguous (the prefill's packed K/V, or a padded [batch, capacity, hkv, d]).
//
// The decode is HBM bound: each cached row is read once per KV head for all g
// query heads of its group, 4 per pass.  The rows of one (sequence, KV head)
// are split over a cluster of `splits` CTAs; in a CTA each group of d/8 lanes
// of a warp takes one row at a time, 8 elements per lane in one 16-byte load
// (the next row's loads in flight while the current one is used), scores are
// reduced over the group's lanes with shuffles, and each group keeps a running
// (max, sum, output) per head in the log2 domain.  Groups merge through
// shuffles; warps through shared memory and the cluster's CTAs through
// distributed shared memory, each with one thread per (head, element), rank 0
// writing O and LSE.
#pragma once

#include <cooperative_groups.h>

#include "lt_device.cuh"

namespace lt {

namespace dcg = cooperative_groups;

__global__ void stream_ring_init_kernel(const int32_t* len, int32_t* next, int batch, int S, int W) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < batch) next[b] = len[b] < S + W ? len[b] : S;
}

// One CTA per sequence: the new rows of every KV head go to slot next[b]; then
// one thread advances len and next.  len > S+W is read as a full cache.
__global__ void stream_append_kernel(uint4* Ks, uint4* Vs, int32_t* len, int32_t* next, const uint4* k_new,
                                     const uint4* v_new, int hkv, int D, int S, int W) {
  const int b = blockIdx.x;
  const int slots = S + W;
  const int slot = next[b];
  const int n = len[b];
  // A state no ring operation can produce (slot outside the cache, or a free
  // slot other than the one after the last row) is left untouched.
  if (slot < 0 || slot >= slots || n < 0 || (n < slots && slot != n)) return;
  const int pieces = D / 8;
  for (int x = threadIdx.x; x < hkv * pieces; x += blockDim.x) {
    const int kh = x / pieces, piece = x - kh * pieces;
    const size_t dst = ((size_t(b) * hkv + kh) * slots + slot) * pieces + piece;
    const size_t src = (size_t(b) * hkv + kh) * pieces + piece;
    Ks[dst] = k_new[src];
    Vs[dst] = v_new[src];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (n < slots) {
      len[b] = n + 1;
      next[b] = n + 1 < slots ? n + 1 : S;
    } else {
      next[b] = S + (slot - S + 1) % W;
    }
  }
}

// Element offsets: row r of KV head kh of sequence b starts at
//   (seq_start ? seq_start[b] * row_stride : b * seq_stride) + r * row_stride + kh * head_stride.
struct DecodeParams {
  int batch, hq, hkv, group, splits, max_len;
  const __nv_bfloat16* q;    // [batch, hq, d]
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  const int32_t* seq_start;  // [batch] first row of each sequence, or null
  long long seq_stride, row_stride, head_stride;
  const int32_t* len;        // [batch] valid rows (clamped to [0, max_len])
  __nv_bfloat16* O;          // [batch, hq, d]
  float* LSE;                // [batch, hq]
  float scale_log2;
};

constexpr int kDecodeThreads = 256;
constexpr int kDecodeWarps = kDecodeThreads / 32;
constexpr int kDecodeHeads = 4;   // query heads per pass over the cache
constexpr int kDecodeMaxSplits = 16;

// Merges running softmax state (m2, l2, o2) into (m1, l1, o1); log2 domain.
template <int E>
__device__ __forceinline__ void softmax_merge(float& m1, float& l1, float (&o1)[E], float m2, float l2,
                                              const float (&o2)[E]) {
  const float M = fmaxf(m1, m2);
  const float c1 = M == -INFINITY ? 0.f : fast_exp2(m1 - M);
  const float c2 = M == -INFINITY ? 0.f : fast_exp2(m2 - M);
  l1 = l1 * c1 + l2 * c2;
#pragma unroll
  for (int e = 0; e < E; ++e) o1[e] = o1[e] * c1 + o2[e] * c2;
  m1 = M;
}

template <int D>
__global__ void __launch_bounds__(kDecodeThreads) decode_kernel(const DecodeParams p) {
  // Programmatic dependent launch: this kernel may start while the previous
  // one in the stream finishes; it waits for it before touching memory.
  pdl_wait();
  pdl_launch_dependents();
  constexpr int E = 8;           // elements of a row per lane (one 16-byte load)
  constexpr int LPR = D / E;     // lanes per row
  constexpr int GPW = 32 / LPR;  // row groups per warp
  dcg::cluster_group cluster = dcg::this_cluster();
  const int split = int(cluster.block_rank());
  const int kh = blockIdx.x / p.splits;
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rgw = lane / LPR;  // row group in the warp
  const int li = lane % LPR;   // lane in the row group
  __shared__ float sm_m[kDecodeWarps][kDecodeHeads], sm_l[kDecodeWarps][kDecodeHeads];
  __shared__ __align__(16) float sm_o[kDecodeWarps][kDecodeHeads][D];
  __shared__ float cta_m[kDecodeHeads], cta_l[kDecodeHeads];
  __shared__ __align__(16) float cta_o[kDecodeHeads][D];

  const int n = min(max(p.len[b], 0), p.max_len);
  const int chunk = (n + p.splits - 1) / p.splits;
  const int r_begin = min(n, split * chunk);
  const int r_end = min(n, r_begin + chunk);
  const long long seq_off = p.seq_start ? (long long)p.seq_start[b] * p.row_stride : (long long)b * p.seq_stride;
  const __nv_bfloat16* Kb = p.K + seq_off + kh * p.head_stride + li * E;
  const __nv_bfloat16* Vb = p.V + seq_off + kh * p.head_stride + li * E;
  constexpr int kRowsPerIter = kDecodeWarps * GPW;

  for (int h0 = 0; h0 < p.group; h0 += kDecodeHeads) {
    const int nh = min(kDecodeHeads, p.group - h0);
    float q[kDecodeHeads][E];
#pragma unroll
    for (int hh = 0; hh < kDecodeHeads; ++hh) {
      const int h = kh * p.group + h0 + min(hh, nh - 1);
      const uint4 w4 = __ldg(reinterpret_cast<const uint4*>(p.q + (size_t(b) * p.hq + h) * D + li * E));
      const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        q[hh][2 * t] = __uint_as_float(w[t] << 16) * p.scale_log2;
        q[hh][2 * t + 1] = __uint_as_float(w[t] & 0xFFFF0000u) * p.scale_log2;
      }
    }
    float m[kDecodeHeads], l[kDecodeHeads], o[kDecodeHeads][E];
#pragma unroll
    for (int hh = 0; hh < kDecodeHeads; ++hh) {
      m[hh] = -INFINITY;
      l[hh] = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) o[hh][e] = 0.f;
    }
    // Each warp takes GPW consecutive rows per iteration; the loop bound is
    // warp-uniform so that every lane reaches every shuffle.
    uint4 kc = make_uint4(0u, 0u, 0u, 0u), vc = kc;
    {
      const int row = r_begin + warp * GPW + rgw;
      if (row < r_end) {
        kc = __ldg(reinterpret_cast<const uint4*>(Kb + row * p.row_stride));
        vc = __ldg(reinterpret_cast<const uint4*>(Vb + row * p.row_stride));
      }
    }
    for (int rb = r_begin + warp * GPW; rb < r_end; rb += kRowsPerIter) {
      const int row = rb + rgw;
      const int row_next = row + kRowsPerIter;
      uint4 kn = make_uint4(0u, 0u, 0u, 0u), vn = kn;
      if (row_next < r_end) {
        kn = __ldg(reinterpret_cast<const uint4*>(Kb + row_next * p.row_stride));
        vn = __ldg(reinterpret_cast<const uint4*>(Vb + row_next * p.row_stride));
      }
      float k[E], v[E];
      {
        const uint32_t kw[4] = {kc.x, kc.y, kc.z, kc.w}, vw[4] = {vc.x, vc.y, vc.z, vc.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          k[2 * t] = __uint_as_float(kw[t] << 16);
          k[2 * t + 1] = __uint_as_float(kw[t] & 0xFFFF0000u);
          v[2 * t] = __uint_as_float(vw[t] << 16);
          v[2 * t + 1] = __uint_as_float(vw[t] & 0xFFFF0000u);
        }
      }
      const bool valid = row < r_end;
#pragma unroll
      for (int hh = 0; hh < kDecodeHeads; ++hh) {
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) s = fmaf(q[hh][e], k[e], s);
#pragma unroll
        for (int off = 1; off < LPR; off <<= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (valid) {
          const float m_new = fmaxf(m[hh], s);
          const float corr = fast_exp2(m[hh] - m_new);   // 0 on the group's first row (m = -inf)
          const float w = fast_exp2(s - m_new);
          l[hh] = l[hh] * corr + w;
#pragma unroll
          for (int e = 0; e < E; ++e) o[hh][e] = fmaf(o[hh][e], corr, w * v[e]);
          m[hh] = m_new;
        }
      }
      kc = kn;
      vc = vn;
    }
    // Merge the GPW row groups of the warp (lanes li + LPR * g).
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
      for (int hh = 0; hh < kDecodeHeads; ++hh) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m[hh], off);
        const float l2 = __shfl_xor_sync(0xffffffffu, l[hh], off);
        float o2[E];
#pragma unroll
        for (int e = 0; e < E; ++e) o2[e] = __shfl_xor_sync(0xffffffffu, o[hh][e], off);
        softmax_merge<E>(m[hh], l[hh], o[hh], m2, l2, o2);
      }
    }
    if (rgw == 0) {
#pragma unroll
      for (int hh = 0; hh < kDecodeHeads; ++hh) {
        if (li == 0) {
          sm_m[warp][hh] = m[hh];
          sm_l[warp][hh] = l[hh];
        }
#pragma unroll
        for (int e = 0; e < E; ++e) sm_o[warp][hh][li * E + e] = o[hh][e];
      }
    }
    __syncthreads();
    // Merge the warps into the CTA's partial state: one thread per (head,
    // element) combines the warps' states against their common maximum.
    for (int i = threadIdx.x; i < kDecodeHeads * D; i += kDecodeThreads) {
      const int hh = i / D, e = i - hh * D;
      float M = -INFINITY;
#pragma unroll
      for (int w2 = 0; w2 < kDecodeWarps; ++w2) M = fmaxf(M, sm_m[w2][hh]);
      float ll = 0.f, oo = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < kDecodeWarps; ++w2) {
        const float c = M == -INFINITY ? 0.f : fast_exp2(sm_m[w2][hh] - M);
        ll = fmaf(sm_l[w2][hh], c, ll);
        oo = fmaf(sm_o[w2][hh][e], c, oo);
      }
      cta_o[hh][e] = oo;
      if (e == 0) {
        cta_m[hh] = M;
        cta_l[hh] = ll;
      }
    }
    cluster.sync();   // every CTA's partial state is visible cluster-wide
    // Rank 0: one thread per (head, element) combines the cluster's CTAs (in
    // distributed shared memory) and writes the result.
    if (split == 0) {
      for (int i = threadIdx.x; i < kDecodeHeads * D; i += kDecodeThreads) {
        const int hh = i / D, e = i - hh * D;
        if (hh >= nh) continue;
        float M = -INFINITY;
        for (int r = 0; r < p.splits; ++r) M = fmaxf(M, cluster.map_shared_rank(&cta_m[0], r)[hh]);
        float ll = 0.f, oo = 0.f;
        for (int r = 0; r < p.splits; ++r) {
          const float mr = cluster.map_shared_rank(&cta_m[0], r)[hh];
          const float c = M == -INFINITY ? 0.f : fast_exp2(mr - M);
          ll = fmaf(cluster.map_shared_rank(&cta_l[0], r)[hh], c, ll);
          oo = fmaf(cluster.map_shared_rank(&cta_o[0][0], r)[hh * D + e], c, oo);
        }
        const int h = kh * p.group + h0 + hh;
        const float inv = ll > 0.f ? 1.f / ll : 0.f;
        p.O[(size_t(b) * p.hq + h) * D + e] = __float2bfloat16_rn(oo * inv);
        if (e == 0)
          p.LSE[size_t(b) * p.hq + h] = ll > 0.f ? (M + fast_log2(ll)) * 0.69314718055994531f : -INFINITY;
      }
    }
    cluster.sync();   // rank 0 is done reading before any CTA's state is reused or released
  }
}

// ----------------------------------------------------------- split-K decode
//
// Long caches: the cluster split above puts at most kDecodeMaxSplits CTAs on a
// (sequence, KV head), so a batch-1 decode over 8 KV heads uses 128 of the
// 148 SMs with one row in flight per lane group, and is bound by memory
// latency, not bandwidth.  Here the rows of a (sequence, KV head) are split
// over `splits` independent CTAs (any number, no cluster), each lane group
// takes two rows per iteration (both prefetched one iteration ahead, so four
// 16-byte loads are in flight per lane), and each CTA writes its partial
// softmax state -- running max and sum in the log2 domain and the unnormalised
// output of each query head -- to a workspace; decode_merge_kernel then
// combines the splits of each head in split order.  The workspace is the only
// memory written beyond the outputs.
constexpr int kDecodeMaxSplitK = 128;
constexpr int kDecodeMinRowsPerSplit = 256;    // rows per split, short caches
constexpr int kDecodeMaxRowsPerSplit = 1024;   // rows per split, long caches

// CTAs per (sequence, KV head) of the split-K decode for caches of up to
// max_len rows (a pure function of max_len, so a caller can size the
// workspace without the device).  A split takes max_len / 16 rows, at least
// 256 and at most 1024: short caches get more, smaller splits (4096 rows, 8 KV
// heads, d 128: 19.0 us at 256 rows a split against 36.9 at 1024), long ones
// fewer, larger (32 768 rows: 58.4 us at 1024 against 79.9 at 256).
__host__ __device__ inline int decode_splitk_splits(int max_len) {
  int rows = (max_len + 15) / 16;
  rows = rows < kDecodeMinRowsPerSplit ? kDecodeMinRowsPerSplit
                                       : (rows > kDecodeMaxRowsPerSplit ? kDecodeMaxRowsPerSplit : rows);
  const int s = (max_len + rows - 1) / rows;
  return s < 1 ? 1 : (s > kDecodeMaxSplitK ? kDecodeMaxSplitK : s);
}

// Floats of split-K workspace: [batch, hq, splits, D + 2] (output, max, sum).
__host__ __device__ inline size_t decode_splitk_floats(int batch, int hq, int head_dim, int max_len) {
  return size_t(batch) * hq * decode_splitk_splits(max_len) * (head_dim + 2);
}

// kMinBlocks CTAs a SM: 2 for long caches (the compiler then fits a thread in
// 128 registers, with a few bytes of spills, and twice the loads are in flight
// per SM: 131 072 rows, d 128: 194 against 230 us), 1 for short ones (where
// the register limit costs more than the extra occupancy brings).
template <int D, int kMinBlocks>
__global__ void __launch_bounds__(kDecodeThreads, kMinBlocks) decode_splitk_kernel(const DecodeParams p,
                                                                                 float* part) {
  pdl_wait();
  pdl_launch_dependents();
  constexpr int E = 8;           // elements of a row per lane (one 16-byte load)
  constexpr int LPR = D / E;     // lanes per row
  constexpr int GPW = 32 / LPR;  // row groups per warp
  const int split = blockIdx.x % p.splits;
  const int kh = blockIdx.x / p.splits;
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rgw = lane / LPR;
  const int li = lane % LPR;
  __shared__ float sm_m[kDecodeWarps][kDecodeHeads], sm_l[kDecodeWarps][kDecodeHeads];
  __shared__ __align__(16) float sm_o[kDecodeWarps][kDecodeHeads][D];

  const int n = min(max(p.len[b], 0), p.max_len);
  const int chunk = (n + p.splits - 1) / p.splits;
  const int r_begin = min(n, split * chunk);
  const int r_end = min(n, r_begin + chunk);
  const long long seq_off = p.seq_start ? (long long)p.seq_start[b] * p.row_stride : (long long)b * p.seq_stride;
  const __nv_bfloat16* Kb = p.K + seq_off + kh * p.head_stride + li * E;
  const __nv_bfloat16* Vb = p.V + seq_off + kh * p.head_stride + li * E;
  constexpr int kRowsPerIter = kDecodeWarps * GPW;   // rows of one sweep of the CTA
  constexpr int kStep = 2 * kRowsPerIter;             // two sweeps per iteration

  auto unpack = [](const uint4& w4, float (&x)[E]) {
    const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      x[2 * t] = __uint_as_float(w[t] << 16);
      x[2 * t + 1] = __uint_as_float(w[t] & 0xFFFF0000u);
    }
  };

  for (int h0 = 0; h0 < p.group; h0 += kDecodeHeads) {
    const int nh = min(kDecodeHeads, p.group - h0);
    float q[kDecodeHeads][E];
#pragma unroll
    for (int hh = 0; hh < kDecodeHeads; ++hh) {
      const int h = kh * p.group + h0 + min(hh, nh - 1);
      const uint4 w4 = __ldg(reinterpret_cast<const uint4*>(p.q + (size_t(b) * p.hq + h) * D + li * E));
      unpack(w4, q[hh]);
#pragma unroll
      for (int e = 0; e < E; ++e) q[hh][e] *= p.scale_log2;
    }
    float m[kDecodeHeads], l[kDecodeHeads], o[kDecodeHeads][E];
#pragma unroll
    for (int hh = 0; hh < kDecodeHeads; ++hh) {
      m[hh] = -INFINITY;
      l[hh] = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) o[hh][e] = 0.f;
    }
    // Rows rb + rgw and rb + rgw + kRowsPerIter per iteration; the loop bound is
    // warp-uniform so every lane reaches every shuffle.
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    uint4 ka = z, va = z, kb = z, vb = z;
    {
      const int r0 = r_begin + warp * GPW + rgw, r1 = r0 + kRowsPerIter;
      if (r0 < r_end) {
        ka = __ldg(reinterpret_cast<const uint4*>(Kb + r0 * p.row_stride));
        va = __ldg(reinterpret_cast<const uint4*>(Vb + r0 * p.row_stride));
      }
      if (r1 < r_end) {
        kb = __ldg(reinterpret_cast<const uint4*>(Kb + r1 * p.row_stride));
        vb = __ldg(reinterpret_cast<const uint4*>(Vb + r1 * p.row_stride));
      }
    }
    for (int rb = r_begin + warp * GPW; rb < r_end; rb += kStep) {
      const int r0 = rb + rgw, r1 = r0 + kRowsPerIter;
      const int n0 = r0 + kStep, n1 = r1 + kStep;
      uint4 kan = z, van = z, kbn = z, vbn = z;
      if (n0 < r_end) {
        kan = __ldg(reinterpret_cast<const uint4*>(Kb + n0 * p.row_stride));
        van = __ldg(reinterpret_cast<const uint4*>(Vb + n0 * p.row_stride));
      }
      if (n1 < r_end) {
        kbn = __ldg(reinterpret_cast<const uint4*>(Kb + n1 * p.row_stride));
        vbn = __ldg(reinterpret_cast<const uint4*>(Vb + n1 * p.row_stride));
      }
      float k0[E], v0[E], k1[E], v1[E];
      unpack(ka, k0);
      unpack(va, v0);
      unpack(kb, k1);
      unpack(vb, v1);
      const bool ok0 = r0 < r_end, ok1 = r1 < r_end;
#pragma unroll
      for (int hh = 0; hh < kDecodeHeads; ++hh) {
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          s0 = fmaf(q[hh][e], k0[e], s0);
          s1 = fmaf(q[hh][e], k1[e], s1);
        }
#pragma unroll
        for (int off = 1; off < LPR; off <<= 1) {
          s0 += __shfl_xor_sync(0xffffffffu, s0, off);
          s1 += __shfl_xor_sync(0xffffffffu, s1, off);
        }
        s0 = ok0 ? s0 : -INFINITY;
        s1 = ok1 ? s1 : -INFINITY;
        const float m_new = fmax3(m[hh], s0, s1);
        if (m_new != -INFINITY) {
          const float corr = fast_exp2(m[hh] - m_new);   // 0 on the group's first row (m = -inf)
          const float w0 = fast_exp2(s0 - m_new);
          const float w1 = fast_exp2(s1 - m_new);
          l[hh] = l[hh] * corr + w0 + w1;
#pragma unroll
          for (int e = 0; e < E; ++e) o[hh][e] = fmaf(o[hh][e], corr, fmaf(w0, v0[e], w1 * v1[e]));
          m[hh] = m_new;
        }
      }
      ka = kan;
      va = van;
      kb = kbn;
      vb = vbn;
    }
    // Merge the GPW row groups of the warp (lanes li + LPR * g).
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
      for (int hh = 0; hh < kDecodeHeads; ++hh) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m[hh], off);
        const float l2 = __shfl_xor_sync(0xffffffffu, l[hh], off);
        float o2[E];
#pragma unroll
        for (int e = 0; e < E; ++e) o2[e] = __shfl_xor_sync(0xffffffffu, o[hh][e], off);
        softmax_merge<E>(m[hh], l[hh], o[hh], m2, l2, o2);
      }
    }
    if (rgw == 0) {
#pragma unroll
      for (int hh = 0; hh < kDecodeHeads; ++hh) {
        if (li == 0) {
          sm_m[warp][hh] = m[hh];
          sm_l[warp][hh] = l[hh];
        }
#pragma unroll
        for (int e = 0; e < E; ++e) sm_o[warp][hh][li * E + e] = o[hh][e];
      }
    }
    __syncthreads();
    // The CTA's partial state of each head, merged over the warps in warp
    // order, to the workspace: [b, h, split] = (o[0..D), m, l).
    for (int i = threadIdx.x; i < kDecodeHeads * D; i += kDecodeThreads) {
      const int hh = i / D, e = i - hh * D;
      if (hh >= nh) continue;
      float M = -INFINITY;
#pragma unroll
      for (int w2 = 0; w2 < kDecodeWarps; ++w2) M = fmaxf(M, sm_m[w2][hh]);
      float ll = 0.f, oo = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < kDecodeWarps; ++w2) {
        const float c = M == -INFINITY ? 0.f : fast_exp2(sm_m[w2][hh] - M);
        ll = fmaf(sm_l[w2][hh], c, ll);
        oo = fmaf(sm_o[w2][hh][e], c, oo);
      }
      const int h = kh * p.group + h0 + hh;
      float* dst = part + ((size_t(b) * p.hq + h) * p.splits + split) * (D + 2);
      dst[e] = oo;
      if (e == 0) {
        dst[D] = M;
        dst[D + 1] = ll;
      }
    }
    __syncthreads();   // the warps' states are read before the next head group overwrites them
  }
}

// Merge of the split-K partial states: one CTA of D threads per (sequence,
// query head), thread e combining element e of every split in split order.
template <int D>
__global__ void __launch_bounds__(D) decode_merge_kernel(const float* part, int hq, int splits, __nv_bfloat16* O,
                                                         float* LSE) {
  pdl_wait();
  pdl_launch_dependents();
  const int h = blockIdx.x, b = blockIdx.y, e = threadIdx.x;
  const float* src = part + (size_t(b) * hq + h) * splits * (D + 2);
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, src[size_t(s) * (D + 2) + D]);
  float ll = 0.f, oo = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float* ps = src + size_t(s) * (D + 2);
    const float c = M == -INFINITY ? 0.f : fast_exp2(ps[D] - M);
    ll = fmaf(ps[D + 1], c, ll);
    oo = fmaf(ps[e], c, oo);
  }
  const float inv = ll > 0.f ? 1.f / ll : 0.f;
  O[(size_t(b) * hq + h) * D + e] = __float2bfloat16_rn(oo * inv);
  if (e == 0) LSE[size_t(b) * hq + h] = ll > 0.f ? (M + fast_log2(ll)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace lt
