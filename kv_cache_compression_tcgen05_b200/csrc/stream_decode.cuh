// stream_decode.cuh -- decode on a demoted layer's streaming KV cache.
//
// Press-release page ("LLM突破：推理加速，长CoT生成惊艳"): the converted layers
// use streaming attention, which needs only a constant-size KV cache; the
// LightTransfer project page: the lazy layers pay attention mostly to the
// initial and the recent tokens.  After compaction a lazy layer keeps, per
// sequence and KV head, S + W rows: the S sink positions and the W most recent
// ones.  At decode the new token's key/value enter the window (replacing its
// oldest row once the cache is full) and the token attends to the cached rows:
//     K_p = [0, min(S, p+1)) U [max(S, p-W+1), p]   (p = the token's position)
// -- the same key set the lazy ratio measures.
//
// Cache layout: [batch, hkv, S+W, d] bf16 (as lt_compact_kv writes it), with
// len[b] valid rows; rows [0, S) are the sinks, rows [S, S+W) the window, used
// as a ring once full: next[b] is the slot the next token goes to.
//
// The decode is bandwidth bound (each cached row is read once per KV head for
// all g query heads of the group): one CTA per (KV head, sequence), 4 warps,
// each 8-lane group of a warp takes one key row at a time with 16-byte loads;
// scores are reduced over the 8 lanes with shuffles, each row group keeps a
// running (max, sum, output) per head in the log2 domain, and the 16 row
// groups are merged through shuffles and shared memory.
#pragma once

#include "lt_device.cuh"

namespace lt {

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

struct DecodeParams {
  int batch, hq, hkv, group, slots;
  const __nv_bfloat16* q;   // [batch, hq, d]
  const __nv_bfloat16* K;   // [batch, hkv, slots, d]
  const __nv_bfloat16* V;
  const int32_t* len;       // [batch]
  __nv_bfloat16* O;         // [batch, hq, d]
  float* LSE;               // [batch, hq]
  float scale_log2;
};

constexpr int kDecodeHeads = 4;   // query heads per pass over the cache

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
__global__ void __launch_bounds__(128) stream_decode_kernel(const DecodeParams p) {
  constexpr int E = D / 8;                 // elements of a row per lane
  const int kh = blockIdx.x;
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rg = lane >> 3;                // row group in the warp
  const int li = lane & 7;                 // lane in the row group
  __shared__ float sm_m[4][kDecodeHeads], sm_l[4][kDecodeHeads];
  __shared__ float sm_o[4][kDecodeHeads][D];
  const int n = min(p.len[b], p.slots);
  const size_t row0 = (size_t(b) * p.hkv + kh) * p.slots;

  for (int h0 = 0; h0 < p.group; h0 += kDecodeHeads) {
    const int nh = min(kDecodeHeads, p.group - h0);
    float q[kDecodeHeads][E];
#pragma unroll
    for (int hh = 0; hh < kDecodeHeads; ++hh) {
      const int h = kh * p.group + h0 + min(hh, nh - 1);
      const __nv_bfloat16* qr = p.q + (size_t(b) * p.hq + h) * D + li * E;
#pragma unroll
      for (int e = 0; e < E; ++e) q[hh][e] = __bfloat162float(qr[e]) * p.scale_log2;
    }
    float m[kDecodeHeads], l[kDecodeHeads], o[kDecodeHeads][E];
#pragma unroll
    for (int hh = 0; hh < kDecodeHeads; ++hh) {
      m[hh] = -INFINITY;
      l[hh] = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) o[hh][e] = 0.f;
    }
    for (int row = warp * 4 + rg; row < n; row += 16) {
      const uint4* kr = reinterpret_cast<const uint4*>(p.K + (row0 + row) * D + li * E);
      const uint4* vr = reinterpret_cast<const uint4*>(p.V + (row0 + row) * D + li * E);
      float k[E], v[E];
#pragma unroll
      for (int c = 0; c < E / 8; ++c) {
        const uint4 kk = kr[c], vv = vr[c];
        const uint32_t kw[4] = {kk.x, kk.y, kk.z, kk.w}, vw[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          k[c * 8 + 2 * t] = __uint_as_float(kw[t] << 16);
          k[c * 8 + 2 * t + 1] = __uint_as_float(kw[t] & 0xFFFF0000u);
          v[c * 8 + 2 * t] = __uint_as_float(vw[t] << 16);
          v[c * 8 + 2 * t + 1] = __uint_as_float(vw[t] & 0xFFFF0000u);
        }
      }
#pragma unroll
      for (int hh = 0; hh < kDecodeHeads; ++hh) {
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) s = fmaf(q[hh][e], k[e], s);
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        s += __shfl_xor_sync(0xffffffffu, s, 4);
        const float m_new = fmaxf(m[hh], s);
        const float corr = fast_exp2(m[hh] - m_new);   // 0 on the first row (m = -inf)
        const float w = fast_exp2(s - m_new);
        l[hh] = l[hh] * corr + w;
#pragma unroll
        for (int e = 0; e < E; ++e) o[hh][e] = fmaf(o[hh][e], corr, w * v[e]);
        m[hh] = m_new;
      }
    }
    // Merge the 4 row groups of the warp (lanes li, li+8, li+16, li+24).
#pragma unroll
    for (int off = 8; off <= 16; off <<= 1) {
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
    if (rg == 0) {
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
    // Warp 0, row group 0: merge the 4 warps and write the result.
    if (warp == 0 && rg == 0) {
#pragma unroll
      for (int hh = 0; hh < kDecodeHeads; ++hh) {
        float mm = sm_m[0][hh], ll = sm_l[0][hh], oo[E];
#pragma unroll
        for (int e = 0; e < E; ++e) oo[e] = sm_o[0][hh][li * E + e];
        for (int w2 = 1; w2 < 4; ++w2) {
          float o2[E];
#pragma unroll
          for (int e = 0; e < E; ++e) o2[e] = sm_o[w2][hh][li * E + e];
          softmax_merge<E>(mm, ll, oo, sm_m[w2][hh], sm_l[w2][hh], o2);
        }
        if (hh < nh) {
          const int h = kh * p.group + h0 + hh;
          const float inv = ll > 0.f ? 1.f / ll : 0.f;
          __nv_bfloat16* orow = p.O + (size_t(b) * p.hq + h) * D + li * E;
#pragma unroll
          for (int e = 0; e < E; e += 2)
            *reinterpret_cast<uint32_t*>(orow + e) = pack_bf16x2(oo[e] * inv, oo[e + 1] * inv);
          if (li == 0)
            p.LSE[size_t(b) * p.hq + h] = ll > 0.f ? (mm + fast_log2(ll)) * 0.69314718055994531f : -INFINITY;
        }
      }
    }
    __syncthreads();
  }
}

}  // namespace lt
