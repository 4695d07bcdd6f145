// lazy_ratio.cuh -- lazy ratio of each (sequence, query head) from the LSE.
//
// Press-release page ("LLM突破：推理加速，长CoT生成惊艳", section
// "LightTransfer方法详解"): the lazy ratio sums the attention weights from a
// query to the initial and the recent keys.  LightTransfer write-up (first
// solution of LightTransfer-Test): FlashAttention's LSE is the denominator, so
// each query only visits its S + W numerator keys:
//     K_i = [0, min(S, i+1)) U [max(S, i-W+1), i]
//     r_i = sum_{j in K_i} exp2(log2e * scale * q_i.k_j - log2e * LSE_i)
//     ratio[b, h] = mean of r_i over the last n' = min(n_obs, N_b) rows.
//
// The scores of one (sequence, query head) form a dense contraction of its
// observed query rows with the key band [0, min(S, N)) ++
// [max(S, N - n' - W + 1), N) of its KV head; they run on the tensor cores
// (mma.sync m16n8k16, bf16 in, fp32 accumulate: the tiles are a few KB, far
// too small to amortise tcgen05's TMEM allocation and mbarrier hand-offs).
//
// Work split: one cluster of C <= 8 CTAs per (sequence, query head), CTA
// `rank` taking a contiguous slice of the band (about 160 keys), so the grid
// (C x hq x batch) covers every SM at the benchmark's shapes.  Each warp takes
// a 16-row block of the observed rows (its Q fragments loaded from global
// memory while the CTA's key slice is still being staged in shared memory by
// cp.async) and a share of the slice's 8-key tiles; tiles no row of the block
// needs are skipped, every score is masked to K_i of its row, turned into
// exp2(. - LSE) and summed.  The warps' sums are added in warp order, the
// CTAs' in rank order through distributed shared memory: deterministic, with
// no atomics and no global scratch.
#pragma once

#include <cooperative_groups.h>

#include "lt_device.cuh"

namespace lt {

struct RatioParams {
  int batch;
  int total_tokens;
  int hq;
  int hkv;
  int group;
  int S;
  int W;
  int n_obs;
  const int32_t* cu_seqlens;
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  const float* LSE;
  float scale_log2;  // softmax scale * log2(e)
  float* ratio;      // [batch, hq]
};

constexpr int kRatioWarps = 8;
constexpr int kRatioMaxCluster = 8;
constexpr int kRatioKeysPerCta = 160;   // target slice of the band per CTA

template <int D>
struct RatioLayout {
  static constexpr int kRowElems = D + 8;             // padded key row: conflict-free fragment loads
  static constexpr int kPiece = 256;                  // keys staged at a time
  static constexpr int kKeyBytes = kPiece * kRowElems * 2;
  static constexpr int kBytes = kKeyBytes + kRatioWarps * 4 + 16;
};

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void mma_m16n8k16_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int D>
__global__ void __launch_bounds__(kRatioWarps * 32) lazy_ratio_kernel(const RatioParams p) {
  using Lay = RatioLayout<D>;
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(16) uint8_t smem[];
  __nv_bfloat16* keys = reinterpret_cast<__nv_bfloat16*>(smem);
  float* warp_sum = reinterpret_cast<float*>(smem + Lay::kKeyBytes);   // [kRatioWarps]
  float* cta_sum = warp_sum + kRatioWarps;                              // [1], read by rank 0

  const int C = int(cluster.num_blocks());
  const int rank = int(cluster.block_rank());
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int kh = h / p.group;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int gq = lane >> 2;  // fragment row (and row + 8)
  const int tq = lane & 3;   // fragment column pair

  int start = 0, N = p.total_tokens;
  if (p.cu_seqlens) {
    start = p.cu_seqlens[b];
    N = p.cu_seqlens[b + 1] - start;
  }
  const int nb = N < p.n_obs ? N : p.n_obs;   // observed rows: [N - nb, N)
  const int nrb = (nb + 15) / 16;

  // The key band of all observed rows, as a list: sinks, then the window.
  const int n_sink = min(p.S, N);
  const int w_lo = max(p.S, N - nb - p.W + 1);
  const int nk = n_sink + max(0, N - w_lo);
  int per = (nk + C - 1) / C;
  per = (per + 7) & ~7;
  const int x_begin = min(nk, rank * per);
  const int x_end = min(nk, x_begin + per);
  auto pos_of = [&](int x) { return x < n_sink ? x : w_lo + (x - n_sink); };

  // Warps per row block: all eight warps share the row blocks, and the
  // warps of one block split its key tiles.
  int blocks_per_pass = 1;
  while (blocks_per_pass * 2 <= min(nrb, kRatioWarps)) blocks_per_pass *= 2;
  const int wprb = kRatioWarps / blocks_per_pass;
  const int rb_first = warp / wprb;
  const int tg_first = warp % wprb;

  // Q fragments and LSE of one 16-row block (rows i0 .. i0+15).
  uint32_t afrag[D / 16][4];
  float lse2[2];
  bool rvalid[2];
  int rb_loaded = -1;
  auto load_rows = [&](int rb) {
    const int rows = min(16, nb - rb * 16);
    const int i0 = N - nb + rb * 16;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int r = gq + half * 8;
      rvalid[half] = r < rows;
      const int i = i0 + (rvalid[half] ? r : 0);
      lse2[half] = rvalid[half] ? p.LSE[size_t(h) * p.total_tokens + start + i] * 1.4426950408889634f : 0.f;
      const uint32_t* qrow = reinterpret_cast<const uint32_t*>(p.Q + ((size_t(start) + i) * p.hq + h) * D);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        afrag[ks][half] = rvalid[half] ? qrow[ks * 8 + tq] : 0u;
        afrag[ks][half + 2] = rvalid[half] ? qrow[ks * 8 + 4 + tq] : 0u;
      }
    }
    rb_loaded = rb;
  };

  float acc_row[2] = {0.f, 0.f};
  for (int p0 = x_begin; p0 < x_end; p0 += Lay::kPiece) {
    const int p1 = min(x_end, p0 + Lay::kPiece);
    const int ntiles = (p1 - p0 + 7) >> 3;
    __syncthreads();   // the previous piece is no longer read
    {
      const uint32_t base = smem_u32(keys);
      const int pieces = ntiles * 8 * (D / 8);
      for (int x = threadIdx.x; x < pieces; x += blockDim.x) {
        const int key = x / (D / 8);
        const int part = x - key * (D / 8);
        const int kx = p0 + key;
        const bool in = kx < p1;
        const __nv_bfloat16* src = p.K + ((size_t(start) + (in ? pos_of(kx) : 0)) * p.hkv + kh) * D + part * 8;
        cp_async_16(base + (key * Lay::kRowElems + part * 8) * 2, src, in ? 16u : 0u);
      }
      cp_async_commit();
    }
    // The warp's first row block is fetched while the keys are in flight.
    if (rb_first < nrb && rb_loaded < 0) load_rows(rb_first);
    cp_async_wait_all();
    __syncthreads();

    const int ngroups = (ntiles + 3) >> 2;   // four 8-key tiles per pass
    for (int rb = rb_first; rb < nrb; rb += blocks_per_pass) {
      if (rb != rb_loaded) load_rows(rb);
      const int i0 = N - nb + rb * 16;
      const int i_last = i0 + min(16, nb - rb * 16) - 1;
      const int win_lo = i0 - p.W + 1;   // earliest window key of the block's rows
      for (int tg = tg_first; tg < ngroups; tg += wprb) {
        const int nt0 = tg * 4;
        bool need[4];
        float acc[4][4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int nt = nt0 + q;
          const int xa = p0 + nt * 8;
          need[q] = false;
          if (nt < ntiles) {
            const int pmin = pos_of(xa);
            const int pmax = pos_of(min(xa + 7, p1 - 1));
            need[q] = pmin <= i_last && (pmin < p.S || pmax >= win_lo);   // warp-uniform
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[q][e] = 0.f;
        }
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (!need[q]) continue;
            const uint32_t* krow = reinterpret_cast<const uint32_t*>(keys + ((nt0 + q) * 8 + gq) * Lay::kRowElems);
            mma_m16n8k16_bf16(acc[q], afrag[ks], krow[ks * 8 + tq], krow[ks * 8 + 4 + tq]);
          }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (!need[q]) continue;
          const int xa = p0 + (nt0 + q) * 8;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int half = e >> 1;
            const int kx = xa + 2 * tq + (e & 1);
            const int j = pos_of(kx);
            const int i = i0 + gq + half * 8;
            const bool take = rvalid[half] && kx < p1 && j <= i && (j < p.S || j >= i - p.W + 1);
            const float w = fast_exp2(fmaf(acc[q][e], p.scale_log2, -lse2[half]));
            acc_row[half] += take ? w : 0.f;
          }
        }
      }
    }
  }

  // Fixed-order reduction: lanes, then warps, then the cluster's CTAs.
  float v = acc_row[0] + acc_row[1];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  if (lane == 0) warp_sum[warp] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < kRatioWarps; ++w) t += warp_sum[w];
    *cta_sum = t;
  }
  cluster.sync();
  if (rank == 0 && threadIdx.x == 0) {
    float total = 0.f;
    for (int r = 0; r < C; ++r) total += *cluster.map_shared_rank(cta_sum, r);
    p.ratio[size_t(b) * p.hq + h] = nb > 0 ? total / float(nb) : 0.f;
  }
  cluster.sync();   // rank 0 has read every CTA's sum before any CTA exits
}

}  // namespace lt
