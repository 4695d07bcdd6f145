// attn_fwd.cuh -- causal GQA prefill attention with per-row LSE for sm_100a.
//
// The LightTransfer write-up (xzbcqc.com news page, first solution of
// LightTransfer-Test) reuses the log-sum-exp that a FlashAttention-style prefill
// produces as the denominator of the lazy ratio.  This kernel is that prefill,
// built for B200:
//
//   * persistent: one CTA per SM walks a list of (q-tile, sequence, head) work
//     items, heaviest causal tiles first, in snake order across CTAs;
//   * warp-specialised, 6 warps:
//       warp 0      TMA producer: Q tile (double buffered) and a ring of K/V
//                   tiles (128 keys x d, 128-byte swizzle), one mbarrier each;
//       warp 1      owns the TMEM allocation; one thread issues tcgen05.mma:
//                   S = Q K^T into one of two TMEM score buffers, then
//                   O += P V into the TMEM output accumulator;
//       warps 2..5  softmax: thread = query row = TMEM lane.  tcgen05.ld of the
//                   128 scores, causal mask on the diagonal tile, running max
//                   in the log2 domain, exp2, bf16 P written to shared memory in
//                   the MMA's swizzled K-major layout, lazy O rescale (only when
//                   the running max grows by more than 2^8), epilogue O / l and
//                   LSE = (m + log2 l) ln 2 written once.
//   * tiles: 128 query rows x 128 keys; M = 128, N = 128 (S) and N = d (PV),
//     K-step 16 per tcgen05.mma.
//
// TMEM columns: [0,128) S buffer 0, [128,256) S buffer 1, [256, 256+d) O.
#pragma once

#include "lt_device.cuh"

namespace lt {

struct AttnParams {
  int batch;
  int total_tokens;
  int hq;
  int hkv;
  int n_qtiles;     // ceil(max_seqlen / 128)
  int num_tiles;    // n_qtiles * batch * hq
  const int32_t* cu_seqlens;  // device [batch+1] or null (one sequence)
  __nv_bfloat16* O;
  float* LSE;
  float scale_log2;  // softmax scale * log2(e)
  unsigned* status;
};

template <int D>
struct AttnLayout {
  static constexpr int kBlock = 128;                  // query rows = keys per tile
  static constexpr int kTileBytes = kBlock * D * 2;   // one Q, K or V tile
  static constexpr int kSub = 16384;                  // one 128 x 64 bf16 swizzled sub-tile
  static constexpr int kStages = D == 64 ? 4 : 3;     // K/V ring slots
  static constexpr int kPBytes = kBlock * kBlock * 2;
  static constexpr int kQOff = 0;
  static constexpr int kRingOff = kQOff + 2 * kTileBytes;
  static constexpr int kPOff = kRingOff + kStages * kTileBytes;
  static constexpr int kBarOff = kPOff + 2 * kPBytes;
  static constexpr int kNumBars = 2 + 2 + 2 * kStages + 2 + 2 + 2 + 1 + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;        // room to align the base to 1024 B
  static constexpr int kThreads = 192;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kTmemO = 256;
};

struct AttnTile {
  int b, h, qt, start, len;
};

// Work item t -> (sequence, head, q-tile); false when the q-tile lies beyond the
// sequence.  Items are ordered heaviest q-tile first; within one q-tile the
// heads of one sequence are consecutive, so CTAs running at the same time share
// K/V tiles through L2.
__device__ __forceinline__ bool attn_decode(const AttnParams& p, int t, AttnTile& tile) {
  const int bh = p.batch * p.hq;
  tile.qt = p.n_qtiles - 1 - t / bh;
  const int rem = t - (t / bh) * bh;
  tile.b = rem / p.hq;
  tile.h = rem - tile.b * p.hq;
  if (p.cu_seqlens) {
    tile.start = p.cu_seqlens[tile.b];
    tile.len = p.cu_seqlens[tile.b + 1] - tile.start;
  } else {
    tile.start = 0;
    tile.len = p.total_tokens;
  }
  return tile.qt * 128 < tile.len;
}

// Snake order: CTA c takes item k*G + c on even rounds and k*G + (G-1-c) on odd
// rounds, so the heaviest items are spread evenly.
__device__ __forceinline__ int attn_item(int round, int cta, int grid) {
  return round * grid + ((round & 1) ? (grid - 1 - cta) : cta);
}

template <int D>
__global__ void __launch_bounds__(AttnLayout<D>::kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using Lay = AttnLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + Lay::kQOff;
  uint8_t* sRing = smem + Lay::kRingOff;
  uint8_t* sP = smem + Lay::kPOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBarOff);
  uint64_t* q_full = bars;                       // [2]  TMA -> MMA
  uint64_t* q_empty = q_full + 2;                // [2]  MMA -> TMA
  uint64_t* kv_full = q_empty + 2;               // [kStages]
  uint64_t* kv_empty = kv_full + Lay::kStages;   // [kStages]
  uint64_t* s_full = kv_empty + Lay::kStages;    // [2]  MMA -> softmax
  uint64_t* p_full = s_full + 2;                 // [2]  softmax -> MMA (128 arrivals)
  uint64_t* pv_done = p_full + 2;                // [2]  MMA -> softmax
  uint64_t* o_empty = pv_done + 2;               // [1]  softmax -> MMA (128 arrivals)
  uint64_t* drain = o_empty + 1;                 // [1]  MMA drain on abort
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMiscOff + 4);
  // Never raised: the drain waits after an abort end on completion or time only.
  volatile int* no_abort = reinterpret_cast<volatile int*>(smem + Lay::kMiscOff + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int grid = gridDim.x;
  const int cta = blockIdx.x;
  const int group = p.hq / p.hkv;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
      mbar_init(&pv_done[i], 1);
    }
    for (int i = 0; i < Lay::kStages; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(o_empty, 128);
    mbar_init(drain, 1);
    *abort_flag = 0;
    *no_abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Lay::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.status};

  if (warp == 0) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      int it = 0, tl = 0;
      bool ok = true;
      for (int round = 0; ok && round * grid < p.num_tiles; ++round) {
        const int t = attn_item(round, cta, grid);
        AttnTile tile;
        if (t >= p.num_tiles || !attn_decode(p, t, tile)) continue;
        const int qb = tl & 1;
        if (tl >= 2 && !(ok = mbar_wait(&q_empty[qb], ((tl >> 1) - 1) & 1, ctl))) break;
        mbar_expect_tx(&q_full[qb], Lay::kTileBytes);
        for (int st = 0; st < D / 64; ++st)
          tma_load_3d(sQ + qb * Lay::kTileBytes + st * Lay::kSub, &tmQ, &q_full[qb], st * 64, tile.h,
                      tile.start + tile.qt * 128);
        const int n = tile.qt + 1;
        const int kh = tile.h / group;
        // Order of use by the MMA thread: K0, K1, V0, K2, V1, ..., V(n-1).
        for (int step = 0; ok && step <= n; ++step) {
          for (int which = 0; which < 2; ++which) {
            const bool isK = which == 0;
            if (isK ? step >= n : step < 1) continue;
            const int j = isK ? step : step - 1;
            const int slot = it % Lay::kStages;
            if (it >= Lay::kStages && !(ok = mbar_wait(&kv_empty[slot], ((it / Lay::kStages) - 1) & 1, ctl)))
              break;
            mbar_expect_tx(&kv_full[slot], Lay::kTileBytes);
            for (int st = 0; st < D / 64; ++st)
              tma_load_3d(sRing + slot * Lay::kTileBytes + st * Lay::kSub, isK ? &tmK : &tmV, &kv_full[slot],
                          st * 64, kh, tile.start + j * 128);
            ++it;
          }
        }
        ++tl;
      }
      if (!ok) {
        // Let the loads already issued land before the CTA's shared memory is
        // released (bounded; the abort flag is ignored here).
        const int first = it > Lay::kStages ? it - Lay::kStages : 0;
        for (int x = first; x < it; ++x) {
          const WaitCtl drain_ctl{no_abort, p.status};
          mbar_wait(&kv_full[x % Lay::kStages], (x / Lay::kStages) & 1, drain_ctl);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t kIdPV = idesc_bf16_f32(128, D, 0, 1);
      int it = 0, js = 0, tl = 0;
      bool ok = true;
      for (int round = 0; ok && round * grid < p.num_tiles; ++round) {
        const int t = attn_item(round, cta, grid);
        AttnTile tile;
        if (t >= p.num_tiles || !attn_decode(p, t, tile)) continue;
        const int qb = tl & 1;
        if (!(ok = mbar_wait(&q_full[qb], (tl >> 1) & 1, ctl))) break;
        const uint32_t q_addr = smem_u32(sQ + qb * Lay::kTileBytes);
        const int n = tile.qt + 1;

        auto issue_s = [&](int g) -> bool {
          const int slot = it % Lay::kStages;
          if (!mbar_wait(&kv_full[slot], (it / Lay::kStages) & 1, ctl)) return false;
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sRing + slot * Lay::kTileBytes);
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = (k >> 2) * Lay::kSub + (k & 3) * 32;
            mma_bf16_ss(tmem + (g & 1) * 128, smem_desc_sw128(q_addr + off, 16, 1024),
                        smem_desc_sw128(k_addr + off, 16, 1024), kIdS, k > 0 ? 1u : 0u);
          }
          mma_commit(&kv_empty[slot]);
          mma_commit(&s_full[g & 1]);
          ++it;
          return true;
        };
        auto issue_pv = [&](int g, int j) -> bool {
          if (!mbar_wait(&p_full[g & 1], (g >> 1) & 1, ctl)) return false;
          if (j == 0 && tl > 0 && !mbar_wait(o_empty, (tl - 1) & 1, ctl)) return false;
          const int slot = it % Lay::kStages;
          if (!mbar_wait(&kv_full[slot], (it / Lay::kStages) & 1, ctl)) return false;
          tc_fence_after();
          const uint32_t p_addr = smem_u32(sP + (g & 1) * Lay::kPBytes);
          const uint32_t v_addr = smem_u32(sRing + slot * Lay::kTileBytes);
#pragma unroll
          for (int k = 0; k < 128 / 16; ++k) {
            const uint64_t a = smem_desc_sw128(p_addr + (k >> 2) * Lay::kSub + (k & 3) * 32, 16, 1024);
            const uint64_t b = smem_desc_sw128(v_addr + k * 2048, Lay::kSub, 1024);
            mma_bf16_ss(tmem + Lay::kTmemO, a, b, kIdPV, (j > 0 || k > 0) ? 1u : 0u);
          }
          mma_commit(&kv_empty[slot]);
          mma_commit(&pv_done[g & 1]);
          ++it;
          return true;
        };

        if (!(ok = issue_s(js))) break;
        if (n == 1) mma_commit(&q_empty[qb]);
        for (int j = 0; ok && j < n; ++j) {
          if (j + 1 < n) {
            if (!(ok = issue_s(js + j + 1))) break;
            if (j + 2 == n) mma_commit(&q_empty[qb]);
          }
          ok = issue_pv(js + j, j);
        }
        js += n;
        ++tl;
      }
      if (!ok) {
        mma_commit(drain);
        const WaitCtl drain_ctl{no_abort, p.status};
        mbar_wait(drain, 0, drain_ctl);
      }
    }
  } else {
    // --------------------------------------------------------------- softmax
    const int wq = warp & 3;                  // TMEM lane quarter of this warp
    const int row = wq * 32 + lane;           // query row within the tile
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const float sl2 = p.scale_log2;
    int js = 0, tl = 0;
    bool ok = true;
    for (int round = 0; ok && round * grid < p.num_tiles; ++round) {
      const int t = attn_item(round, cta, grid);
      AttnTile tile;
      if (t >= p.num_tiles || !attn_decode(p, t, tile)) continue;
      const int n = tile.qt + 1;
      const int qpos = tile.qt * 128 + row;
      float m_run = -INFINITY;   // running max of scale*log2(e)*s, possibly stale by < 8
      float l_run = 0.f;         // running sum of exp2(.. - m_run)
      for (int j = 0; j < n; ++j) {
        const int g = js + j;
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[g & 1], (g >> 1) & 1, ctl));
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[128];
        {
          uint32_t(&c0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
          uint32_t(&c1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
          uint32_t(&c2)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[64]);
          uint32_t(&c3)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[96]);
          const uint32_t sa = tmem + lane_off + (g & 1) * 128;
          tmem_ld32(sa + 0, c0);
          tmem_ld32(sa + 32, c1);
          tmem_ld32(sa + 64, c2);
          tmem_ld32(sa + 96, c3);
          tmem_wait_ld();
        }
        float s[128];
#pragma unroll
        for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(sr[c]);
        if (j == tile.qt) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c > row) s[c] = -INFINITY;
        }
        // Row maximum as 8 independent chains (short dependency chains).
        float mx8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx8[k] = s[k];
#pragma unroll
        for (int c = 8; c < 128; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], s[c]);
        const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        const float m_new = fmaxf(m_run, mx * sl2);
        const bool need = m_new > m_run + 8.f;
        float alpha = 1.f;
        if (need) {
          alpha = fast_exp2(m_run - m_new);
          m_run = m_new;
        }
        l_run *= alpha;
        uint32_t pk[64];
        float sum8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        const float neg_m = -m_run;
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float p0 = fast_exp2(fmaf(s[2 * c], sl2, neg_m));
          const float p1 = fast_exp2(fmaf(s[2 * c + 1], sl2, neg_m));
          sum8[c & 7] += p0 + p1;
          pk[c] = pack_bf16x2(p0, p1);
        }
        l_run += ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7]));
        // The P buffer of this tile was last read by PV(g-2).
        if (g >= 2) {
          ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[g & 1], ((g - 2) >> 1) & 1, ctl));
          if (!ok) break;
        }
        {
          const uint32_t pbase = smem_u32(sP + (g & 1) * Lay::kPBytes) + row * 128;
#pragma unroll
          for (int ch = 0; ch < 16; ++ch) {
            const uint32_t addr = pbase + (ch >> 3) * Lay::kSub + (uint32_t(((ch & 7) ^ (row & 7))) << 4);
            st_shared_v4(addr, pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
          }
        }
        fence_proxy_async_smem();
        if (j > 0 && __any_sync(0xffffffffu, need)) {
          // Rescale the output accumulator once PV(g-1) has landed in it.
          ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1, ctl));
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int cb = 0; cb < D / 32; ++cb) {
            uint32_t o[32];
            const uint32_t oa = tmem + lane_off + Lay::kTmemO + cb * 32;
            tmem_ld32(oa, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(oa, o);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        mbar_arrive(&p_full[g & 1]);
      }
      if (!ok) break;
      // --------------------------------------------------------- epilogue
      const int gl = js + n - 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[gl & 1], (gl >> 1) & 1, ctl));
      if (!ok) break;
      tc_fence_after();
      const bool valid = qpos < tile.len;
      const float inv_l = 1.f / l_run;
      const size_t orow = (size_t(tile.start) + qpos) * p.hq + tile.h;
#pragma unroll
      for (int cb = 0; cb < D / 32; ++cb) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_off + Lay::kTmemO + cb * 32, o);
        tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          w[c] = pack_bf16x2(__uint_as_float(o[2 * c]) * inv_l, __uint_as_float(o[2 * c + 1]) * inv_l);
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(p.O + orow * D + cb * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
        }
      }
      if (valid)
        p.LSE[size_t(tile.h) * p.total_tokens + tile.start + qpos] = (m_run + fast_log2(l_run)) * 0.69314718055994531f;
      tc_fence_before();
      mbar_arrive(o_empty);
      js += n;
      ++tl;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::kTmemCols);
  }
}

}  // namespace lt
