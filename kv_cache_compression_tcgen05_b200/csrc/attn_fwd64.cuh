// attn_fwd64.cuh -- the head_dim 64 variant of the prefill attention (with
// per-row LSE, optionally fused with the lazy ratio), for sm_100a.
//
// Same method and work decomposition as attn_fwd_kernel (LightTransfer
// write-up, first solution of LightTransfer-Test: the FlashAttention-style
// prefill whose LSE is the lazy ratio's denominator), with a schedule that
// removes the serial chain of the aliased design.  There, P_X(j) overwrites
// the scores S_X(j), so the next scores S_X(j+1) can only be computed after
// P_X(j) V_j has read P: per key tile a query tile waits for its softmax and
// then for its own two MMA groups, one after the other.
//
// At d = 64 the tensor memory holds P in columns of its own:
//     [0,128) S of tile A, [128,256) S of tile B,
//     [256,320) P of A, [320,384) P of B, [384,448) O of A, [448,512) O of B.
// The softmax releases S_X(j) as soon as it has loaded it into registers
// (s_free), so S_X(j+1) = Q_X K_{j+1}^T runs on the tensor core while the
// softmax exponentiates S_X(j); the softmax writes P_X(j) to TMEM in chunks,
// the first once P_X(j-1) V_{j-1} has finished reading the P columns
// (pv_done).  Each query tile has its own
// MMA-issuing thread (warp 1 for tile A, warp 10 for tile B), so the
// barrier waits and commits of one tile do not delay the other's MMAs.
// The K/V ring stages and the Q buffers are released by both issuers
// (two arrivals); an issuer with no work on a stage (an item without tile B,
// or the extra last key tile of the later q-tile) waits for the stage to be
// filled and then arrives, so barrier phases never run ahead.
//
// Per issuer, per key tile j of its query tile X, in issue order:
//     S_X(j+1)  after s_free(j)   (j+1 < n_X)
//     PV_X(j)   after p_full(j)   commit pv_done; the last one commits o_full
// S_X(j+1) is issued after PV_X(j-1), so when the softmax sees S_X(j+1)
// complete, PV_X(j-1) is complete as well.
#pragma once

#include "attn_fwd.cuh"

namespace lt {

struct Attn64Layout {
  static constexpr int D = 64;
  static constexpr int kTileBytes = 128 * D * 2;      // one Q, K or V tile (16 KB)
  static constexpr int kStages = 6;                   // K/V ring slots
  static constexpr int kQOff = 0;                     // [2 buffers][2 tiles]
  static constexpr int kRingOff = kQOff + 4 * kTileBytes;
  static constexpr int kBarOff = kRingOff + kStages * kTileBytes;
  // q_full/q_empty [2+2], kv_full/kv_empty [2*kStages], s_full, s_free,
  // p_full, pv_done, o_full, o_empty [2 each], drain [2]
  static constexpr int kNumBars = 4 + 2 * kStages + 12 + 2;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 64;
  static constexpr int kAlloc = kBytes + 1024;        // room to align the base to 1024 B
  // 11 working warps (producer, two MMA issuers, eight softmax warps) and one
  // idle warp; 384 threads x 168 registers fit one CTA per SM.
  static constexpr int kThreads = 384;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kTmemP = 256;
  static constexpr uint32_t kTmemO = 384;
  static constexpr int kIssuerB = 10;                 // warp of tile B's MMA issuer
};

// Exponential pairs per 16 of a row chunk that are evaluated on the FMA pipe
// (exp2_fma) instead of MUFU: with both softmax warps of a sub-partition in
// their exponential phase, the MUFU unit is the shared limit.
constexpr int kPolyPairs = 2;

template <bool kRatio>
__global__ void __launch_bounds__(Attn64Layout::kThreads, 1)
    attn_fwd64_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const AttnParams p,
                      const __grid_constant__ AttnSchedule sched) {
  using Lay = Attn64Layout;
  constexpr int D = Lay::D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + Lay::kQOff;
  uint8_t* sRing = smem + Lay::kRingOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBarOff);
  uint64_t* q_full = bars;                       // [2 buffers]   TMA -> issuers
  uint64_t* q_empty = q_full + 2;                // [2 buffers]   issuers -> TMA (2 arrivals)
  uint64_t* kv_full = q_empty + 2;               // [kStages]     TMA -> issuers
  uint64_t* kv_empty = kv_full + Lay::kStages;   // [kStages]     issuers -> TMA (2 arrivals)
  uint64_t* s_full = kv_empty + Lay::kStages;    // [2 tiles]     MMA -> softmax
  uint64_t* s_free = s_full + 2;                 // [2 tiles]     softmax -> MMA (one arrival per warp)
  uint64_t* p_full = s_free + 2;                 // [2 tiles]     softmax -> MMA (one arrival per warp)
  uint64_t* pv_done = p_full + 2;                // [2 tiles]     MMA -> softmax (P columns free again)
  uint64_t* o_full = pv_done + 2;                // [2 tiles]     MMA -> epilogue
  uint64_t* o_empty = o_full + 2;                // [2 tiles]     epilogue -> MMA (one arrival per warp)
  uint64_t* drain = o_empty + 2;                 // [2 issuers]   MMA drain on abort
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMiscOff + 4);
  // Never raised: the drain waits after an abort end on completion or time only.
  volatile int* no_abort = reinterpret_cast<volatile int*>(smem + Lay::kMiscOff + 8);
  float* ratio_part = reinterpret_cast<float*>(smem + Lay::kMiscOff + 16);   // [2 tiles][4 warps]
  int* ratio_cnt = reinterpret_cast<int*>(smem + Lay::kMiscOff + 48);        // [2 tiles] warps done

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int grid = gridDim.x;
  const int cta = blockIdx.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 2);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
      mbar_init(&p_full[i], 4);
      mbar_init(&pv_done[i], 1);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_empty[i], 4);
      mbar_init(&drain[i], 1);
    }
    for (int i = 0; i < Lay::kStages; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 2);
    }
    *abort_flag = 0;
    *no_abort = 0;
    ratio_cnt[0] = ratio_cnt[1] = 0;
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
  // The set-up above touches no global memory: it overlaps the previous
  // kernel's tail under a programmatic launch.
  pdl_wait();
  pdl_launch_dependents();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.status};
  const WaitCtl drain_ctl{no_abort, p.status};
  if (warp == 0) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      int ring = 0, nq = 0;
      bool ok = true;
      for (int round = 0, rounds = attn_rounds(sched, p, cta, grid); ok && round < rounds; ++round) {
        const int t = attn_item(sched, round, cta, grid);
        AttnItem it;
        if (t >= p.num_items || !attn_decode(p, t, it)) continue;
        const int qb = nq & 1;
        if (nq >= 2 && !(ok = mbar_wait(&q_empty[qb], ((nq >> 1) - 1) & 1, ctl))) break;
        const int ntile = it.hasB ? 2 : 1;
        mbar_expect_tx(&q_full[qb], ntile * Lay::kTileBytes);
        for (int x = 0; x < ntile; ++x)
          tma_load_3d(sQ + (qb * 2 + x) * Lay::kTileBytes, &tmQ, &q_full[qb], 0, it.h[x],
                      it.start + it.qt[x] * 128);
        ++nq;
        // Ring order: K0, V0, K1, V1, ...
        for (int j = 0; ok && j < it.n[0]; ++j) {
          for (int kv = 0; kv < 2; ++kv) {
            const int slot = ring % Lay::kStages;
            if (ring >= Lay::kStages && !(ok = mbar_wait(&kv_empty[slot], ((ring / Lay::kStages) - 1) & 1, ctl)))
              break;
            mbar_expect_tx(&kv_full[slot], Lay::kTileBytes);
            tma_load_3d(sRing + slot * Lay::kTileBytes, kv == 0 ? &tmK : &tmV, &kv_full[slot], 0, it.kh,
                        it.start + j * 128);
            ++ring;
          }
        }
      }
      if (!ok) {
        // Let the loads already issued land before the CTA's shared memory is
        // released (bounded; the abort flag is ignored here).
        for (int x = ring > Lay::kStages ? ring - Lay::kStages : 0; x < ring; ++x)
          mbar_wait(&kv_full[x % Lay::kStages], (x / Lay::kStages) & 1, drain_ctl);
        for (int x = nq > 2 ? nq - 2 : 0; x < nq; ++x) mbar_wait(&q_full[x & 1], (x >> 1) & 1, drain_ctl);
      }
    }
  } else if (warp == 1 || warp == Lay::kIssuerB) {
    // --------------------------------------------------- MMA issuer of tile x
    if (lane == 0) {
      const int x = warp == 1 ? 0 : 1;
      constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t kIdPV = idesc_bf16_f32(128, D, 0, 1);
      // Shared-memory descriptors differ only in the start-address field
      // (address / 16): built once, advanced by byte offset / 16 per MMA.
      const uint64_t q_desc = smem_desc_sw128(smem_u32(sQ), 16, 1024) + uint64_t((x * Lay::kTileBytes) >> 4);
      const uint64_t k_desc = smem_desc_sw128(smem_u32(sRing), 16, 1024);
      const uint64_t v_desc = smem_desc_sw128(smem_u32(sRing), 16384, 1024);
      const uint32_t s_tm = tmem + x * 128;
      const uint32_t p_tm = tmem + Lay::kTmemP + x * 64;
      const uint32_t o_tm = tmem + Lay::kTmemO + x * D;
      int ring = 0, nq = 0;
      int cnt_sfree = 0, cnt_p = 0, cnt_o = 0;
      bool ok = true;
      for (int round = 0, rounds = attn_rounds(sched, p, cta, grid); ok && round < rounds; ++round) {
        const int t = attn_item(sched, round, cta, grid);
        AttnItem it;
        if (t >= p.num_items || !attn_decode(p, t, it)) continue;
        const int qb = nq & 1;
        if (!(ok = mbar_wait(&q_full[qb], (nq >> 1) & 1, ctl))) break;
        ++nq;
        const int base = ring;
        const int n = it.n[0];
        const int nx = x == 0 ? n : (it.hasB ? it.n[1] : 0);
        ring = base + 2 * n;
        auto slot_of = [&](int j, int kv) { return (base + 2 * j + kv) % Lay::kStages; };
        auto phase_of = [&](int j, int kv) { return ((base + 2 * j + kv) / Lay::kStages) & 1; };
        // S_x(j) = Q_x K_j^T; the stage of K_j is released (this issuer's share).
        auto issue_s = [&](int j) -> bool {
          const int slot = slot_of(j, 0);
          if (!mbar_wait(&kv_full[slot], phase_of(j, 0), ctl)) return false;
          tc_fence_after();
          const uint64_t qd = q_desc + uint64_t((qb * 2 * Lay::kTileBytes) >> 4);
          const uint64_t kd = k_desc + uint64_t((slot * Lay::kTileBytes) >> 4);
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off16 = ((k & 3) * 32) >> 4;
            mma_bf16_ss(s_tm, qd + off16, kd + off16, kIdS, k > 0 ? 1u : 0u);
          }
          mma_commit(&s_full[x]);
          mma_commit(&kv_empty[slot]);
          return true;
        };
        if (nx > 0) {
          ok = issue_s(0);
          for (int j = 0; ok && j < nx; ++j) {
            // The next scores, as soon as the softmax has loaded S_x(j).
            if (!(ok = mbar_wait(&s_free[x], cnt_sfree & 1, ctl))) break;
            ++cnt_sfree;
            if (j + 1 < nx && !(ok = issue_s(j + 1))) break;
            // O_x += P_x(j) V_j.
            if (!(ok = mbar_wait(&p_full[x], cnt_p & 1, ctl))) break;
            ++cnt_p;
            if (j == 0 && cnt_o > 0 && !(ok = mbar_wait(&o_empty[x], (cnt_o - 1) & 1, ctl))) break;
            const int slot = slot_of(j, 1);
            if (!(ok = mbar_wait(&kv_full[slot], phase_of(j, 1), ctl))) break;
            tc_fence_after();
            const uint64_t vd = v_desc + uint64_t((slot * Lay::kTileBytes) >> 4);
#pragma unroll
            for (int k = 0; k < 128 / 16; ++k)
              mma_bf16_ts(o_tm, p_tm + k * 8, vd + uint64_t((k * 2048) >> 4), kIdPV, (j > 0 || k > 0) ? 1u : 0u);
            mma_commit(&pv_done[x]);
            mma_commit(&kv_empty[slot]);
            if (j == nx - 1) {
              mma_commit(&o_full[x]);
              ++cnt_o;
            }
          }
          if (!ok) break;
          mma_commit(&q_empty[qb]);
        }
        // Stages of this item that the tile does not read: release this
        // issuer's share once each has been filled.
        for (int j = nx; ok && j < n; ++j)
          for (int kv = 0; kv < 2; ++kv) {
            const int slot = slot_of(j, kv);
            if (!(ok = mbar_wait(&kv_full[slot], phase_of(j, kv), ctl))) break;
            mbar_arrive(&kv_empty[slot]);
          }
        if (ok && nx == 0) mbar_arrive(&q_empty[qb]);
      }
      if (!ok) {
        mma_commit(&drain[x]);
        mbar_wait(&drain[x], 0, drain_ctl);
      }
    }
  } else if (warp >= 2 && warp < 10) {
    // --------------------------------------------------------------- softmax
    const int x = (warp - 2) >> 2;             // tile slot: 0 = A (warps 2..5), 1 = B (warps 6..9)
    const int wq = warp & 3;                   // TMEM lane quarter of this warp
    const int row = wq * 32 + lane;            // query row within the tile
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const uint32_t s_col = tmem + lane_off + x * 128;
    const uint32_t p_col = tmem + lane_off + Lay::kTmemP + x * 64;
    const uint32_t o_col = tmem + lane_off + Lay::kTmemO + x * D;
    const float sl2 = p.scale_log2;
    int cnt_s = 0, cnt_o = 0, cnt_pv = 0;
    bool ok = true;
    for (int round = 0, rounds = attn_rounds(sched, p, cta, grid); ok && round < rounds; ++round) {
      const int t = attn_item(sched, round, cta, grid);
      AttnItem it;
      if (t >= p.num_items || !attn_decode(p, t, it)) continue;
      if (x == 1 && !it.hasB) continue;
      const int qt = x ? it.qt[1] : it.qt[0];   // selects, not a local-memory index
      const int n = x ? it.n[1] : it.n[0];
      const int h = x ? it.h[1] : it.h[0];
      const int qpos = qt * 128 + row;
      // Fused ratio: is this row one of the last n_obs rows of its sequence?
      int n_obs_seq = 0, obs_lo = 0;
      bool tile_obs = false, row_obs = false;
      if constexpr (kRatio) {
        n_obs_seq = min(p.n_obs, it.len);
        obs_lo = it.len - n_obs_seq;
        tile_obs = qt * 128 + 127 >= obs_lo && qt * 128 < it.len;
        row_obs = tile_obs && qpos >= obs_lo && qpos < it.len;
      }
      // The tile loop and epilogue in two copies: items holding observed rows
      // run the one with the ratio steps, all others the plain kernel's code.
      const auto run_item = [&](auto obs) {
        constexpr bool kObs = decltype(obs)::value;
        float m_run = -INFINITY;   // running max of scale*log2(e)*s, possibly stale by < 8
        float l_run = 0.f;         // running sum of exp2(.. - m_run)
        float num = 0.f;           // fused ratio numerator, same frame as l_run
        for (int j = 0; j < n; ++j) {
          ok = __all_sync(0xffffffffu, mbar_wait(&s_full[x], cnt_s & 1, ctl));
          if (!ok) break;
          ++cnt_s;
          tc_fence_after();
          const bool diag = j == qt;
          uint32_t sr[128];
          {
            uint32_t(&c0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
            uint32_t(&c1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
            uint32_t(&c2)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[64]);
            uint32_t(&c3)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[96]);
            tmem_ld32(s_col + 0, c0);
            tmem_ld32(s_col + 32, c1);
            tmem_ld32(s_col + 64, c2);
            tmem_ld32(s_col + 96, c3);
            tmem_wait_ld();
          }
          if (diag) {
#pragma unroll
            for (int c = 0; c < 128; ++c)
              if (c > row) sr[c] = __float_as_uint(-INFINITY);
          }
          // Row maximum: 8 independent chains of three-input max.
          float mx8[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) mx8[k] = fmaxf(__uint_as_float(sr[k]), __uint_as_float(sr[8 + k]));
#pragma unroll
          for (int c = 16; c < 128; c += 16)
#pragma unroll
            for (int k = 0; k < 8; ++k) mx8[k] = fmax3(mx8[k], __uint_as_float(sr[c + k]), __uint_as_float(sr[c + 8 + k]));
          const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
          const float m_new = fmaxf(m_run, mx * sl2);
          const bool need = m_new > m_run + 8.f;
          float alpha = 1.f;
          if (need) {
            alpha = fast_exp2(m_run - m_new);
            m_run = m_new;
          }
          l_run *= alpha;
          if constexpr (kObs) num *= alpha;
          // S_x(j) is in registers: its columns may take S_x(j+1).
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s_free[x]);
          const float neg_m = -m_run;
          // Fused ratio: the weights of the keys in K_i = [0, min(S, i+1)) U
          // [max(S, i-W+1), i] within this key tile (columns c = key - 128 j).
          // Keys after i carry weight 0 (causal mask), so a tile that starts
          // inside the window counts whole (added below, from the tile's row
          // sum); only the tile holding the window's first key and the tile
          // holding the sinks need a per-key mask, summed in fp32 from the
          // scores before P is built.  Items with no observed row (tile_obs false,
          // the same in every thread of the tile) skip all of it, the vote
          // included.
          bool whole = false;
          if constexpr (kObs) {
            {
              const int win_c = qpos - p.W + 1 - j * 128;   // first window column
              const int sink_c = p.S - j * 128;              // columns below it are sinks
              whole = row_obs && win_c <= 0;
              const bool part = row_obs && !whole && (win_c < 128 || sink_c > 0);
              if (__any_sync(0xffffffffu, part)) {
                // All 128 columns, masked by value: at head_dim 64 this measured
                // faster than masked_score_sum's column-skipping branches.
                float acc = 0.f;
#pragma unroll
                for (int c = 0; c < 128; ++c) {
                  const float w = fast_exp2(fmaf(__uint_as_float(sr[c]), sl2, neg_m));
                  acc += (c < sink_c || c >= win_c) ? w : 0.f;
                }
                if (part) num += acc;
              }
            }
          }
          // P_x(j) in four 32-column chunks of bf16 pairs; the first two are
          // held in registers and written with the third.  Before the first
          // write, P_x(j-1) V_{j-1} must be done with the P columns (and with O,
          // before a rescale): within an item that is one phase of pv_done per
          // key tile; the first tile follows the previous item's epilogue,
          // which consumed the last PV's phase.  Waiting two chunks in gives
          // that PV time to finish.
          float2 sum4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
          const float2 sl2x2 = make_float2(sl2, sl2), neg_mx2 = make_float2(neg_m, neg_m);
          uint32_t pk0[16], pk1[16];
#pragma unroll
          for (int cb = 0; cb < 4; ++cb) {
            uint32_t pk[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const int c0 = cb * 32 + 2 * c;
              const float2 xx = fma_f32x2(make_float2(__uint_as_float(sr[c0]), __uint_as_float(sr[c0 + 1])), sl2x2,
                                          neg_mx2);
              // kPolyPairs of every 16 pairs go to the FMA pipe, the rest to MUFU.
              const bool poly = (c & 15) >= 16 - kPolyPairs;
              const float p0 = poly ? exp2_fma(xx.x) : fast_exp2(xx.x);
              const float p1 = poly ? exp2_fma(xx.y) : fast_exp2(xx.y);
              sum4[c & 3] = add_f32x2(sum4[c & 3], make_float2(p0, p1));
              pk[c] = pack_bf16x2(p0, p1);
            }
            if (cb == 2 && j > 0) {
              ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[x], cnt_pv & 1, ctl));
              ++cnt_pv;
              tc_fence_after();
            }
            if (cb == 0) {
#pragma unroll
              for (int c = 0; c < 16; ++c) pk0[c] = pk[c];
            } else if (cb == 1) {
#pragma unroll
              for (int c = 0; c < 16; ++c) pk1[c] = pk[c];
            } else {
              if (cb == 2) {
                tmem_st16(p_col, pk0);
                tmem_st16(p_col + 16, pk1);
              }
              tmem_st16(p_col + cb * 16, pk);
            }
          }
          if (!ok) break;
          const float2 s01 = add_f32x2(sum4[0], sum4[1]), s23 = add_f32x2(sum4[2], sum4[3]);
          const float2 s0123 = add_f32x2(s01, s23);
          const float tile_sum = s0123.x + s0123.y;
          l_run += tile_sum;
          if constexpr (kObs) {
            if (whole) num += tile_sum;
          }
          if (j > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll
            for (int cb = 0; cb < D / 32; ++cb) {
              uint32_t o[32];
              tmem_ld32(o_col + cb * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
              tmem_st32(o_col + cb * 32, o);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_full[x]);
        }
        if (!ok) return;
        // --------------------------------------------------------- epilogue
        ok = __all_sync(0xffffffffu, mbar_wait(&o_full[x], cnt_o & 1, ctl));
        if (!ok) return;
        ++cnt_o;
        // The last PV's pv_done phase (complete by now): consumed so that every
        // wait on the barrier follows the completion of the phase before it.
        ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[x], cnt_pv & 1, ctl));
        if (!ok) return;
        ++cnt_pv;
        tc_fence_after();
        const bool valid = qpos < it.len;
        const float inv_l = 1.f / l_run;
        const size_t orow = (size_t(it.start) + qpos) * p.hq + h;
#pragma unroll
        for (int cb = 0; cb < D / 32; ++cb) {
          uint32_t o[32];
          tmem_ld32(o_col + cb * 32, o);
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
          p.LSE[size_t(h) * p.total_tokens + it.start + qpos] = (m_run + fast_log2(l_run)) * 0.69314718055994531f;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&o_empty[x]);
        if constexpr (kObs) {
          {
            // This tile's share of mean_i r_i: its rows added in a fixed order.
            float r = row_obs ? num * inv_l : 0.f;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) r += __shfl_xor_sync(0xffffffffu, r, off);
            // No barrier (a sibling warp may have left on a timed-out wait): the
            // fourth warp to finish adds the four partials in warp order.
            if (lane == 0) {
              ratio_part[x * 4 + wq] = r;
              __threadfence_block();
              if (atomicAdd(&ratio_cnt[x], 1) == 3) {
                __threadfence_block();
                const volatile float* part = ratio_part + x * 4;
                const float tot = (part[0] + part[1]) + (part[2] + part[3]);
                atomicAdd(p.ratio + size_t(it.b) * p.hq + h, tot / float(n_obs_seq));
                ratio_cnt[x] = 0;
              }
            }
          }
        }
      };
      if (tile_obs)
        run_item(BoolTag<true>{});
      else
        run_item(BoolTag<false>{});
      if (!ok) break;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::kTmemCols);
  }
  if constexpr (kRatio) {
    // Fused queue push: the last CTA to finish pushes every sequence's score.
    if (p.dq_state)
      dq_last_cta_push(p.dq_state, p.dq_L, p.batch, p.dq_layer, p.ratio, p.hq, *abort_flag != 0,
                       reinterpret_cast<int*>(smem + Lay::kMiscOff + 56));
  }
}

}  // namespace lt
