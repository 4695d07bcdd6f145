// attn_fwd.cuh -- causal GQA prefill attention with per-row LSE (optionally
// fused with the lazy ratio) for sm_100a.
//
// The LightTransfer write-up (xzbcqc.com news page, first solution of
// LightTransfer-Test) reuses the log-sum-exp that a FlashAttention-style prefill
// produces as the denominator of the lazy ratio.  This kernel is that prefill,
// built for B200 (the library runs it at head_dim 128; head_dim 64 runs the
// variant in attn_fwd64.cuh, whose P has TMEM columns of its own):
//
//   * persistent: one CTA per SM walks a list of work items.  A work item is
//     two 128-row query tiles that read the same K/V stream: two query heads
//     of one KV head at the same q-tile when the GQA group is even, otherwise
//     two consecutive q-tiles of one head (the earlier tile then skips the last
//     key tile).  The order (attn_decode): heaviest q-tile first; for a long
//     single sequence and for packed batches, sequence by sequence and in
//     q-tile bands KV head by KV head (concurrent CTAs share one KV head's K/V
//     in L2); CTAs take items in a snake order, or, for a short single
//     sequence, as a longest-first assignment computed on the host (the
//     AttnSchedule parameter).
//   * warp-specialised, three warpgroups (12 warps, 10 working); setmaxnreg
//     gives the softmax warpgroups 184 registers a thread and the third 136:
//       warps 0..3  softmax of tile A, warps 4..7 softmax of tile B: thread =
//                   query row = TMEM lane.  tcgen05.ld of the 128 scores, causal
//                   mask on the diagonal tile, running max in the log2 domain
//                   (the O accumulator is rescaled only when the max grows by
//                   more than 2^8; exact, because O and l share the stale max),
//                   exp2 with the scale/shift and row sum in packed two-lane
//                   fp32, bf16 P written back over the scores in TMEM with
//                   tcgen05.st (P is the A operand of O += P V, read from TMEM);
//                   epilogue O / l and LSE = (m + log2 l) ln 2, written once;
//       warp 8      TMA producer: the item's two Q tiles (double buffered) and
//                   a ring of K/V tiles (128 keys x d, 128-byte swizzle);
//       warp 9      owns the TMEM allocation; one thread issues every
//                   tcgen05.mma in the order
//                       S_A(0), S_B(0), [PV_A(j), S_A(j+1), PV_B(j), S_B(j+1)]
//                   so the tensor core works on one tile while the other
//                   tile's softmax runs (shared-memory descriptors are built
//                   once and advanced by address/16, so the single issuing
//                   thread spends little per instruction).
//   * TMEM columns: [0,128) S/P of A, [128,256) S/P of B, [256,256+d) O of A,
//     [256+d, 256+2d) O of B.  P overwrites the first half of its S columns.
//     The MMAs of one thread execute in issue order, so S_X(j+1), issued after
//     PV_X(j), never overwrites P_X(j) before PV_X(j) has read it, and once
//     S_X(j+1) is complete so is PV_X(j): the softmax may rescale O_X as soon
//     as it sees S_X(j+1).
//
// Fused lazy ratio (press-release page, "LightTransfer方法详解": attention
// weights from the query to the initial and the recent keys): for the last
// n_obs rows of each sequence the softmax threads also sum, in the same
// stale-max frame as l, the weights of the keys
//     K_i = [0, min(S, i+1)) U [max(S, i-W+1), i],
// so r_i = num_i / l_i = sum_{j in K_i} exp(s_ij - LSE_i).  The rows of a tile
// are added in a fixed order (lanes, then the tile's four warps) and one
// atomic add per (tile, head) puts the tile's share of the mean into
// ratio[b, h]; with n_obs <= 128 at most two tiles touch a (b, h), and a
// two-term sum does not depend on the order.
#pragma once

#include "dqueue.cuh"
#include "lt_device.cuh"

namespace lt {

struct AttnParams {
  int batch;
  int total_tokens;
  int hq;
  int hkv;
  int group;        // hq / hkv
  int n_qtiles;     // ceil(max_seqlen / 128)
  int pair_heads;   // 1: an item pairs two heads; 0: it pairs two q-tiles
  int qt_band;      // > 0 (with pair_heads): items ordered by sequence, then q-tile bands of this many tiles, KV head by KV head
  int num_items;
  const int32_t* cu_seqlens;  // device [batch+1] or null (one sequence)
  __nv_bfloat16* O;
  float* LSE;
  float scale_log2;  // softmax scale * log2(e)
  unsigned* status;
  // fused lazy ratio
  float* ratio;      // [batch, hq], zeroed before the launch
  int S;
  int W;
  int n_obs;
  // fused device-queue push (null: none): after every CTA has added its
  // ratios, the last one pushes layer dq_layer's scores into the queue state
  void* dq_state;
  int dq_L;
  int dq_layer;
};

template <int D>
struct AttnLayout {
  static constexpr int kTileBytes = 128 * D * 2;      // one Q, K or V tile
  static constexpr int kSub = 16384;                  // one 128 x 64 bf16 swizzled sub-tile
  static constexpr int kStages = D == 64 ? 6 : 3;     // K/V ring slots
  static constexpr int kQOff = 0;                     // [2 buffers][2 tiles]
  static constexpr int kRingOff = kQOff + 4 * kTileBytes;
  static constexpr int kBarOff = kRingOff + kStages * kTileBytes;
  static constexpr int kNumBars = 2 + 2 + 2 * kStages + 2 + 2 + 2 + 2 + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 64;
  static constexpr int kAlloc = kBytes + 1024;        // room to align the base to 1024 B
  // Three warpgroups: softmax of tile A (warps 0..3) and of tile B (4..7),
  // and a third holding the TMA producer (warp 8), the TMEM owner / MMA
  // issuer (warp 9) and two idle warps.  Launched at 168 registers a thread
  // (one CTA per SM); setmaxnreg then moves registers from the third
  // warpgroup to the softmax ones.
  static constexpr int kThreads = 384;
  static constexpr int kLaunchRegs = 168;
  static constexpr int kRegsSoftmax = 184;
  static constexpr int kRegsOther = 3 * kLaunchRegs - 2 * kRegsSoftmax;   // 136
  static constexpr int kWarpProducer = 8;
  static constexpr int kWarpMma = 9;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kTmemO = 256;
};

// Compile-time flag passed to generic lambdas (selects one of two copies of a body).
template <bool B>
struct BoolTag {
  static constexpr bool value = B;
};

struct AttnItem {
  int b, kh, start, len;
  int h[2], qt[2], n[2];
  bool hasB;
};

// Fused ratio's masked sum of one key tile, in fp32 from the tile's scores
// (scores sr, scale sl2 and shift neg_m as the exponential loop uses them):
// the weights of the sink columns c < sink_c (the same for every row of the
// tile) and of the window columns c >= max(win_c, sink_c), for threads whose
// `part` is set (0 for the others).  Only those columns are exponentiated:
// columns below sink_c and from the smallest first window column of the
// warp's rows on (both bounds warp-uniform: each column's test is a uniform
// branch, and the unrolled loop indexes the scores with constants).  The
// whole warp calls it.
__device__ __forceinline__ float masked_score_sum(const uint32_t (&sr)[128], float sl2, float neg_m, int sink_c,
                                                  int win_c, bool part) {
  float acc = 0.f;
  const int w0 = max(win_c, sink_c);
  const int lo = int(__reduce_min_sync(0xffffffffu, unsigned(part ? max(w0, 0) : 128)));
#pragma unroll
  for (int c = 0; c < 128; ++c) {
    if (c < sink_c || c >= lo) {   // warp-uniform: sink_c and lo are the same in every lane
      const float w = fast_exp2(fmaf(__uint_as_float(sr[c]), sl2, neg_m));
      acc += (c < sink_c || c >= w0) ? w : 0.f;
    }
  }
  return part ? acc : 0.f;
}

__device__ __forceinline__ void seq_bounds(const AttnParams& p, int b, int& start, int& len) {
  if (p.cu_seqlens) {
    start = p.cu_seqlens[b];
    len = p.cu_seqlens[b + 1] - start;
  } else {
    start = 0;
    len = p.total_tokens;
  }
}

// Work item t -> its one or two tiles; false when the item has no valid tile.
// Items are ordered heaviest first; the items of one q position are consecutive
// (heads of a sequence next to each other, so concurrent CTAs share K/V in L2).
__device__ __forceinline__ bool attn_decode(const AttnParams& p, int t, AttnItem& it) {
  if (p.pair_heads && p.qt_band > 0) {
    // Banded order: sequence by sequence (a packed batch), q-tiles in bands of
    // qt_band (heaviest band first), and within a band one KV head after
    // another, so the CTAs running at the same time stream the same KV head's
    // K/V (which then stays in L2) instead of every KV head's (and every
    // sequence's) at once.  A long single sequence takes bands of about one
    // wave of the grid, a packed batch one band per sequence.
    const int ppk = p.group >> 1;                       // head pairs per KV head
    const int per_kh = p.qt_band * ppk;
    const int per_band = per_kh * p.hkv;
    const int per_seq = ((p.n_qtiles + p.qt_band - 1) / p.qt_band) * per_band;
    it.b = t / per_seq;
    int rem = t - it.b * per_seq;
    const int band = rem / per_band;
    rem -= band * per_band;
    const int kh = rem / per_kh;
    rem -= kh * per_kh;
    const int qin = rem / ppk;
    const int hp = kh * ppk + (rem - qin * ppk);
    const int qt = p.n_qtiles - 1 - (band * p.qt_band + qin);
    if (qt < 0) return false;                           // the last band's unused places
    seq_bounds(p, it.b, it.start, it.len);
    it.h[0] = 2 * hp;
    it.h[1] = 2 * hp + 1;
    it.qt[0] = it.qt[1] = qt;
    it.n[0] = it.n[1] = qt + 1;
    it.hasB = true;
    it.kh = it.h[0] / p.group;
    return qt * 128 < it.len;
  }
  if (p.pair_heads) {
    const int hp_count = p.hq >> 1;
    const int per_q = p.batch * hp_count;
    const int qt = p.n_qtiles - 1 - t / per_q;
    const int rem = t - (t / per_q) * per_q;
    it.b = rem / hp_count;
    const int hp = rem - it.b * hp_count;
    seq_bounds(p, it.b, it.start, it.len);
    it.h[0] = 2 * hp;
    it.h[1] = 2 * hp + 1;
    it.qt[0] = it.qt[1] = qt;
    it.n[0] = it.n[1] = qt + 1;
    it.hasB = true;
    it.kh = it.h[0] / p.group;
    return qt * 128 < it.len;
  }
  const int per_q = p.batch * p.hq;
  const int npairs = (p.n_qtiles + 1) >> 1;
  const int qp = npairs - 1 - t / per_q;
  const int rem = t - (t / per_q) * per_q;
  it.b = rem / p.hq;
  const int h = rem - it.b * p.hq;
  seq_bounds(p, it.b, it.start, it.len);
  it.h[0] = it.h[1] = h;
  it.kh = h / p.group;
  const int t1 = 2 * qp + 1, t0 = 2 * qp;
  if (t1 * 128 < it.len) {
    it.qt[0] = t1;
    it.qt[1] = t0;
    it.n[0] = t1 + 1;
    it.n[1] = t0 + 1;
    it.hasB = true;
    return true;
  }
  it.qt[0] = it.qt[1] = t0;
  it.n[0] = it.n[1] = t0 + 1;
  it.hasB = false;
  return t0 * 128 < it.len;
}

// Snake order: CTA c takes item k*G + c on even rounds and k*G + (G-1-c) on odd
// rounds, so the heaviest items are spread evenly.
__device__ __forceinline__ int attn_item_index(int round, int cta, int grid) {
  return round * grid + ((round & 1) ? (grid - 1 - cta) : cta);
}

// A static assignment of work items to CTAs, computed on the host for small
// launches (a few items per CTA, where the snake order cannot balance the
// heaviest items, and the fused ratio's extra work on the items holding the
// observed rows would add to the slowest CTA): CTA c runs items
// item[off[c] .. off[c+1]) in that order.  Passed as a kernel parameter.
constexpr int kSchedMaxItems = 1536;
constexpr int kSchedMaxCtas = 160;
struct AttnSchedule {
  int used;                            // 0: the snake order over all items
  uint16_t off[kSchedMaxCtas + 1];
  uint16_t item[kSchedMaxItems];
};

__device__ __forceinline__ int attn_rounds(const AttnSchedule& s, const AttnParams& p, int cta, int grid) {
  return s.used ? int(s.off[cta + 1]) - int(s.off[cta]) : (p.num_items + grid - 1) / grid;
}
__device__ __forceinline__ int attn_item(const AttnSchedule& s, int round, int cta, int grid) {
  return s.used ? int(s.item[s.off[cta] + round]) : attn_item_index(round, cta, grid);
}

template <int D, bool kRatio>
__global__ void __launch_bounds__(AttnLayout<D>::kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const AttnParams p,
                    const __grid_constant__ AttnSchedule sched) {
  using Lay = AttnLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + Lay::kQOff;
  uint8_t* sRing = smem + Lay::kRingOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBarOff);
  uint64_t* q_full = bars;                       // [2 buffers]   TMA -> MMA
  uint64_t* q_empty = q_full + 2;                // [2 buffers]   MMA -> TMA
  uint64_t* kv_full = q_empty + 2;               // [kStages]
  uint64_t* kv_empty = kv_full + Lay::kStages;   // [kStages]
  uint64_t* s_full = kv_empty + Lay::kStages;    // [2 tiles]     MMA -> softmax
  uint64_t* p_full = s_full + 2;                 // [2 tiles]     softmax -> MMA (128 arrivals)
  uint64_t* o_full = p_full + 2;                 // [2 tiles]     MMA -> epilogue
  uint64_t* o_empty = o_full + 2;                // [2 tiles]     epilogue -> MMA (128 arrivals)
  uint64_t* drain = o_empty + 2;                 // [1]           MMA drain on abort
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
  constexpr int kWarpProducer = Lay::kWarpProducer, kWarpMma = Lay::kWarpMma;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_empty[i], 128);
    }
    mbar_init(drain, 1);
    for (int i = 0; i < Lay::kStages; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    *abort_flag = 0;
    *no_abort = 0;
    ratio_cnt[0] = ratio_cnt[1] = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == kWarpMma) {
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
  // Role dispatch by warpgroup: setmaxnreg is executed by all four warps of
  // a warpgroup at the start of its branch, so each branch is compiled under
  // its own register limit.  2 * kRegsSoftmax + kRegsOther = 3 * the
  // launch's 168 registers a thread (checked on the host against the
  // compiled kernel before any launch).
  if (warp >= 8) {
    regs_decrease<Lay::kRegsOther>();
    if (warp == kWarpProducer) {
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
            for (int st = 0; st < D / 64; ++st)
              tma_load_3d(sQ + (qb * 2 + x) * Lay::kTileBytes + st * Lay::kSub, &tmQ, &q_full[qb], st * 64, it.h[x],
                          it.start + it.qt[x] * 128);
          ++nq;
          // Ring order: K0, V0, K1, V1, ...
          for (int j = 0; ok && j < it.n[0]; ++j) {
            for (int kv = 0; kv < 2; ++kv) {
              const int slot = ring % Lay::kStages;
              if (ring >= Lay::kStages && !(ok = mbar_wait(&kv_empty[slot], ((ring / Lay::kStages) - 1) & 1, ctl)))
                break;
              mbar_expect_tx(&kv_full[slot], Lay::kTileBytes);
              for (int st = 0; st < D / 64; ++st)
                tma_load_3d(sRing + slot * Lay::kTileBytes + st * Lay::kSub, kv == 0 ? &tmK : &tmV, &kv_full[slot],
                            st * 64, it.kh, it.start + j * 128);
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
    } else if (warp == kWarpMma) {
      // ------------------------------------------------------------------- MMA
      if (lane == 0) {
        constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, 0, 0);
        constexpr uint32_t kIdPV = idesc_bf16_f32(128, D, 0, 1);
        // Shared-memory descriptors differ only in the start-address field
        // (address / 16, 14 bits; the shared window is below 256 KB): built once,
        // advanced by byte offset / 16 per MMA.
        const uint64_t q_desc = smem_desc_sw128(smem_u32(sQ), 16, 1024);
        const uint64_t k_desc = smem_desc_sw128(smem_u32(sRing), 16, 1024);
        const uint64_t v_desc = smem_desc_sw128(smem_u32(sRing), Lay::kSub, 1024);
        int ring = 0, nq = 0;
        int cnt_p0 = 0, cnt_p1 = 0;   // P tiles consumed, per tile slot
        int cnt_o0 = 0, cnt_o1 = 0;   // items finished, per tile slot
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
          const int nB = it.hasB ? it.n[1] : 0;
          ring = base + 2 * n;
          auto slot_of = [&](int j, int kv) { return (base + 2 * j + kv) % Lay::kStages; };
          auto phase_of = [&](int j, int kv) { return ((base + 2 * j + kv) / Lay::kStages) & 1; };
          // S_x(j) = Q_x K_j^T into the tile's TMEM score columns.
          auto issue_s = [&](int x, int j) -> bool {
            const int slot = slot_of(j, 0);
            if (x == 0) {   // tile A always uses K_j first
              if (!mbar_wait(&kv_full[slot], phase_of(j, 0), ctl)) return false;
            }
            tc_fence_after();
            const uint64_t qd = q_desc + uint64_t(((qb * 2 + x) * Lay::kTileBytes) >> 4);
            const uint64_t kd = k_desc + uint64_t((slot * Lay::kTileBytes) >> 4);
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
              const uint32_t off16 = ((k >> 2) * Lay::kSub + (k & 3) * 32) >> 4;
              mma_bf16_ss(tmem + x * 128, qd + off16, kd + off16, kIdS, k > 0 ? 1u : 0u);
            }
            mma_commit(&s_full[x]);
            const bool last_use = x == 1 || j >= nB;
            if (last_use) mma_commit(&kv_empty[slot]);
            if (last_use && j == n - 1) mma_commit(&q_empty[qb]);
            return true;
          };
          // O_x += P_x(j) V_j, P_x(j) read from TMEM.
          auto issue_pv = [&](int x, int j) -> bool {
            int& cnt_p = x ? cnt_p1 : cnt_p0;
            int& cnt_o = x ? cnt_o1 : cnt_o0;
            if (!mbar_wait(&p_full[x], cnt_p & 1, ctl)) return false;
            ++cnt_p;
            if (j == 0 && cnt_o > 0 && !mbar_wait(&o_empty[x], (cnt_o - 1) & 1, ctl)) return false;
            const int slot = slot_of(j, 1);
            if (x == 0 && !mbar_wait(&kv_full[slot], phase_of(j, 1), ctl)) return false;
            tc_fence_after();
            const uint64_t vd = v_desc + uint64_t((slot * Lay::kTileBytes) >> 4);
            const uint32_t o_tmem = tmem + Lay::kTmemO + x * D;
#pragma unroll
            for (int k = 0; k < 128 / 16; ++k)
              mma_bf16_ts(o_tmem, tmem + x * 128 + k * 8, vd + uint64_t((k * 2048) >> 4), kIdPV,
                          (j > 0 || k > 0) ? 1u : 0u);
            const bool last_use = x == 1 || j >= nB;
            if (last_use) mma_commit(&kv_empty[slot]);
            if ((x == 0 && j == n - 1) || (x == 1 && j == nB - 1)) {
              mma_commit(&o_full[x]);
              ++cnt_o;
            }
            return true;
          };

          ok = issue_s(0, 0) && (nB == 0 || issue_s(1, 0));
          for (int j = 0; ok && j < n; ++j) {
            ok = issue_pv(0, j) && (j + 1 >= n || issue_s(0, j + 1));
            if (ok && j < nB) ok = issue_pv(1, j) && (j + 1 >= nB || issue_s(1, j + 1));
          }
        }
        if (!ok) {
          mma_commit(drain);
          mbar_wait(drain, 0, drain_ctl);
        }
      }
    }
  } else {
    regs_increase<Lay::kRegsSoftmax>();
    // --------------------------------------------------------------- softmax
    const int x = warp >> 2;                   // tile slot: 0 = A (warps 0..3), 1 = B (warps 4..7)
    const int wq = warp & 3;                   // TMEM lane quarter of this warp
    const int row = wq * 32 + lane;            // query row within the tile
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const uint32_t s_col = tmem + lane_off + x * 128;
    const uint32_t o_col = tmem + lane_off + Lay::kTmemO + x * D;
    const float sl2 = p.scale_log2;
    int cnt_s = 0, cnt_o = 0;
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
          // All 128 scores of the row in one batch of TMEM loads (a single
          // wait: the load latency is paid once per tile).
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
          // Columns 0..15 seed the chains; c = 16, 32, ..., 112 covers 16..127.
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
          const float neg_m = -m_run;
          // Fused ratio: the weights of the keys in K_i = [0, min(S, i+1)) U
          // [max(S, i-W+1), i] within this key tile (columns c = key - 128 j).
          // Keys after i carry weight 0 (causal mask), so a tile that starts
          // inside the window counts whole (its row sum, below); only the tile
          // holding the window's first key and the tile holding the sinks need
          // a per-key mask, summed in fp32 from the scores before P is built
          // (masked_score_sum exponentiates only the columns that count).
          // Items with no observed row (tile_obs false, the same in every
          // thread of the tile) skip all of it, the vote included.
          bool whole = false;
          if constexpr (kObs) {
            {
              const int win_c = qpos - p.W + 1 - j * 128;   // first window column
              const int sink_c = p.S - j * 128;              // columns below it are sinks
              whole = row_obs && win_c <= 0;
              const bool part = row_obs && !whole && (win_c < 128 || sink_c > 0);
              if (__any_sync(0xffffffffu, part)) num += masked_score_sum(sr, sl2, neg_m, sink_c, win_c, part);
            }
          }
          // exp2 in 32-column chunks; each chunk's bf16 P goes to TMEM (16
          // columns) as soon as it is packed.
          // The scale/shift and the row sum use the packed two-lane fp32
          // instructions (one issue slot per pair of columns).
          float2 sum4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
          const float2 sl2x2 = make_float2(sl2, sl2), neg_mx2 = make_float2(neg_m, neg_m);
#pragma unroll
          for (int cb = 0; cb < 4; ++cb) {
            uint32_t pk[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const int c0 = cb * 32 + 2 * c;
              const float2 xx = fma_f32x2(make_float2(__uint_as_float(sr[c0]), __uint_as_float(sr[c0 + 1])), sl2x2,
                                          neg_mx2);
              const float p0 = fast_exp2(xx.x);
              const float p1 = fast_exp2(xx.y);
              sum4[c & 3] = add_f32x2(sum4[c & 3], make_float2(p0, p1));
              pk[c] = pack_bf16x2(p0, p1);
            }
            tmem_st16(s_col + cb * 16, pk);
          }
          const float2 s01 = add_f32x2(sum4[0], sum4[1]), s23 = add_f32x2(sum4[2], sum4[3]);
          const float2 s0123 = add_f32x2(s01, s23);
          const float tile_sum = s0123.x + s0123.y;
          l_run += tile_sum;
          if constexpr (kObs) {
            if (whole) num += tile_sum;
          }
          if (j > 0 && __any_sync(0xffffffffu, need)) {
            // PV(j-1) is complete (S(j) was issued after it by the same thread):
            // rescale O in TMEM before PV(j) accumulates onto it.
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
          mbar_arrive(&p_full[x]);
        }
        if (!ok) return;
        // --------------------------------------------------------- epilogue
        ok = __all_sync(0xffffffffu, mbar_wait(&o_full[x], cnt_o & 1, ctl));
        if (!ok) return;
        ++cnt_o;
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
        mbar_arrive(&o_empty[x]);
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
  if (warp == kWarpMma) {
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
