/*
 * lt.h -- C ABI of the LightTransfer-Test prefill hot path on B200 (sm_100a).
 *
 * LightTransfer-Test converts "lazy" layers of a dense transformer to streaming
 * attention on the fly, from the prefill alone.  The path has four steps:
 *
 *   1. lt_prefill_attn  causal GQA prefill attention that also writes the per-row
 *                       log-sum-exp (LSE) of the attention logits;
 *   2. lt_lazy_ratio    the lazy ratio of each (sequence, query head), computed
 *                       with that LSE as its denominator so that only the S sink
 *                       and W recent keys of each observed query are visited;
 *   3. lt_select_layers / lt_queue_*  the layer priority queue that demotes the
 *                       layer with the highest ratio once more than the allowed
 *                       number of full-KV layers are queued;
 *   4. lt_compact_kv    the gather that keeps a demoted layer's sink and recent
 *                       rows as its streaming KV cache.
 *
 * Sources (the LightTransfer pages):
 *   - LightTransfer write-up (xzbcqc.com news page), the two problems of
 *     LightTransfer-Test and their solutions: FlashAttention does not store the
 *     attention weights, so the LSE it produces is used as the ratio's
 *     denominator and the numerator costs O(1) per query instead of O(seq_len);
 *     a priority queue keyed by lazy ratio keeps the prefill's peak memory at
 *     most 50% full KV + 50% streaming KV.
 *   - Press-release page "LLM突破：推理加速，长CoT生成惊艳", section
 *     "LightTransfer方法详解": the lazy ratio is the sum of the attention weights
 *     from the query to the initial and the recent keys.
 *   - LightTransfer project page, Methodology / LightTransfer-Test, Figure 2
 *     caption: after each layer the ratio and layer index enter the queue; once
 *     it is full the layer with the highest ratio is made lazy and its KV cache
 *     reduced, freeing memory for the current layer.
 *
 * Conventions for every call:
 *   - Tensor pointers marked "device" are caller-owned CUDA device memory; the
 *     library never allocates, frees or keeps them.  Tensors are row-major and
 *     contiguous; bf16 tensors are passed as void*; every device pointer must be
 *     16-byte aligned.  When total_tokens is 0 the token-indexed inputs and
 *     outputs (Q, K, V, O, LSE) are not accessed and may be null.
 *   - Calls that take a stream only enqueue work on it (they never synchronise
 *     the device); their outputs are ready when the stream reaches them.  Most
 *     kernels are launched with programmatic dependent launch: one may start
 *     while the kernel before it in the stream is finishing, and waits for that
 *     kernel's completion (all its writes visible) before it touches memory, so
 *     to the caller this is ordinary stream order.  They
 *     launch on the calling thread's current CUDA device: the stream and every
 *     device pointer must belong to that device (the library cannot check a
 *     pointer's device; the Python binding checks its tensors').
 *   - Arguments are checked before anything is enqueued.  A failed check returns
 *     LT_ERR_INVALID_ARG (or LT_ERR_UNSUPPORTED for a head_dim other than 64 or
 *     128) and enqueues nothing.  A launch failure returns LT_ERR_CUDA.
 *   - Kernels never wait unboundedly: a wait that exceeds its limit sets a
 *     device status word and the kernel returns early; lt_device_status reports
 *     it as LT_ERR_TIMEOUT.
 */
#ifndef LT_H_
#define LT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LT_OK = 0,
  LT_ERR_INVALID_ARG = 1, /* a pointer, size or layout is invalid */
  LT_ERR_UNSUPPORTED = 2, /* valid but not implemented (head_dim not 64/128) */
  LT_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
  LT_ERR_TIMEOUT = 4      /* a kernel gave up a bounded wait (see lt_device_status) */
} lt_status;

/* A cudaStream_t (the runtime's stream handle); NULL is the legacy default stream. */
typedef struct CUstream_st* lt_stream;

/*
 * Shape of one packed prefill batch.
 *   batch        number of sequences (>= 1)
 *   total_tokens T = sum of the sequence lengths (>= 0)
 *   max_seqlen   the longest sequence length; every sequence must be at most
 *                this long (tiles beyond it are never scheduled)
 *   hq, hkv      query heads and key/value heads; hq % hkv == 0, query head h
 *                reads KV head h / (hq / hkv)
 *   head_dim     d, 64 or 128
 *   cu_seqlens   device int32 [batch + 1]: sequence b is tokens
 *                [cu_seqlens[b], cu_seqlens[b+1]); NULL means batch == 1 and one
 *                sequence of total_tokens tokens.
 */
typedef struct {
  int batch;
  int total_tokens;
  int max_seqlen;
  int hq;
  int hkv;
  int head_dim;
  const int32_t* cu_seqlens;
} lt_shape;

/*
 * Causal GQA prefill attention with the per-row LSE.
 *   For sequence b, query row i (position inside b), query head h, KV head
 *   kh = h / (hq/hkv):  s_ij = scale * q_i . k_j for j <= i (same sequence),
 *   LSE_i = log sum_j exp(s_ij),  O_i = sum_j exp(s_ij - LSE_i) v_j.
 * Q: device bf16 [T, hq, d]; K, V: device bf16 [T, hkv, d].
 * O: device bf16 [T, hq, d] (written); LSE: device fp32 [hq, T] (natural log,
 * written).  softmax_scale <= 0 selects 1/sqrt(d).
 * Source: the write-up's first solution (FlashAttention's LSE as the ratio's
 * denominator); the attention itself is plain causal softmax attention.
 */
lt_status lt_prefill_attn(const lt_shape* shape, const void* Q, const void* K, const void* V, void* O,
                          float* LSE, float softmax_scale, lt_stream stream);

/*
 * The assignment of attention work items to CTAs that lt_prefill_attn (fused
 * = 0) or lt_prefill_attn_ratio (fused = 1) computes on the host for one
 * sequence of `len` tokens passed without cu_seqlens, on a device with `grid`
 * SMs.  Host-only and synchronous; needs no device.  The pages have no
 * counterpart: the kernels' items are tiles of the causal attention (two query
 * tiles of 128 rows on one K/V stream, numbered heaviest first), and this call
 * exposes the launch's choice so that it can be checked.  A long sequence takes
 * the banded item order and a short one, when a longest-first assignment
 * (cost = key tiles per item, plus, with fused, the lazy ratio's masked key
 * tiles for S, W and n_obs as in lt_prefill_attn_ratio) lowers the slowest
 * CTA's load below the plain round-robin order's, that assignment.
 * Writes *num_items (the launch's item count) and *used: 1 when the static
 * assignment is used, 0 otherwise.  With *used = 1, CTA c (c < min(grid,
 * num_items)) runs item[off[c]] .. item[off[c+1] - 1] in that order; off: host
 * int32 [grid + 1], item: host int32 [capacity], capacity >= *num_items
 * (LT_ERR_INVALID_ARG otherwise, after *num_items and *used are written; off
 * and item are untouched when *used = 0).  head_dim 64 or 128, len >= 1,
 * hq a multiple of hkv, grid >= 1; with fused, S, W and n_obs as for
 * lt_prefill_attn_ratio.
 */
lt_status lt_attn_schedule(int head_dim, int fused, int len, int hq, int hkv, int S, int W, int n_obs, int grid,
                           int* used, int* num_items, int32_t* off, int32_t* item, int capacity);

/*
 * The same attention fused with the lazy ratio: O and LSE as lt_prefill_attn,
 * and ratio[b, h] as lt_lazy_ratio computes it (same S, W, n_obs and limits),
 * accumulated inside the attention's online softmax: for the observed rows the
 * weights of the keys in K_i are summed in the running-max frame of the
 * softmax denominator, so r_i = num_i / l_i = sum_{j in K_i} exp(s_ij - LSE_i)
 * with no second pass over the keys.  ratio: device fp32 [batch, hq], zeroed
 * by this call on `stream` and then written.  For n_obs <= 128 the result is
 * bitwise reproducible; above, the shares of more than two query tiles are
 * added by atomics and may round differently from run to run.
 * Sources: as lt_prefill_attn and lt_lazy_ratio (the write-up's first solution:
 * the ratio rides on the prefill's own softmax statistics).
 */
lt_status lt_prefill_attn_ratio(const lt_shape* shape, const void* Q, const void* K, const void* V, void* O,
                                float* LSE, float softmax_scale, int S, int W, int n_obs, float* ratio,
                                lt_stream stream);

/*
 * lt_prefill_attn_ratio without the zeroing: the kernel adds each query
 * tile's share of ratio[b, h] to what the buffer holds, so ratio must be zero
 * on entry (e.g. all layers' ratios cleared by one memset per prefill, instead
 * of one zeroing launch per layer).  Otherwise identical.
 */
lt_status lt_prefill_attn_ratio_acc(const lt_shape* shape, const void* Q, const void* K, const void* V, void* O,
                                    float* LSE, float softmax_scale, int S, int W, int n_obs, float* ratio,
                                    lt_stream stream);

/*
 * lt_prefill_attn_ratio_acc followed, inside the same kernel, by the
 * device-queue push of this layer (lt_dqueue_push(state, L, batch, layer,
 * ratio, hq)): the last CTA of the attention to finish -- after every CTA has
 * added its share of the ratios -- pushes each sequence's score, so a layer of
 * the prefill costs one launch fewer.  ratio must be zero on entry (as for
 * lt_prefill_attn_ratio_acc); state, L and the push's rule, slots and errors
 * are those of lt_dqueue_push.  If the attention gives up a bounded wait the
 * push is skipped, no layer is recorded as demoted by it and the queue's
 * error bit 4 is set (lt_dqueue_error).  With no tokens the push still
 * happens (every ratio 0).  The state also holds the launch's completion
 * counter: two launches that use the same state must not overlap.
 * Sources: as lt_prefill_attn_ratio and lt_dqueue_push.
 */
lt_status lt_prefill_attn_ratio_push(const lt_shape* shape, const void* Q, const void* K, const void* V, void* O,
                                     float* LSE, float softmax_scale, int S, int W, int n_obs, float* ratio,
                                     void* state, int L, int layer, lt_stream stream);

/*
 * Lazy ratio from the LSE.
 *   For every sequence b (length N), query head h and each of the last
 *   n' = min(n_obs, N) rows i of b:
 *     K_i = [0, min(S, i+1))  U  [max(S, i-W+1), i]      (sink + recent keys)
 *     r_i = sum_{j in K_i} exp(scale * q_i . k_j - LSE_i)
 *   ratio[b, h] = mean of r_i over those rows (0 when N == 0).
 * Q, K as for lt_prefill_attn; LSE: device fp32 [hq, T] as written by it.
 * ratio: device fp32 [batch, hq] (written).  S >= 0, W >= 0, S + W >= 1,
 * 1 <= n_obs <= 4096; hq and batch at most 65535 (one cluster of CTAs per
 * (sequence, query head)).  Deterministic: the same inputs give the same bits.
 * Sources: the press-release page's definition (attention weights to the
 * initial and recent keys) and the write-up's first solution (LSE as the
 * denominator; O(S+W) work per query).
 */
lt_status lt_lazy_ratio(const lt_shape* shape, const void* Q, const void* K, const float* LSE,
                        float softmax_scale, int S, int W, int n_obs, float* ratio, lt_stream stream);

/* Score of one layer of one sequence: the mean of its hq ratios (host). */
float lt_layer_score(const float* ratio_of_heads, int hq);

/*
 * Offline selection (every layer's ratio known; the post-prefill route the
 * write-up contrasts the queue with).  ratios: host fp32 [L, batch, hq].  For each
 * sequence the layers are ranked by (score descending, layer ascending) and
 * the first `budget` are lazy.  lazy_mask: host uint8 [batch, L] (written, 0/1);
 * order: host int32 [batch, budget] (nullable; written in rank order).
 * 0 <= budget <= L.  A non-finite score (NaN or +-inf) is rejected with
 * LT_ERR_INVALID_ARG, as lt_queue_push rejects it.  Host-only, synchronous.
 */
lt_status lt_select_layers(const float* ratios, int L, int batch, int hq, int budget, uint8_t* lazy_mask,
                           int32_t* order);

/*
 * Online layer priority queue of one sequence (project page, Figure 2 caption;
 * write-up, second solution).  Capacity C = L - budget full-KV layers.
 * lt_queue_push adds (layer, score); if more than C layers are then queued, the
 * best-ranked one (highest score; lower index on a tie) is popped and returned
 * in *demoted (else -1): that layer becomes a streaming layer.  Pushing each
 * of the L layers once demotes exactly `budget` layers, the same set as
 * lt_select_layers.  A layer pushed twice, out of range, or with a non-finite
 * score is rejected with LT_ERR_INVALID_ARG and leaves the queue unchanged.
 * Host-only, synchronous; one queue per sequence; not thread-safe.
 */
typedef struct lt_queue lt_queue;
lt_status lt_queue_create(int L, int budget, lt_queue** queue);
lt_status lt_queue_push(lt_queue* queue, int layer, float score, int* demoted);
int lt_queue_size(const lt_queue* queue);
void lt_queue_destroy(lt_queue* queue);

/*
 * KV-cache compaction of one layer to its streaming version.
 *   For every sequence b with mask[b] != 0 (length N):
 *     p = [0, min(S, N)) ++ [max(S, N - W), N)      (kept positions, in order)
 *     K_stream[b, kh, r, :] = K[cu[b] + p_r, kh, :]  for r < len = |p| = min(N, S+W)
 *     rows r >= len are zero; stream_len[b] = len.  Same for V.
 *   Sequences with mask[b] == 0 are not touched and get stream_len[b] = 0.
 * K, V: device bf16 [T, hkv, d]; mask: device uint8 [batch];
 * K_stream, V_stream: device bf16 [batch, hkv, S + W, d]; stream_len: device
 * int32 [batch].  S >= 0, W >= 0, S + W >= 1.  After this call is enqueued the
 * caller may release the layer's full K/V in stream order (the write-up's
 * "switch its KV cache to the streaming version").
 */
lt_status lt_compact_kv(const lt_shape* shape, const void* K, const void* V, const uint8_t* mask, int S, int W,
                        void* K_stream, void* V_stream, int32_t* stream_len, lt_stream stream);

/*
 * The same compaction for several layers in one launch, every sequence:
 *   K_pool[k, b, kh, r, :] = K_{layers[k]}[cu[b] + p_r, kh, :],
 *   pool_len[k, b] = |p|,  rows r >= |p| zero,  for k < n.
 * A layer index outside [0, L) leaves slot k untouched.  K_layers, V_layers:
 * device arrays of L device pointers (layer l's K/V [T, hkv, d] bf16);
 * layers: device int32 [n], 0 <= n <= L; K_pool, V_pool: device bf16
 * [n, batch, hkv, S+W, d]; pool_len: device int32 [n, batch].  One layer's
 * compaction is a few MB and bound by latency; the demoted layers of a whole
 * prefill together give the copy engine enough independent work.
 */
lt_status lt_compact_kv_layers(const lt_shape* shape, const void* const* K_layers, const void* const* V_layers, int L,
                               const int32_t* layers, int n, int S, int W, void* K_pool, void* V_pool,
                               int32_t* pool_len, lt_stream stream);

/*
 * Device-resident layer queue (the queue of lt_queue_push kept in device
 * memory, one per sequence of a batch), so that a whole prefill -- attention,
 * ratio, queue, compaction for every layer -- is one stream of kernels with no
 * host round trip (capturable in a CUDA graph).  Same rule and tie-break as
 * lt_queue_push; the score is the mean of the layer's hq ratios computed exactly
 * as lt_layer_score does, so host and device queues demote the same layers.
 *
 * state: caller-allocated device memory of lt_dqueue_state_bytes(L, batch)
 * bytes (4 * (8 + 3 batch + 5 batch L)), 16-byte aligned; lt_dqueue_init
 * (re)initialises it on `stream`.
 *
 * The queue also assigns full-KV slots for a memory-capped prefill
 * (lt_kv_pool_commit): each queued layer owns one of C = L - budget slots.
 * A pushed layer takes a never-used slot (slot n-1 for the n-th queued
 * layer) while no layer has been demoted, afterwards the slot of the layer
 * its push demotes, or none when it is demoted by its own push.
 * lt_dqueue_push: ratio is device fp32 [batch, hq] (e.g. the ratio output of
 * lt_prefill_attn_ratio for this layer).  A push that is invalid for a
 * sequence (layer out of range or pushed twice, non-finite score) leaves that
 * sequence's queue unchanged and sets an error bit that lt_dqueue_error
 * reads (synchronously).  L, batch must match the values given to init.
 * lt_dqueue_result writes lazy_mask (device uint8 [batch, L]) and, if not
 * null, order (device int32 [batch, budget]: demoted layers in demotion
 * order, -1 past the number demoted so far).
 */
size_t lt_dqueue_state_bytes(int L, int batch);
lt_status lt_dqueue_init(void* state, int L, int budget, int batch, lt_stream stream);
lt_status lt_dqueue_push(void* state, int L, int batch, int layer, const float* ratio, int hq, lt_stream stream);

/*
 * lt_dqueue_push for ratios gathered from head-sharded ranks: ratio is device
 * fp32 [shards, batch, hq_shard], where shard n holds query heads
 * [n hq_shard, (n+1) hq_shard) -- the buffer an all-gather of every rank's
 * [batch, hq_shard] lt_prefill_attn_ratio output fills.  The score of sequence
 * b is the mean of its shards * hq_shard head ratios, summed in head order, so
 * it equals bit for bit the score lt_dqueue_push computes from the same ratios
 * laid out [batch, hq]; every rank that pushes the same gathered buffer makes
 * the same demotion.  (The pages describe a single GPU; this split of the
 * heads over GPUs is this library's reading, with one exchange per layer.)
 * lt_dqueue_push(..., hq) is lt_dqueue_push_gathered(..., 1, hq).  Errors as
 * lt_dqueue_push; shards < 1 or hq_shard < 1 is LT_ERR_INVALID_ARG.
 */
lt_status lt_dqueue_push_gathered(void* state, int L, int batch, int layer, const float* ratio, int shards,
                                  int hq_shard, lt_stream stream);
lt_status lt_dqueue_result(const void* state, int L, int batch, int budget, uint8_t* lazy_mask, int32_t* order,
                           lt_stream stream);
/* Error bits of the queue (synchronous): 1 an invalid push, 2 a call whose
 * L / batch differ from init's, 4 a fused push skipped (lt_prefill_attn_ratio_push). */
lt_status lt_dqueue_error(const void* state, int* error_bits);
/* slots: device int32 [batch, L] (written): the full-KV slot of each layer of
 * each sequence, -1 for a layer that holds none (demoted, or not pushed). */
lt_status lt_dqueue_slots(const void* state, int L, int batch, int32_t* slots, lt_stream stream);

/*
 * Compaction driven by the device queue: for every sequence b whose latest
 * lt_dqueue_push demoted a layer m (the k-th demotion of b, k from 0), the
 * streaming rows of layer m (as lt_compact_kv: p = [0, min(S,N)) ++
 * [max(S, N-W), N), zero past the kept count) are written to pool slot k:
 *   K_pool[k, b, kh, r, :] = K_m[cu[b] + p_r, kh, :],  pool_len[k, b] = |p|.
 * Sequences with no demotion in the latest push are not touched.
 * K_layers, V_layers: device arrays of L device pointers (layer l's K/V
 * [T, hkv, d] bf16).  K_pool, V_pool: device bf16 [budget, batch, hkv, S+W, d];
 * pool_len: device int32 [budget, batch].  Enqueue it right after the push
 * (same stream) and before the next push.
 */
lt_status lt_compact_kv_pending(const lt_shape* shape, const void* const* K_layers, const void* const* V_layers,
                                const void* state, int L, int budget, int S, int W, void* K_pool, void* V_pool,
                                int32_t* pool_len, lt_stream stream);

/*
 * One layer of the prefill under the peak-memory cap: "the layer with the
 * highest ratio is made lazy and its KV cache reduced, freeing memory for
 * storing the KV cache of the current layer" (project page, Methodology,
 * LightTransfer-Test, Figure 2 caption; the write-up's second solution:
 * at most 50% full KV + 50% streaming KV at the prefill's peak).  Enqueue it
 * right after the push of `layer` (lt_dqueue_push or
 * lt_prefill_attn_ratio_push).  For every sequence b:
 *   - if the push demoted a layer m (the k-th demotion of b), m's streaming
 *     rows p = [0, min(S,N)) ++ [max(S, N-W), N) are written to streaming slot
 *     k (as lt_compact_kv_pending; zero past the kept count, stream_len[k, b]
 *     = |p|), read from K_cur/V_cur when m == layer, else from m's full-KV slot;
 *   - if the current layer holds a full-KV slot s after the push (it was not
 *     demoted), its rows are stored there: K_full[s, cu[b] + r] = K_cur[cu[b] + r]
 *     for every r < N (same for V) -- when m != layer, s is the slot m just
 *     released, and m's kept rows are read before they are overwritten.
 * K_cur, V_cur: device bf16 [T, hkv, d], the current layer's K/V in a buffer of
 * the caller's (read only; with the full-KV slots, at most C + 1 layers' full
 * KV exist at once).  K_full, V_full: device bf16 [L - budget, T, hkv, d]
 * (unused when budget == L).  K_stream, V_stream: device bf16
 * [budget, batch, hkv, S+W, d]; stream_len: device int32 [budget, batch]
 * (unused when budget == 0).  The layer -> slot map is read back with
 * lt_dqueue_slots (e.g. for decode of the full layers: sequence b's rows of
 * layer l start at row slot * T + cu[b] of K_full viewed as [(L-budget) T, hkv, d]).
 * Errors: LT_ERR_INVALID_ARG for a bad shape, state size, layer or window, or
 * misaligned buffers.  Asynchronous on `stream`; nothing is allocated.
 */
lt_status lt_kv_pool_commit(const lt_shape* shape, const void* K_cur, const void* V_cur, const void* state, int L,
                            int budget, int layer, int S, int W, void* K_full, void* V_full, void* K_stream,
                            void* V_stream, int32_t* stream_len, lt_stream stream);

/*
 * Decode on a demoted layer's streaming KV cache (press-release page: the
 * converted layers use streaming attention with a constant-size KV cache).
 * The cache is the [batch, hkv, S+W, d] bf16 layout lt_compact_kv writes, with
 * stream_len[b] valid rows: rows [0, S) hold the sink positions and rows
 * [S, S+W) the recent window, used as a ring once full.
 *
 * lt_stream_ring_init: next_slot[b] = stream_len[b] < S+W ? stream_len[b] : S,
 * the slot the next token goes to (device int32 [batch]).  Call once after
 * compaction.
 * lt_stream_append: writes the new token's key and value (k_new, v_new: device
 * bf16 [batch, hkv, d]) into slot next_slot[b] of every KV head, then advances
 * stream_len / next_slot: while the cache is not full the token is appended;
 * once full it replaces the window's oldest row.  The cache then holds the key
 * set K_p = [0, min(S, p+1)) U [max(S, p-W+1), p] of the token at position p.
 * W >= 1.  A sequence whose (stream_len, next_slot) no init/append sequence can
 * produce (next_slot outside [0, S+W), or a non-full cache whose next_slot is
 * not stream_len) is skipped: nothing is written for it.
 * lt_stream_decode: for each sequence b and query head h (KV head h / g):
 *   LSE[b, h] = log sum_{r < len} exp(scale q . K_s[b, kh, r]),
 *   O[b, h]   = sum_r exp(scale q . K_s[b, kh, r] - LSE) V_s[b, kh, r]
 * q, O: device bf16 [batch, hq, d]; LSE: device fp32 [batch, hq] (natural log;
 * -inf and O = 0 for a sequence with no rows).  slots = S + W of the cache;
 * stream_len[b] above slots is read as slots.  Errors: LT_ERR_INVALID_ARG for
 * misaligned pointers (q, K/V, O 16 bytes), batch outside [1, 65535], hq not a
 * multiple of hkv, slots < 1 or a non-finite scale; LT_ERR_UNSUPPORTED for
 * head_dim other than 64 and 128.  Buffers are the caller's; nothing is
 * allocated.  Asynchronous on `stream`.
 *
 * lt_decode_attn: the same decode step on a kept (full-attention) layer's
 * cache, token-major K/V [rows, hkv, d] bf16 with the rows of one sequence
 * contiguous: sequence b's position r is row seq_start[b] + r (device int32
 * [batch], e.g. the prefill's cu_seqlens) or, with seq_start NULL, row
 * b * seq_capacity + r (a padded [batch, seq_capacity, hkv, d] cache).  len:
 * device int32 [batch], positions attended (read clamped to [0, max_len]);
 * max_len >= 1 bounds every len[b] (and seq_capacity >= max_len when seq_start
 * is NULL).  The caller guarantees the rows read lie inside K and V.  O and LSE
 * as for lt_stream_decode.  Both decode calls split each (sequence, KV head)
 * over a cluster of up to 16 CTAs merged in distributed shared memory; no
 * memory beyond the arguments is written.
 */
lt_status lt_stream_ring_init(const int32_t* stream_len, int32_t* next_slot, int batch, int S, int W,
                              lt_stream stream);
lt_status lt_stream_append(void* K_stream, void* V_stream, int32_t* stream_len, int32_t* next_slot, const void* k_new,
                           const void* v_new, int batch, int hkv, int head_dim, int S, int W, lt_stream stream);
lt_status lt_stream_decode(const void* q, const void* K_stream, const void* V_stream, const int32_t* stream_len,
                           int batch, int hq, int hkv, int head_dim, int slots, void* O, float* LSE,
                           float softmax_scale, lt_stream stream);
lt_status lt_decode_attn(const void* q, const void* K, const void* V, const int32_t* seq_start, int seq_capacity,
                         const int32_t* len, int batch, int hq, int hkv, int head_dim, int max_len, void* O,
                         float* LSE, float softmax_scale, lt_stream stream);

/*
 * lt_decode_attn split over many CTAs: the same decode step (same arguments,
 * layouts, results and errors, except head_dim 64/128 and the workspace),
 * with the rows of each (sequence, KV head) split over ceil(max_len / r) CTAs,
 * r = ceil(max_len / 16) clamped to [256, 1024] rows (at most 128 CTAs; any
 * number, where lt_decode_attn's cluster split stops at 16), so that a
 * batch-1 decode over a few KV heads keeps every SM streaming K/V.  Each CTA writes its partial softmax state
 * (running max and sum, unnormalised output of every query head) to
 * `workspace`; a second kernel merges the splits of each head in split order
 * (deterministic).  workspace: caller-allocated device memory of at least
 * lt_decode_splitk_workspace_bytes(batch, hq, head_dim, max_len) bytes
 * (batch * hq * splits * (head_dim + 2) floats), 16-byte aligned; its
 * contents on entry do not matter and on return are scratch.  Two launches on
 * `stream`; calls that share a workspace must not overlap.
 * LT_ERR_INVALID_ARG also for a missing or too small workspace.
 */
size_t lt_decode_splitk_workspace_bytes(int batch, int hq, int head_dim, int max_len);
lt_status lt_decode_attn_splitk(const void* q, const void* K, const void* V, const int32_t* seq_start,
                                int seq_capacity, const int32_t* len, int batch, int hq, int hkv, int head_dim,
                                int max_len, void* O, float* LSE, float softmax_scale, void* workspace,
                                size_t workspace_bytes, lt_stream stream);

/*
 * lt_decode_attn_splitk for callers that cannot allocate device memory when
 * they decode -- e.g. a plugin whose host framework owns all device memory,
 * or a serving loop where cudaMalloc's implicit synchronisation is not
 * allowed.  (The pages have no counterpart: this is an interface choice of
 * this library.)  Same arguments, results and errors as lt_decode_attn_splitk
 * without the workspace: the partial states go to a fixed array inside the
 * library's own device memory, lt_decode_splitk_noalloc_capacity_bytes()
 * bytes (4 MiB), which every device that loads the library holds until the
 * process exits.  A call whose lt_decode_splitk_workspace_bytes(batch, hq,
 * head_dim, max_len) exceeds it returns LT_ERR_INVALID_ARG and enqueues
 * nothing.  Nothing is allocated: the first library call on a device (this
 * one or any other) looks up the array's device address once, so make that
 * first call before any stream capture.  All calls on a device share the
 * array and it keeps the last call's contents; nothing in it needs to start
 * at zero, but calls that overlap on the GPU (other streams, or graphs
 * replayed concurrently) race on it and must be serialised by the caller.
 */
size_t lt_decode_splitk_noalloc_capacity_bytes(void);
lt_status lt_decode_attn_splitk_noalloc(const void* q, const void* K, const void* V, const int32_t* seq_start,
                                        int seq_capacity, const int32_t* len, int batch, int hq, int hkv,
                                        int head_dim, int max_len, void* O, float* LSE, float softmax_scale,
                                        lt_stream stream);

/*
 * Device status word of the current device: LT_OK, or LT_ERR_TIMEOUT if a kernel
 * gave up a bounded wait since the last clear.  Synchronises the device.
 * clear != 0 resets the word.
 */
lt_status lt_device_status(int clear);

/*
 * Self-test of the kernels' bounded waits: enqueues a one-thread kernel that
 * waits, with the same wait routine the kernels use, on an mbarrier nothing
 * arrives on; after limit_us microseconds (1 .. 10^7) it gives up, sets the
 * device status word and returns.  A following lt_device_status reports
 * LT_ERR_TIMEOUT; the device and the context stay usable.
 */
lt_status lt_selftest_wait_timeout(unsigned limit_us, lt_stream stream);

/* Human-readable name of a status. */
const char* lt_status_string(lt_status status);

/* Library version as major * 10000 + minor * 100 + patch. */
int lt_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LT_H_ */
