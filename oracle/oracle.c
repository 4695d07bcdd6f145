/*
 * oracle.c -- plain, slow fp64 CPU oracle for the LightTransfer-Test prefill path.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check of the package entry
 * file and the CPU-baseline / reference leg of the benchmark load this library.
 * The CUDA product path never calls it, shares no code, header, table or helper
 * with it, and fails loudly when its own extension is missing.
 *
 * What it computes (every function is a definition written out, no blocking, no
 * fusion, no reordering beyond what the definition states):
 *
 *  - oracle_attn: causal self-attention of one prefill with the per-row
 *    log-sum-exp.  The LightTransfer write-up (xzbcqc.com news page, the
 *    "solution" paragraph under the Flash-Attention problem) takes the LSE that
 *    FlashAttention produces during the prefill as the denominator of the lazy
 *    ratio; FlashAttention's online softmax reaches exactly the plain softmax up
 *    to rounding, so the oracle is the plain definition:
 *        s_ij  = scale * q_i . k_j            (j <= i, same sequence)
 *        LSE_i = m_i + log sum_j exp(s_ij - m_i),   m_i = max_j s_ij
 *        O_i   = sum_j exp(s_ij - LSE_i) v_j
 *    Query head h reads key/value head floor(h / g), g = hq / hkv.
 *
 *  - oracle_lazy_ratio_rows / oracle_lazy_ratio: the lazy ratio. The press-release
 *    page ("LLM突破：推理加速，长CoT生成惊艳", section "LightTransfer方法详解")
 *    defines it as the sum of the attention weights from a query to the initial
 *    and the recent keys; the write-up's solution paragraph computes it with the
 *    LSE as denominator so that only the few keys of the numerator are visited.
 *    Reading adopted: for row i the key set is
 *        K_i = [0, min(S, i+1))  U  [max(S, i-W+1), i]
 *    (S sink keys, the W most recent keys up to and including i, no key twice),
 *    and
 *        route A:  r_i = sum_{j in K_i} exp(s_ij - LSE_i)
 *        route B:  r_i = sum_{j in K_i} p_ij,  p = the normalised softmax row.
 *    The ratio of (sequence, head) is the mean of r_i over the last
 *    min(n_obs, N_b) rows of the sequence.
 *
 *  - oracle_layer_scores: score of a layer = mean over query heads of its ratio.
 *
 *  - oracle_select_layers / oracle_queue_online: the layer priority queue of the
 *    LightTransfer project page (Methodology, LightTransfer-Test, Figure 2
 *    caption) and of the write-up's second solution paragraph: layers are pushed
 *    with their lazy ratio after each layer of the prefill; while more than
 *    C = L - budget layers are queued, the layer with the highest ratio is popped
 *    and becomes a streaming (lazy) layer.  Equal scores pop the lower layer
 *    index first.  oracle_select_layers is the offline route: a full sort by
 *    (score descending, layer ascending), first `budget` layers.
 *
 *  - oracle_compact_kv: the streaming version of a demoted layer's KV cache keeps
 *    the rows p = [0, min(S, N)) ++ [max(S, N - W), N) of every KV head.
 *
 *  - oracle_attn_keys: attention of one query row over an explicit set of key
 *    rows -- what a streaming (sink + recent window) layer computes at decode
 *    (press-release page: the converted layers use streaming attention, which
 *    needs only a constant-size KV cache):
 *        LSE = log sum_j exp(scale q.k_j),  O = sum_j exp(scale q.k_j - LSE) v_j.
 *
 * Inputs are bf16 bit patterns (uint16), decoded exactly to double.  All
 * arithmetic is fp64 with libm exp/log.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_bits_to_double(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Sequence b holding packed token t; -1 if t is outside [0, cu[batch]). */
static int sequence_of(const int32_t* cu, int batch, int64_t t) {
  for (int b = 0; b < batch; ++b)
    if (t >= cu[b] && t < cu[b + 1]) return b;
  return -1;
}

typedef struct {
  const int32_t* cu;
  int batch, hq, hkv, d;
  const uint16_t* Q;
  const uint16_t* K;
  const uint16_t* V;
  double scale;
} problem_t;

static double score(const problem_t* p, int64_t tq, int h, int64_t tk) {
  const int kh = h / (p->hq / p->hkv);
  const uint16_t* q = p->Q + ((size_t)tq * p->hq + h) * p->d;
  const uint16_t* k = p->K + ((size_t)tk * p->hkv + kh) * p->d;
  double acc = 0.0;
  for (int c = 0; c < p->d; ++c) acc += bf16_bits_to_double(q[c]) * bf16_bits_to_double(k[c]);
  return p->scale * acc;
}

/* LSE of query row (token t, head h); s receives the scores of keys 0..i. */
static double row_lse(const problem_t* p, int64_t t, int h, double* s, int64_t* start_out, int64_t* i_out) {
  const int b = sequence_of(p->cu, p->batch, t);
  const int64_t start = p->cu[b];
  const int64_t i = t - start;
  double m = -INFINITY;
  for (int64_t j = 0; j <= i; ++j) {
    s[j] = score(p, t, h, start + j);
    if (s[j] > m) m = s[j];
  }
  double sum = 0.0;
  for (int64_t j = 0; j <= i; ++j) sum += exp(s[j] - m);
  *start_out = start;
  *i_out = i;
  return m + log(sum);
}

/* ------------------------------------------------------------------ threads */

typedef struct {
  void (*fn)(void* ctx, int64_t item, double* scratch);
  void* ctx;
  int64_t begin, end;
  int64_t scratch_len;
  int failed;
} chunk_t;

static void* run_chunk(void* arg) {
  chunk_t* c = (chunk_t*)arg;
  double* scratch = (double*)malloc(sizeof(double) * (size_t)(c->scratch_len > 0 ? c->scratch_len : 1));
  if (!scratch) { c->failed = 1; return NULL; }
  for (int64_t it = c->begin; it < c->end; ++it) c->fn(c->ctx, it, scratch);
  free(scratch);
  return NULL;
}

/* Runs fn over items [0, n) split into nthreads contiguous ranges. */
static int parallel_for(void (*fn)(void*, int64_t, double*), void* ctx, int64_t n, int64_t scratch_len, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (n < nthreads) nthreads = n > 0 ? (int)n : 1;
  chunk_t chunks[256];
  pthread_t tids[256];
  int started[256];
  for (int k = 0; k < nthreads; ++k) {
    chunks[k].fn = fn;
    chunks[k].ctx = ctx;
    chunks[k].begin = n * k / nthreads;
    chunks[k].end = n * (k + 1) / nthreads;
    chunks[k].scratch_len = scratch_len;
    chunks[k].failed = 0;
    started[k] = 0;
  }
  for (int k = 1; k < nthreads; ++k)
    started[k] = pthread_create(&tids[k], NULL, run_chunk, &chunks[k]) == 0;
  run_chunk(&chunks[0]);
  int failed = chunks[0].failed;
  for (int k = 1; k < nthreads; ++k) {
    if (started[k]) pthread_join(tids[k], NULL);
    else run_chunk(&chunks[k]);
    failed |= chunks[k].failed;
  }
  return failed ? -2 : 0;
}

static int check_problem(const problem_t* p) {
  if (!p->cu || !p->Q || !p->K || p->batch < 1 || p->hq < 1 || p->hkv < 1 || p->d < 1) return -1;
  if (p->hq % p->hkv != 0) return -1;
  if (p->cu[0] != 0) return -1;
  for (int b = 0; b < p->batch; ++b)
    if (p->cu[b + 1] < p->cu[b]) return -1;
  return 0;
}

static int64_t max_seqlen(const problem_t* p) {
  int64_t mx = 0;
  for (int b = 0; b < p->batch; ++b)
    if (p->cu[b + 1] - p->cu[b] > mx) mx = p->cu[b + 1] - p->cu[b];
  return mx;
}

/* --------------------------------------------------------------- attention */

typedef struct {
  problem_t p;
  const int32_t* tokens;
  const int32_t* heads;
  double* O;
  double* LSE;
} attn_ctx_t;

static void attn_item(void* vctx, int64_t it, double* s) {
  attn_ctx_t* c = (attn_ctx_t*)vctx;
  const problem_t* p = &c->p;
  const int64_t t = c->tokens[it];
  const int h = c->heads[it];
  int64_t start, i;
  const double lse = row_lse(p, t, h, s, &start, &i);
  const int kh = h / (p->hq / p->hkv);
  double* o = c->O + (size_t)it * p->d;
  for (int ch = 0; ch < p->d; ++ch) o[ch] = 0.0;
  for (int64_t j = 0; j <= i; ++j) {
    const double w = exp(s[j] - lse);
    const uint16_t* v = p->V + ((size_t)(start + j) * p->hkv + kh) * p->d;
    for (int ch = 0; ch < p->d; ++ch) o[ch] += w * bf16_bits_to_double(v[ch]);
  }
  c->LSE[it] = lse;
}

/*
 * Attention output and LSE for the listed query rows.
 * cu_seqlens: host int32 [batch+1] (cu[0] = 0, non-decreasing).
 * Q [T, hq, d], K/V [T, hkv, d]: bf16 bits.  Item k is (tokens[k], heads[k]).
 * O: [n_items, d] double; LSE: [n_items] double.  Returns 0, -1 on bad args,
 * -2 on allocation failure.
 */
int oracle_attn(const int32_t* cu_seqlens, int batch, int hq, int hkv, int d, const uint16_t* Q,
                const uint16_t* K, const uint16_t* V, double scale, const int32_t* tokens,
                const int32_t* heads, int64_t n_items, double* O, double* LSE, int nthreads) {
  attn_ctx_t c = {{cu_seqlens, batch, hq, hkv, d, Q, K, V, scale}, tokens, heads, O, LSE};
  if (check_problem(&c.p) || !V || (n_items > 0 && (!tokens || !heads || !O || !LSE))) return -1;
  for (int64_t it = 0; it < n_items; ++it)
    if (tokens[it] < 0 || tokens[it] >= cu_seqlens[batch] || heads[it] < 0 || heads[it] >= hq) return -1;
  return parallel_for(attn_item, &c, n_items, max_seqlen(&c.p) + 1, nthreads);
}

/* -------------------------------------------------------------- lazy ratio */

/* Is key position j in the key set K_i of query position i? */
static int in_key_set(int64_t i, int64_t j, int S, int W) {
  if (j < 0 || j > i) return 0;
  if (j < S) return 1;                 /* the S initial (sink) keys */
  return j >= i - (int64_t)W + 1;      /* the W most recent keys, ending at i */
}

typedef struct {
  problem_t p;
  int S, W, route;
  const int32_t* tokens;
  const int32_t* heads;
  const double* lse_in;
  double* r;
} ratio_ctx_t;

static void ratio_item(void* vctx, int64_t it, double* s) {
  ratio_ctx_t* c = (ratio_ctx_t*)vctx;
  const problem_t* p = &c->p;
  const int64_t t = c->tokens[it];
  const int h = c->heads[it];
  int64_t start, i;
  double r = 0.0;
  if (c->route == 0) {
    /* Route A: numerator over K_i only, denominator exp(LSE_i). */
    double lse;
    if (c->lse_in) {
      const int b = sequence_of(p->cu, p->batch, t);
      start = p->cu[b];
      i = t - start;
      lse = c->lse_in[it];
    } else {
      lse = row_lse(p, t, h, s, &start, &i);
    }
    for (int64_t j = 0; j <= i; ++j)
      if (in_key_set(i, j, c->S, c->W)) r += exp(score(p, t, h, start + j) - lse);
  } else {
    /* Route B: the attention weights of the whole row, normalised, then the
       weights of the keys in K_i summed. */
    int64_t st, ii;
    (void)row_lse(p, t, h, s, &st, &ii);
    start = st;
    i = ii;
    double m = -INFINITY;
    for (int64_t j = 0; j <= i; ++j)
      if (s[j] > m) m = s[j];
    double z = 0.0;
    for (int64_t j = 0; j <= i; ++j) z += exp(s[j] - m);
    for (int64_t j = 0; j <= i; ++j)
      if (in_key_set(i, j, c->S, c->W)) r += exp(s[j] - m) / z;
  }
  c->r[it] = r;
}

/*
 * Per-row lazy ratio r_i for the listed (token, head) items.
 * lse_in: nullable [n_items]; when given, route A uses it as LSE_i instead of
 * computing the row's LSE.  route: 0 = A, 1 = B (lse_in ignored).
 */
int oracle_lazy_ratio_rows(const int32_t* cu_seqlens, int batch, int hq, int hkv, int d,
                           const uint16_t* Q, const uint16_t* K, double scale, int S, int W,
                           const int32_t* tokens, const int32_t* heads, int64_t n_items,
                           const double* lse_in, int route, double* r_out, int nthreads) {
  ratio_ctx_t c = {{cu_seqlens, batch, hq, hkv, d, Q, K, NULL, scale}, S, W, route, tokens, heads,
                   lse_in, r_out};
  if (check_problem(&c.p) || S < 0 || W < 0 || (route != 0 && route != 1)) return -1;
  if (n_items > 0 && (!tokens || !heads || !r_out)) return -1;
  for (int64_t it = 0; it < n_items; ++it)
    if (tokens[it] < 0 || tokens[it] >= cu_seqlens[batch] || heads[it] < 0 || heads[it] >= hq) return -1;
  return parallel_for(ratio_item, &c, n_items, max_seqlen(&c.p) + 1, nthreads);
}

/*
 * ratio[b, h] = mean over the last min(n_obs, N_b) rows i of sequence b of r_i
 * (route A, LSE computed by the oracle unless lse_in [hq, T] is given).
 * An empty sequence gets ratio 0.
 */
int oracle_lazy_ratio(const int32_t* cu_seqlens, int batch, int hq, int hkv, int d, const uint16_t* Q,
                      const uint16_t* K, double scale, int S, int W, int n_obs, const double* lse_in,
                      double* ratio, int nthreads) {
  if (!cu_seqlens || batch < 1 || hq < 1 || n_obs < 0 || !ratio) return -1;
  const int64_t T = cu_seqlens[batch];
  int64_t n_items = 0;
  for (int b = 0; b < batch; ++b) {
    const int64_t N = cu_seqlens[b + 1] - cu_seqlens[b];
    n_items += (int64_t)hq * (N < n_obs ? N : n_obs);
  }
  int32_t* tokens = (int32_t*)malloc(sizeof(int32_t) * (size_t)(n_items + 1));
  int32_t* heads = (int32_t*)malloc(sizeof(int32_t) * (size_t)(n_items + 1));
  double* lse = lse_in ? (double*)malloc(sizeof(double) * (size_t)(n_items + 1)) : NULL;
  double* r = (double*)malloc(sizeof(double) * (size_t)(n_items + 1));
  int rc = -2;
  if (!tokens || !heads || !r || (lse_in && !lse)) goto done;
  int64_t k = 0;
  for (int b = 0; b < batch; ++b) {
    const int64_t N = cu_seqlens[b + 1] - cu_seqlens[b];
    const int64_t nb = N < n_obs ? N : n_obs;
    for (int h = 0; h < hq; ++h)
      for (int64_t x = 0; x < nb; ++x) {
        tokens[k] = (int32_t)(cu_seqlens[b + 1] - nb + x);
        heads[k] = h;
        if (lse) lse[k] = lse_in[(size_t)h * T + tokens[k]];
        ++k;
      }
  }
  rc = oracle_lazy_ratio_rows(cu_seqlens, batch, hq, hkv, d, Q, K, scale, S, W, tokens, heads, n_items,
                              lse, 0, r, nthreads);
  if (rc) goto done;
  k = 0;
  for (int b = 0; b < batch; ++b) {
    const int64_t N = cu_seqlens[b + 1] - cu_seqlens[b];
    const int64_t nb = N < n_obs ? N : n_obs;
    for (int h = 0; h < hq; ++h) {
      double sum = 0.0;
      for (int64_t x = 0; x < nb; ++x) sum += r[k++];
      ratio[(size_t)b * hq + h] = nb > 0 ? sum / (double)nb : 0.0;
    }
  }
done:
  free(tokens);
  free(heads);
  free(lse);
  free(r);
  return rc;
}

/* scores[b, l] = mean over h of ratios[l, b, h]. */
int oracle_layer_scores(const double* ratios, int L, int batch, int hq, double* scores) {
  if (!ratios || !scores || L < 0 || batch < 1 || hq < 1) return -1;
  for (int b = 0; b < batch; ++b)
    for (int l = 0; l < L; ++l) {
      double sum = 0.0;
      for (int h = 0; h < hq; ++h) sum += ratios[((size_t)l * batch + b) * hq + h];
      scores[(size_t)b * L + l] = sum / (double)hq;
    }
  return 0;
}

/* ------------------------------------------------------------ layer queue */

/* Does layer a (score sa) outrank layer b (score sb)? Higher score first; on a
   tie the lower layer index. */
static int outranks(double sa, int a, double sb, int b) {
  if (sa != sb) return sa > sb;
  return a < b;
}

/*
 * Offline selection: sort the L layers by (score desc, layer asc); the first
 * `budget` are lazy.  lazy: [L] 0/1.  order: nullable [budget], the lazy layers
 * in rank order.
 */
int oracle_select_layers(const double* scores, int L, int budget, uint8_t* lazy, int32_t* order) {
  if (!scores || !lazy || L < 0 || budget < 0 || budget > L) return -1;
  for (int l = 0; l < L; ++l)
    if (scores[l] != scores[l]) return -1;
  int* idx = (int*)malloc(sizeof(int) * (size_t)(L > 0 ? L : 1));
  if (!idx) return -2;
  for (int l = 0; l < L; ++l) idx[l] = l;
  /* insertion sort: plain and obviously correct for the small L involved */
  for (int a = 1; a < L; ++a) {
    int cur = idx[a];
    int k = a - 1;
    while (k >= 0 && outranks(scores[cur], cur, scores[idx[k]], idx[k])) {
      idx[k + 1] = idx[k];
      --k;
    }
    idx[k + 1] = cur;
  }
  for (int l = 0; l < L; ++l) lazy[l] = 0;
  for (int r = 0; r < budget; ++r) {
    lazy[idx[r]] = 1;
    if (order) order[r] = idx[r];
  }
  free(idx);
  return 0;
}

/*
 * Online queue: push layers in push_order (nullable: 0..L-1), each with its
 * score; after each push, while more than C = L - budget layers are queued,
 * pop the highest-ranked one.  popped: [budget] in pop order; *n_popped gets
 * the count.
 */
int oracle_queue_online(const double* scores, int L, int budget, const int32_t* push_order,
                        int32_t* popped, int* n_popped) {
  if (!scores || !popped || !n_popped || L < 0 || budget < 0 || budget > L) return -1;
  const int cap = L - budget;
  int* queued = (int*)malloc(sizeof(int) * (size_t)(L + 1));
  if (!queued) return -2;
  int size = 0, np = 0;
  for (int step = 0; step < L; ++step) {
    const int l = push_order ? push_order[step] : step;
    if (l < 0 || l >= L || scores[l] != scores[l]) { free(queued); return -1; }
    queued[size++] = l;
    while (size > cap) {
      int best = 0;
      for (int k = 1; k < size; ++k)
        if (outranks(scores[queued[k]], queued[k], scores[queued[best]], queued[best])) best = k;
      popped[np++] = queued[best];
      queued[best] = queued[--size];
    }
  }
  *n_popped = np;
  free(queued);
  return 0;
}

/* -------------------------------------------------------------- compaction */

/*
 * For every sequence b with mask[b] != 0: Ks[b, kh, r, :] = K[cu[b] + p_r, kh, :]
 * (same for V) with p = [0, min(S, N)) ++ [max(S, N - W), N); rows r >= len of
 * the S+W slots are zero; len[b] = number of kept rows.  Sequences with
 * mask[b] == 0 are left untouched and get len[b] = 0.
 * Ks/Vs: [batch, hkv, S+W, d] bf16 bits.
 */
int oracle_compact_kv(const int32_t* cu_seqlens, int batch, int hkv, int d, const uint16_t* K,
                      const uint16_t* V, const uint8_t* mask, int S, int W, uint16_t* Ks, uint16_t* Vs,
                      int32_t* len) {
  if (!cu_seqlens || !K || !V || !mask || !Ks || !Vs || !len || batch < 1 || hkv < 1 || d < 1 || S < 0 ||
      W < 0 || S + W < 1)
    return -1;
  const int slots = S + W;
  for (int b = 0; b < batch; ++b) {
    if (!mask[b]) { len[b] = 0; continue; }
    const int64_t start = cu_seqlens[b];
    const int64_t N = cu_seqlens[b + 1] - start;
    int n = 0;
    for (int64_t pos = 0; pos < N; ++pos) {
      const int sink = pos < S;
      const int recent = pos >= N - W && pos >= S;
      if (sink || recent) {
        for (int kh = 0; kh < hkv; ++kh) {
          const size_t src = ((size_t)(start + pos) * hkv + kh) * d;
          const size_t dst = (((size_t)b * hkv + kh) * slots + n) * d;
          memcpy(Ks + dst, K + src, sizeof(uint16_t) * (size_t)d);
          memcpy(Vs + dst, V + src, sizeof(uint16_t) * (size_t)d);
        }
        ++n;
      }
    }
    for (int r = n; r < slots; ++r)
      for (int kh = 0; kh < hkv; ++kh) {
        const size_t dst = (((size_t)b * hkv + kh) * slots + r) * d;
        memset(Ks + dst, 0, sizeof(uint16_t) * (size_t)d);
        memset(Vs + dst, 0, sizeof(uint16_t) * (size_t)d);
      }
    len[b] = n;
  }
  return 0;
}

/* ------------------------------------------------------- keyed attention */

/*
 * Item n: query q[n, :] against the first m[n] rows of K[n, :, :], V[n, :, :]
 * (each [m_max, d], bf16 bits).  O: [n_items, d]; LSE: [n_items].  An item with
 * no keys gets O = 0 and LSE = -inf.
 */
int oracle_attn_keys(int64_t n_items, int m_max, int d, const uint16_t* q, const uint16_t* K, const uint16_t* V,
                     const int32_t* m, double scale, double* O, double* LSE) {
  if (n_items < 0 || m_max < 0 || d < 1 || (n_items > 0 && (!q || !K || !V || !m || !O || !LSE))) return -1;
  double* s = (double*)malloc(sizeof(double) * (size_t)(m_max > 0 ? m_max : 1));
  if (!s) return -2;
  for (int64_t it = 0; it < n_items; ++it) {
    const int mk = m[it];
    if (mk < 0 || mk > m_max) { free(s); return -1; }
    const uint16_t* qr = q + (size_t)it * d;
    double* o = O + (size_t)it * d;
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    if (mk == 0) { LSE[it] = -INFINITY; continue; }
    double mx = -INFINITY;
    for (int j = 0; j < mk; ++j) {
      const uint16_t* kr = K + ((size_t)it * m_max + j) * d;
      double acc = 0.0;
      for (int c = 0; c < d; ++c) acc += bf16_bits_to_double(qr[c]) * bf16_bits_to_double(kr[c]);
      s[j] = scale * acc;
      if (s[j] > mx) mx = s[j];
    }
    double sum = 0.0;
    for (int j = 0; j < mk; ++j) sum += exp(s[j] - mx);
    const double lse = mx + log(sum);
    for (int j = 0; j < mk; ++j) {
      const double w = exp(s[j] - lse);
      const uint16_t* vr = V + ((size_t)it * m_max + j) * d;
      for (int c = 0; c < d; ++c) o[c] += w * bf16_bits_to_double(vr[c]);
    }
    LSE[it] = lse;
  }
  free(s);
  return 0;
}
