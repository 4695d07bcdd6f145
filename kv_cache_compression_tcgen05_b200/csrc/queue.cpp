// queue.cpp -- host side of the C ABI: the layer priority queue, the offline
// selection, status strings.
//
// LightTransfer project page (Methodology, LightTransfer-Test, Figure 2
// caption) and the LightTransfer write-up (second solution): during the
// prefill each layer enters a priority queue keyed by its lazy ratio; once more
// layers are queued than the full-KV capacity allows, the layer with the
// highest ratio is popped and its KV cache switched to the streaming version.
//
// The queue is a binary max-heap on (score, -layer).  With capacity
// C = L - budget every push that makes the size C + 1 pops exactly one layer,
// so L pushes demote `budget` layers.  A layer among the C lowest-ranked can
// never be the maximum of C + 1 queued layers, so the demoted set equals the
// top `budget` of a full sort (what lt_select_layers computes directly).
#include <cmath>
#include <cstdlib>
#include <new>
#include <vector>

#include "lt.h"

struct lt_queue {
  int L = 0;
  int budget = 0;
  int cap = 0;
  std::vector<float> score;      // score of each layer once pushed
  std::vector<unsigned char> pushed;
  std::vector<int> heap;         // layer indices, max-heap by rank
};

namespace {

// Does layer a outrank layer b (pop first)?  Higher score; lower index on a tie.
bool outranks(float sa, int a, float sb, int b) { return sa != sb ? sa > sb : a < b; }

void sift_up(lt_queue* q, int i) {
  while (i > 0) {
    const int parent = (i - 1) / 2;
    const int a = q->heap[i], b = q->heap[parent];
    if (!outranks(q->score[a], a, q->score[b], b)) break;
    q->heap[i] = b;
    q->heap[parent] = a;
    i = parent;
  }
}

void sift_down(lt_queue* q, int i) {
  const int n = int(q->heap.size());
  for (;;) {
    int best = i;
    for (int c = 2 * i + 1; c <= 2 * i + 2 && c < n; ++c) {
      const int a = q->heap[c], b = q->heap[best];
      if (outranks(q->score[a], a, q->score[b], b)) best = c;
    }
    if (best == i) return;
    const int t = q->heap[i];
    q->heap[i] = q->heap[best];
    q->heap[best] = t;
    i = best;
  }
}

}  // namespace

extern "C" {

lt_status lt_queue_create(int L, int budget, lt_queue** queue) {
  if (!queue || L < 0 || budget < 0 || budget > L) return LT_ERR_INVALID_ARG;
  lt_queue* q = new (std::nothrow) lt_queue;
  if (!q) return LT_ERR_INVALID_ARG;
  q->L = L;
  q->budget = budget;
  q->cap = L - budget;
  q->score.assign(size_t(L), 0.f);
  q->pushed.assign(size_t(L), 0);
  q->heap.reserve(size_t(L) + 1);
  *queue = q;
  return LT_OK;
}

lt_status lt_queue_push(lt_queue* q, int layer, float score, int* demoted) {
  if (!q || !demoted || layer < 0 || layer >= q->L || q->pushed[layer] || !std::isfinite(score))
    return LT_ERR_INVALID_ARG;
  q->pushed[layer] = 1;
  q->score[layer] = score;
  q->heap.push_back(layer);
  sift_up(q, int(q->heap.size()) - 1);
  *demoted = -1;
  if (int(q->heap.size()) > q->cap) {
    *demoted = q->heap[0];
    q->heap[0] = q->heap.back();
    q->heap.pop_back();
    if (!q->heap.empty()) sift_down(q, 0);
  }
  return LT_OK;
}

int lt_queue_size(const lt_queue* q) { return q ? int(q->heap.size()) : 0; }

void lt_queue_destroy(lt_queue* q) { delete q; }

float lt_layer_score(const float* ratio_of_heads, int hq) {
  if (!ratio_of_heads || hq < 1) return NAN;
  double sum = 0.0;
  for (int h = 0; h < hq; ++h) sum += ratio_of_heads[h];
  return float(sum / hq);
}

lt_status lt_select_layers(const float* ratios, int L, int batch, int hq, int budget, uint8_t* lazy_mask,
                           int32_t* order) {
  if (!ratios || !lazy_mask || L < 0 || batch < 1 || hq < 1 || budget < 0 || budget > L) return LT_ERR_INVALID_ARG;
  std::vector<float> score(size_t(L) > 0 ? size_t(L) : 1);
  std::vector<int> idx(size_t(L) > 0 ? size_t(L) : 1);
  for (int b = 0; b < batch; ++b) {
    for (int l = 0; l < L; ++l) {
      score[l] = lt_layer_score(ratios + (size_t(l) * batch + b) * hq, hq);
      if (!std::isfinite(score[l])) return LT_ERR_INVALID_ARG;   // as lt_queue_push
    }
  }
  for (int b = 0; b < batch; ++b) {
    for (int l = 0; l < L; ++l) {
      score[l] = lt_layer_score(ratios + (size_t(l) * batch + b) * hq, hq);
      idx[l] = l;
    }
    // Partial selection by repeated maximum: L is a layer count (tens).
    for (int r = 0; r < budget; ++r) {
      int best = r;
      for (int k = r + 1; k < L; ++k)
        if (outranks(score[idx[k]], idx[k], score[idx[best]], idx[best])) best = k;
      const int t = idx[r];
      idx[r] = idx[best];
      idx[best] = t;
    }
    for (int l = 0; l < L; ++l) lazy_mask[size_t(b) * L + l] = 0;
    for (int r = 0; r < budget; ++r) {
      lazy_mask[size_t(b) * L + idx[r]] = 1;
      if (order) order[size_t(b) * budget + r] = idx[r];
    }
  }
  return LT_OK;
}

const char* lt_status_string(lt_status s) {
  switch (s) {
    case LT_OK: return "LT_OK";
    case LT_ERR_INVALID_ARG: return "LT_ERR_INVALID_ARG";
    case LT_ERR_UNSUPPORTED: return "LT_ERR_UNSUPPORTED";
    case LT_ERR_CUDA: return "LT_ERR_CUDA";
    case LT_ERR_TIMEOUT: return "LT_ERR_TIMEOUT";
  }
  return "LT_ERR_UNKNOWN";
}

int lt_version(void) { return 100; }

}  // extern "C"
