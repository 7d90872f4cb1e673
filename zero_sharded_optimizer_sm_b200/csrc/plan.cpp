#include "plan.hpp"

#include <algorithm>

namespace zsm {

namespace {
int64_t align_up(int64_t x, int64_t m) { return ((x + m - 1) / m) * m; }
}  // namespace

int Plan::layer_of(int64_t i) const {
  int lo = 0, hi = (int)layers.size() - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) / 2;
    if (layers[mid].lo <= i) lo = mid; else hi = mid - 1;
  }
  return lo;
}

bool make_plan(int32_t n_tensors, const int64_t* numel, const int32_t* layer_id, int32_t n_ranks,
               int64_t bucket_elems, Plan* out, std::string* err) {
  if (n_tensors <= 0 || !numel || !layer_id) {
    *err = "layout needs n_tensors >= 1 and non-null numel/layer_id";
    return false;
  }
  if (bucket_elems < 0 || bucket_elems % kGranule != 0) {
    *err = "bucket_elems must be 0 (one bucket) or a positive multiple of 8";
    return false;
  }
  Plan p;
  p.n_ranks = n_ranks;
  p.bucket_elems = bucket_elems;
  p.numel.assign(numel, numel + n_tensors);
  p.layer_id.assign(layer_id, layer_id + n_tensors);
  int64_t cursor = 0;
  for (int32_t k = 0; k < n_tensors; ++k) {
    if (numel[k] < 0) {
      *err = "tensor " + std::to_string(k) + " has a negative size";
      return false;
    }
    if (k > 0 && layer_id[k] < layer_id[k - 1]) {
      *err = "layer ids must be non-decreasing (tensor " + std::to_string(k) + ")";
      return false;
    }
    if (numel[k] > ((int64_t)1 << 50) || cursor > ((int64_t)1 << 52)) {
      *err = "parameter count out of range";
      return false;
    }
    p.start.push_back(cursor);
    p.psi += numel[k];
    cursor = align_up(cursor + numel[k], kGranule);
  }
  p.psi_pad = align_up(std::max<int64_t>(cursor, 1), kGranule * n_ranks);
  p.shard = p.psi_pad / n_ranks;
  for (int32_t k = 0; k < n_tensors; ++k)
    p.slot_end.push_back(k + 1 < n_tensors ? p.start[k + 1] : p.psi_pad);

  // Layers: maximal runs of one id, spanning their tensors' padded slots.
  for (int32_t k = 0; k < n_tensors;) {
    int32_t j = k;
    while (j + 1 < n_tensors && layer_id[j + 1] == layer_id[k]) ++j;
    p.layers.push_back({layer_id[k], p.start[k], p.slot_end[j]});
    p.max_layer = std::max(p.max_layer, p.slot_end[j] - p.start[k]);
    k = j + 1;
  }

  // Bucket schedule, last tensor to first; 0 = one bucket spanning the padded
  // flat space.
  if (bucket_elems == 0) p.bucket_elems = p.psi_pad;
  const int64_t B = p.bucket_elems;
  bool open = false;
  Span cur{0, 0};
  for (int32_t k = n_tensors - 1; k >= 0; --k) {
    const int64_t a = p.start[k], b = p.slot_end[k];
    if (b == a) continue;
    if (b - a > B) {
      if (open) p.buckets.push_back(cur);
      open = false;
      int64_t e = b;
      for (; e - a > B; e -= B) p.buckets.push_back({e - B, e});
      p.buckets.push_back({a, e});
    } else if (open && (cur.hi - cur.lo) + (b - a) <= B) {
      cur.lo = a;
    } else {
      if (open) p.buckets.push_back(cur);
      cur = {a, b};
      open = true;
    }
  }
  if (open) p.buckets.push_back(cur);
  for (const Span& s : p.buckets) p.max_bucket = std::max(p.max_bucket, s.hi - s.lo);
  *out = std::move(p);
  return true;
}

}  // namespace zsm
