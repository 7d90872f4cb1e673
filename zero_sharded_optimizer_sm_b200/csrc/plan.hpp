// Flat layout, ownership partition and schedules of a ZeRO context (host only).
//
// Partition ("ZERO训练技术", section "ZeRO-1", the part on how optimizer states
// are split): the parameter vector is cut into N contiguous segments, rank r
// owns segment r.  Layout choices of this library: tensors laid end to end in
// list order, each starting on a multiple of 8 elements (one 16-byte bf16
// vector), total padded to a multiple of 8*N so the N segments are equal.
//
// Bucket schedule ("ZeRO：从优化器状态到残差状态的显存优化", section 3.3 "CB";
// "ZERO训练技术", section "ZeRO-2", part "2. 反向"): gradients appear from the
// last layer back, so tensors are visited last to first and packed into one
// interval while it stays within the fixed buffer; a tensor that does not fit
// closes the interval; a tensor larger than the buffer is cut into
// buffer-sized chunks from its end, each its own interval.
#pragma once

#include <cstdint>
#include <string>
#include <vector>

namespace zsm {

constexpr int64_t kGranule = 8;

struct Span {
  int64_t lo, hi;
};

struct LayerSpan {
  int32_t id;
  int64_t lo, hi;
};

struct Plan {
  int32_t n_ranks = 0;
  int64_t bucket_elems = 0;
  std::vector<int64_t> numel;
  std::vector<int32_t> layer_id;
  std::vector<int64_t> start;     // flat start of each tensor
  std::vector<int64_t> slot_end;  // end of each tensor's padded slot (next start / psi_pad)
  int64_t psi = 0, psi_pad = 0, shard = 0, max_layer = 0, max_bucket = 0;
  std::vector<Span> buckets;      // schedule order (descending addresses)
  std::vector<LayerSpan> layers;  // layer order

  int32_t owner(int64_t i) const { return (int32_t)(i / shard); }
  // Index of the layer containing flat element i (binary search).
  int layer_of(int64_t i) const;
};

// Builds the plan; returns false with a message on invalid input.
bool make_plan(int32_t n_tensors, const int64_t* numel, const int32_t* layer_id, int32_t n_ranks,
               int64_t bucket_elems, Plan* out, std::string* err);

}  // namespace zsm
