// The clipped step's two passes with bulk stores (two_pass_tma.cu).
#pragma once

#include <cuda_runtime.h>

#include "kernels.cuh"

namespace zsm {

// Pass 2 with bulk stores (two_pass_tma.cu): 1024-element tiles, eight
// consumer warps, a ring of `stages` (2..8, fitted to shared memory); the
// stores carry the L2 evict-first hint when `store_hint`.
cudaError_t launch_adam_bcast_bulk(const AdamBcastArgs& a, int grid, bool uniform, int stages, int store_hint,
                                   cudaStream_t s);
int64_t bulk_bcast_tile();
// Pass 1 with bulk stores (two_pass_tma.cu), N <= 16: 1024-element tiles,
// eight consumer warps, a ring of `stages` (fitted to shared memory).
cudaError_t launch_reduce_bulk(const ReduceArgs& a, int grid, int stages, int store_hint, cudaStream_t s);
// Pass 2 over every layer of a stage-3 step in one cooperative launch (`a`
// at flat element 0, its destinations at the layer buffers' start; `g` the
// layers in schedule order and the zeroed arrival counter).  Returns
// cudaErrorCooperativeLaunchTooLarge, launching nothing, when the device
// cannot hold every CTA at once.
cudaError_t launch_adam_bcast_bulk_layered(const AdamBcastArgs& a, const SegTable& g, int grid, bool uniform,
                                           int stages, int store_hint, cudaStream_t s);

}  // namespace zsm
