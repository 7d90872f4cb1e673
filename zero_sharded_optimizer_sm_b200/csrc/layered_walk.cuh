// Tile walk and store ordering of the layered stage-3 launches, which run a
// stage-3 step's layers in one cooperative launch (fused_bulk.cu: the fused
// step; two_pass_tma.cu: the clipped step's second pass).
//
// Every layer writes the one set of temporary layer buffers.  A CTA walks
// its tiles layer after layer in the schedule's order (tiles blockIdx.x,
// blockIdx.x + G, ... of each layer in turn); its storer issues a layer's
// stores only after every CTA has finished storing the layers before it, so
// the buffers receive the layers in the order of one launch per layer.
#pragma once

#include <cuda_runtime.h>

#include "kernels.cuh"
#include "tma_pipe.cuh"

namespace zsm {
namespace pipe {

// ------------------------------------------------------------ tile walk --
//
// A CTA's tiles in launch order.  One interval: tiles blockIdx.x,
// blockIdx.x + G, ... of [0, n_elem).  Layered (a stage-3 step's layers in one
// launch): the same walk through each segment in turn.  e_src is the tile's
// flat start (gradients, states, shards), e_dst its offset in the N
// destination buffers (the same for one interval; from the layer's start for
// a segment).
struct TileCursor {
  int seg = 0;      // segment of the current tile
  long long t = -1; // tile index inside the segment (-1: before the first)
};

template <int T, bool kLayered>
__device__ __forceinline__ bool cursor_next(TileCursor& c, const SegTable& g, long long n_tiles, long long n_elem,
                                            long long& e_src, long long& e_dst, unsigned& cnt) {
  c.t = c.t < 0 ? (long long)blockIdx.x : c.t + gridDim.x;
  long long rest;
  if constexpr (kLayered) {
    while (c.seg < g.n && c.t * T >= g.len[c.seg]) {
      ++c.seg;
      c.t = blockIdx.x;
    }
    if (c.seg >= g.n) return false;
    e_dst = c.t * T;
    e_src = g.lo[c.seg] + e_dst;
    rest = g.len[c.seg] - e_dst;
  } else {
    if (c.t >= n_tiles) return false;
    e_dst = e_src = c.t * T;
    rest = n_elem - e_src;
  }
  cnt = (unsigned)(rest < T ? rest : T);
  return true;
}

// The layered storers' ordering: a storer that has finished a segment's
// stores waits until their global writes are performed, orders them before
// its generic release (proxy fence) and arrives on the counter; a storer
// about to store segment k waits until all G CTAs have arrived k times and
// orders its bulk stores after that acquire.
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

__device__ __forceinline__ void segment_arrive(unsigned* counter) {
  bulk_wait<0>();
  fence_proxy_async_global();
  asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(counter) : "memory");
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Bounded like the ring waits (limit 0: one test); false when it ran out or
// the CTA aborted.
__device__ __forceinline__ bool segment_wait(const unsigned* counter, unsigned target, volatile int* abort_flag,
                                             unsigned long long limit) {
  bool ok = ld_acquire_gpu(counter) >= target;
  if (!ok && limit > 0) {
    const unsigned long long t0 = now_ns();
    while (!(ok = ld_acquire_gpu(counter) >= target)) {
      if (*abort_flag || now_ns() - t0 > limit) break;
      __nanosleep(32);
    }
  }
  if (ok) fence_proxy_async_global();
  return ok;
}

}  // namespace pipe
}  // namespace zsm
