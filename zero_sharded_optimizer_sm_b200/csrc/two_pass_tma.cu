// The two passes of the clipped / overflow-checked step with their inputs
// staged through shared memory by the Tensor Memory Accelerator (sm_100a).  Same arithmetic, in the same order, as reduce_kernel and
// adam_bcast_kernel in kernels.cu; different data movement, as in the fused
// staged kernel: one persistent CTA per SM, warp 0's elected lane streams each
// 2048-element tile into a ring of shared-memory stages with 1-D bulk copies
// (completion counted in bytes on an mbarrier), eight consumer warps take
// their 8 elements from shared memory, release the stage and store.
//
// Pass 1 (reduce_tma_kernel): the tile's N gradient slices; the consumers add
//   them in rank order, take the 1/N mean, store it into the reduced-gradient
//   shard (stages 2, 3) or back into every replica (stage 1, the all-reduce)
//   and accumulate the gradient norm.
// Pass 2 (adam_bcast_tma_kernel): the owners' reduced gradient and the fp32
//   master, m, v; the consumers run Adam with the loss-scale and clipping
//   factors and store the 16-bit result to every destination.
//
// Every wait is bounded (kWaitNs); one that runs out records an error code,
// stops the producer, drains the copies in flight and ends the CTA.
//
// The passes compute the reduce-scatter / all-reduce and the update +
// all-gather of "ZERO训练技术" sections "ZeRO-1" to "ZeRO-3"; the split into
// two passes is for the global-norm clip and the overflow skip, which are not
// on the pages (both need the whole step's norm before any update).
#include <cuda_runtime.h>

#include <algorithm>

#include "device_math.cuh"
#include "kernels.cuh"
#include "two_pass_bulk.cuh"
#include "tma_pipe.cuh"
#include "layered_walk.cuh"

namespace zsm {
namespace {

using namespace dev;
using namespace pipe;

constexpr int kTpThreads = tma_threads<1>();  // one producer warp + 8 consumer warps
constexpr int kTpStages = 4;                  // ring depth of both passes

__host__ __device__ inline unsigned reduce_stage_bytes(int n_ranks) { return (unsigned)(kTile * 2 * n_ranks); }
// pass 2 stage: [16-bit gradient, 2 B][master, 4 B][m, 4 B][v, 4 B] per element
constexpr unsigned kBcastStageBytes = kTile * 14;

// [stages x stage_bytes][full[stages]][empty[stages]][abort][last_k[stages]]
inline size_t tp_smem_bytes(unsigned stage_bytes, int stages) {
  return (size_t)stages * stage_bytes + 2 * stages * sizeof(uint64_t) + 4 * (stages + 1);
}

struct Ring {
  uint64_t* full;
  uint64_t* empty;
  volatile int* abort_flag;
  volatile int* last_k;
};

__device__ __forceinline__ Ring ring_at(unsigned char* smem, unsigned stage_bytes, int stages) {
  Ring r;
  r.full = reinterpret_cast<uint64_t*>(smem + (size_t)stages * stage_bytes);
  r.empty = r.full + stages;
  r.abort_flag = reinterpret_cast<volatile int*>(r.empty + stages);
  r.last_k = r.abort_flag + 1;
  return r;
}

__device__ __forceinline__ void ring_init(const Ring& r, int stages) {
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&r.full[s], 1);
      mbar_init(&r.empty[s], kConsumerWarps);
      r.last_k[s] = -1;
    }
    *r.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
}

// After the CTA's loops: with an abort, wait (bounded) for the copies already
// issued before the CTA's shared memory goes away.
__device__ __forceinline__ void ring_drain(const Ring& r, int stages, unsigned int* error) {
  __syncthreads();
  if (*r.abort_flag && threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s)
      if (r.last_k[s] >= 0 && !mbar_wait(&r.full[s], (unsigned)r.last_k[s] & 1u)) atomicOr(error, 4u);
  }
}

// Producer side of one ring slot: wait for the consumers to release stage
// `s` (phase k - 1); false (abort recorded) when the wait runs out.
__device__ __forceinline__ bool acquire_stage(const Ring& r, int s, unsigned k, unsigned int* error,
                                              unsigned long long limit) {
  if (k > 0 && !mbar_wait(&r.empty[s], (k - 1) & 1u, limit)) {
    atomicOr(error, 1u);
    *r.abort_flag = 1;
    return false;
  }
  fence_proxy_async_smem();  // the consumers' reads of this stage before the copies refill it
  return true;
}

// Consumer side: wait (warp-uniformly) for stage `s` phase k; false to stop.
__device__ __forceinline__ bool consume_stage(const Ring& r, int s, unsigned k, unsigned int* error, int lane,
                                              unsigned long long limit) {
  const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(&r.full[s], k & 1u, limit));
  if (!ok) {
    if (lane == 0) atomicOr(error, 2u);
    *r.abort_flag = 1;
    return false;
  }
  return !__any_sync(0xFFFFFFFFu, *r.abort_flag != 0);
}

// -------------------------------------------------------------- pass 1 --

template <bool kWriteBack, class F>
__global__ void __launch_bounds__(kTpThreads, 1)
    reduce_tma_kernel(const __grid_constant__ ReduceArgs a, int stages) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int N = a.n_ranks;
  const unsigned stage_bytes = reduce_stage_bytes(N);
  const Ring ring = ring_at(smem, stage_bytes, stages);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_elem = a.n_vec * kVec;
  const int64_t n_tiles = (n_elem + kTile - 1) / kTile;
  ring_init(ring, stages);

  double sq = 0.0;
  unsigned long long nf = 0;
  if (warp == 0) {
    if (lane == 0) {
      const uint64_t policy = evict_first_policy();
      for (int it = 0;; ++it) {
        const int64_t tile = blockIdx.x + (int64_t)it * gridDim.x;
        if (tile >= n_tiles || *ring.abort_flag) break;
        const int s = it % stages;
        const unsigned k = (unsigned)(it / stages);
        if (!acquire_stage(ring, s, k, a.ns.error, a.ns.wait_ns)) break;
        const int64_t e0 = tile * kTile;
        const int64_t cnt = (n_elem - e0) < kTile ? (n_elem - e0) : kTile;
        unsigned char* st = smem + (size_t)s * stage_bytes;
        mbar_expect_tx(&ring.full[s], (unsigned)(cnt * 2 * N));
        for (int r = 0; r < N; ++r)
          bulk_load(st + (size_t)r * 2 * kTile, a.grad[r] + e0, (unsigned)(2 * cnt), &ring.full[s], policy);
        ring.last_k[s] = (int)k;
      }
    }
  } else {
    const int j = (threadIdx.x - 32) * kVec;
    for (int it = 0;; ++it) {
      const int64_t tile = blockIdx.x + (int64_t)it * gridDim.x;
      if (tile >= n_tiles) break;
      const int s = it % stages;
      const unsigned k = (unsigned)(it / stages);
      if (!consume_stage(ring, s, k, a.ns.error, lane, a.ns.wait_ns)) break;
      const int64_t e0 = tile * kTile;
      const int64_t cnt = (n_elem - e0) < kTile ? (n_elem - e0) : kTile;
      const unsigned char* st = smem + (size_t)s * stage_bytes;
      const bool active = j < cnt;  // the last tile may be ragged
      float acc[kVec];
      if (active) {
#pragma unroll
        for (int q = 0; q < kVec; ++q) acc[q] = 0.0f;
        for (int r = 0; r < N; ++r) add8<F>(acc, *reinterpret_cast<const uint4*>(st + (size_t)r * 2 * kTile + 2 * j));
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ring.empty[s]);
      if (active) {
        const int64_t e = e0 + j;
        uint16_t g16[kVec];
        float g[kVec];
        mean_bf16<F>(acc, a.inv_n, g16, g, sq, nf);
        const uint4 gw = pack8(g16);
        if (kWriteBack) {
          for (int r = 0; r < N; ++r) st_out(const_cast<uint16_t*>(a.grad[r]) + e, gw);
        } else {
          st_out(a.shard_out + e, gw);
        }
      }
    }
  }
  ring_drain(ring, stages, a.ns.error);
  norm_epilogue<kTpThreads>(a.ns, sq, nf, a.accumulate);
}

// Pass 1 with bulk stores (N <= 16): the consumers add the tile's N slices
// in rank order and write the rounded mean over rank 0's slice in the stage
// (each lane over the elements it alone read); a storer warp's elected lane
// copies it out with bulk stores -- to the reduced-gradient shard, or back to
// all N replicas (the all-reduce) -- and releases the stage once the copies
// have read it.  Tiles of 1024 elements, eight consumer warps.
constexpr int kBulkRedTile = 1024;
constexpr int kBulkRedWarps = 8;
constexpr int kBulkRedThreads = 32 * (kBulkRedWarps + 2);

inline size_t bulk_reduce_smem_bytes(int n_ranks, int stages) {
  return (size_t)stages * (size_t)(2 * n_ranks * kBulkRedTile) + 3 * (size_t)stages * sizeof(uint64_t) +
         4 * (size_t)(stages + 1);
}

template <bool kWriteBack, class F>
__global__ void __launch_bounds__(kBulkRedThreads, 1)
    reduce_bulk_kernel(const __grid_constant__ ReduceArgs a, int stages, int store_hint) {
  constexpr int T = kBulkRedTile;
  constexpr int W = kBulkRedWarps;
  constexpr int EPT = T / (32 * W);
  static_assert(EPT == 4, "four elements per consumer lane");
  extern __shared__ __align__(128) unsigned char smem[];
  const int N = a.n_ranks;
  const unsigned sb = (unsigned)(2 * N * T);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)stages * sb);
  uint64_t* computed = full + stages;
  uint64_t* empty = computed + stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + stages);
  volatile int* last_k = abort_flag + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_elem = a.n_vec * kVec;
  const int64_t n_tiles = (n_elem + T - 1) / T;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&computed[s], W);
      mbar_init(&empty[s], 1);
      last_k[s] = -1;
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  double sq = 0.0;
  unsigned long long nf = 0;
  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      const uint64_t policy = evict_first_policy();
      for (int it = 0;; ++it) {
        const int64_t tile = blockIdx.x + (int64_t)it * gridDim.x;
        if (tile >= n_tiles || *abort_flag) break;
        const int s = it % stages;
        const unsigned k = (unsigned)(it / stages);
        if (k > 0) {
          const int w = mbar_wait_or_abort(&empty[s], (k - 1) & 1u, abort_flag, a.ns.wait_ns);
          if (w != 0) {
            if (w == 1) atomicOr(a.ns.error, 1u);
            *abort_flag = 1;
            break;
          }
        }
        fence_proxy_async_smem();
        const int64_t e0 = tile * T;
        const int64_t cnt = (n_elem - e0) < T ? (n_elem - e0) : T;
        unsigned char* st = smem + (size_t)s * sb;
        mbar_expect_tx(&full[s], (unsigned)(cnt * 2 * N));
        for (int r = 0; r < N; ++r)
          bulk_load(st + (size_t)r * 2 * T, a.grad[r] + e0, (unsigned)(2 * cnt), &full[s], policy);
        last_k[s] = (int)k;
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------- storer --
    if (lane == 0) {
      const uint64_t spol = evict_first_policy();
      auto put = [&](void* dst, const void* src, unsigned bytes) {
        if (store_hint) bulk_store(dst, src, bytes, spol);
        else bulk_store(dst, src, bytes);
      };
      for (int it = 0;; ++it) {
        const int64_t tile = blockIdx.x + (int64_t)it * gridDim.x;
        if (tile >= n_tiles) break;
        const int s = it % stages;
        const unsigned k = (unsigned)(it / stages);
        const int w = mbar_wait_or_abort(&computed[s], k & 1u, abort_flag, a.ns.wait_ns);
        if (w != 0) {
          if (w == 1) atomicOr(a.ns.error, 8u);
          *abort_flag = 1;
          break;
        }
        const int64_t e0 = tile * T;
        const unsigned cnt = (unsigned)((n_elem - e0) < T ? (n_elem - e0) : T);
        const unsigned char* st = smem + (size_t)s * sb;
        if (kWriteBack) {
          for (int r = 0; r < N; ++r) put(const_cast<uint16_t*>(a.grad[r]) + e0, st, 2 * cnt);
        } else {
          put(a.shard_out + e0, st, 2 * cnt);
        }
        bulk_commit();
        bulk_wait_read<0>();  // the copies have read the stage: hand it back to the producer
        mbar_arrive(&empty[s]);
      }
      bulk_wait<0>();  // every store of this CTA performed before the CTA ends
    }
  } else {
    // ----------------------------------------------------------- consumers --
    const int j = (threadIdx.x - 64) * EPT;
    for (int it = 0;; ++it) {
      const int64_t tile = blockIdx.x + (int64_t)it * gridDim.x;
      if (tile >= n_tiles) break;
      const int s = it % stages;
      const unsigned k = (unsigned)(it / stages);
      const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(&full[s], k & 1u, a.ns.wait_ns));
      if (!ok) {
        if (lane == 0) atomicOr(a.ns.error, 2u);
        *abort_flag = 1;
        break;
      }
      if (__any_sync(0xFFFFFFFFu, *abort_flag != 0)) break;
      const int64_t e0 = tile * T;
      const int64_t cnt = (n_elem - e0) < T ? (n_elem - e0) : T;
      unsigned char* st = smem + (size_t)s * sb;
      if (j < cnt) {  // cnt is a multiple of 8, so a lane's four elements are whole
        float acc[EPT] = {0.0f, 0.0f, 0.0f, 0.0f};
        for (int r = 0; r < N; ++r) {
          const uint2 w2 = *reinterpret_cast<const uint2*>(st + (size_t)r * 2 * T + 2 * j);
          acc[0] = __fadd_rn(acc[0], F::lo(w2.x));
          acc[1] = __fadd_rn(acc[1], F::hi(w2.x));
          acc[2] = __fadd_rn(acc[2], F::lo(w2.y));
          acc[3] = __fadd_rn(acc[3], F::hi(w2.y));
        }
        uint16_t g16[EPT];
#pragma unroll
        for (int q = 0; q < EPT; ++q) {
          g16[q] = F::rn(__fmul_rn(acc[q], a.inv_n));
          const float g = F::f32(g16[q]);
          const double d = (double)g;
          sq = __dadd_rn(sq, __dmul_rn(d, d));  // each square exact (at most 11-bit significands)
          nf += isfinite(g) ? 0ull : 1ull;
        }
        *reinterpret_cast<uint2*>(st + 2 * j) = make_uint2(pack2(g16[0], g16[1]), pack2(g16[2], g16[3]));
      }
      fence_proxy_async_smem();  // this lane's stage writes before the storer's bulk copies read them
      __syncwarp();
      if (lane == 0) mbar_arrive(&computed[s]);
    }
  }
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s)
      if (last_k[s] >= 0 && !mbar_wait(&full[s], (unsigned)last_k[s] & 1u)) atomicOr(a.ns.error, 4u);
  }
  norm_epilogue<kBulkRedThreads>(a.ns, sq, nf, a.accumulate);
}

// Pass 1 above 16 ranks: a tile's N slices do not fit a stage, so the
// producer streams them in chunks of kChunk ranks (32 KB stages) and the
// consumers add each chunk in rank order -- the same sequence of additions.
constexpr int kChunk = 8;
constexpr unsigned kChunkStageBytes = kChunk * 2 * kTile;

template <bool kWriteBack, class F>
__global__ void __launch_bounds__(kTpThreads, 1)
    reduce_chunked_tma_kernel(const __grid_constant__ ReduceArgs a, int stages) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int N = a.n_ranks;
  const int n_chunks = (N + kChunk - 1) / kChunk;
  const Ring ring = ring_at(smem, kChunkStageBytes, stages);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_elem = a.n_vec * kVec;
  const int64_t n_tiles = (n_elem + kTile - 1) / kTile;
  ring_init(ring, stages);

  double sq = 0.0;
  unsigned long long nf = 0;
  if (warp == 0) {
    if (lane == 0) {
      const uint64_t policy = evict_first_policy();
      bool stop = false;
      for (int it = 0; !stop; ++it) {
        const int64_t tile = blockIdx.x + (int64_t)it * gridDim.x;
        if (tile >= n_tiles || *ring.abort_flag) break;
        const int64_t e0 = tile * kTile;
        const int64_t cnt = (n_elem - e0) < kTile ? (n_elem - e0) : kTile;
        for (int c = 0; c < n_chunks; ++c) {
          const int ci = it * n_chunks + c;
          const int s = ci % stages;
          const unsigned k = (unsigned)(ci / stages);
          if (!acquire_stage(ring, s, k, a.ns.error, a.ns.wait_ns)) {
            stop = true;
            break;
          }
          const int r0 = c * kChunk;
          const int r1 = (r0 + kChunk) < N ? (r0 + kChunk) : N;
          unsigned char* st = smem + (size_t)s * kChunkStageBytes;
          mbar_expect_tx(&ring.full[s], (unsigned)(cnt * 2 * (r1 - r0)));
          for (int r = r0; r < r1; ++r)
            bulk_load(st + (size_t)(r - r0) * 2 * kTile, a.grad[r] + e0, (unsigned)(2 * cnt), &ring.full[s], policy);
          ring.last_k[s] = (int)k;
        }
      }
    }
  } else {
    const int j = (threadIdx.x - 32) * kVec;
    bool stop = false;
    for (int it = 0; !stop; ++it) {
      const int64_t tile = blockIdx.x + (int64_t)it * gridDim.x;
      if (tile >= n_tiles) break;
      const int64_t e0 = tile * kTile;
      const int64_t cnt = (n_elem - e0) < kTile ? (n_elem - e0) : kTile;
      const bool active = j < cnt;
      float acc[kVec];
#pragma unroll
      for (int q = 0; q < kVec; ++q) acc[q] = 0.0f;
      for (int c = 0; c < n_chunks; ++c) {
        const int ci = it * n_chunks + c;
        const int s = ci % stages;
        const unsigned k = (unsigned)(ci / stages);
        if (!consume_stage(ring, s, k, a.ns.error, lane, a.ns.wait_ns)) {
          stop = true;
          break;
        }
        const int r0 = c * kChunk;
        const int r1 = (r0 + kChunk) < N ? (r0 + kChunk) : N;
        const unsigned char* st = smem + (size_t)s * kChunkStageBytes;
        if (active)
          for (int r = r0; r < r1; ++r)
            add8<F>(acc, *reinterpret_cast<const uint4*>(st + (size_t)(r - r0) * 2 * kTile + 2 * j));
        __syncwarp();
        if (lane == 0) mbar_arrive(&ring.empty[s]);
      }
      if (stop) break;
      if (active) {
        const int64_t e = e0 + j;
        uint16_t g16[kVec];
        float g[kVec];
        mean_bf16<F>(acc, a.inv_n, g16, g, sq, nf);
        const uint4 gw = pack8(g16);
        if (kWriteBack) {
          for (int r = 0; r < N; ++r) st_out(const_cast<uint16_t*>(a.grad[r]) + e, gw);
        } else {
          st_out(a.shard_out + e, gw);
        }
      }
    }
  }
  ring_drain(ring, stages, a.ns.error);
  norm_epilogue<kTpThreads>(a.ns, sq, nf, a.accumulate);
}

// -------------------------------------------------------------- pass 2 --

// gsrc[r] are flat-element-0 pointers; element i's reduced gradient is read
// from its owner's copy, gsrc[i / shard] (all the same pointer when the
// owners' copies are the one reduced-gradient shard array: `uniform`).
template <class F>
__global__ void __launch_bounds__(kTpThreads, 1)
    adam_bcast_tma_kernel(const __grid_constant__ AdamBcastArgs a, int stages, int uniform) {
  extern __shared__ __align__(128) unsigned char smem[];
  const Ring ring = ring_at(smem, kBcastStageBytes, stages);
  AdamScalars sc = a.sc_dev ? *a.sc_dev : a.sc;
  const bool skip = apply_decision(a.dec, sc);  // a skipped step writes the unchanged parameters only
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_elem = a.n_vec * kVec;
  const int64_t n_tiles = (n_elem + kTile - 1) / kTile;
  ring_init(ring, stages);

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t policy = evict_first_policy();
      for (int it = 0;; ++it) {
        const int64_t tile = blockIdx.x + (int64_t)it * gridDim.x;
        if (tile >= n_tiles || *ring.abort_flag) break;
        const int s = it % stages;
        const unsigned k = (unsigned)(it / stages);
        if (!acquire_stage(ring, s, k, a.error, a.wait_ns)) break;
        const int64_t e0 = tile * kTile;
        const int64_t cnt = (n_elem - e0) < kTile ? (n_elem - e0) : kTile;
        unsigned char* st = smem + (size_t)s * kBcastStageBytes;
        mbar_expect_tx(&ring.full[s], (unsigned)(cnt * 14));
        const int64_t i0 = a.lo + e0;  // flat index of the tile's first element
        if (uniform) {
          bulk_load(st, a.gsrc[0] + i0, (unsigned)(2 * cnt), &ring.full[s], policy);
        } else {
          // one copy per owner: owners change every `shard` elements (a multiple of 8)
          for (int64_t e = 0; e < cnt;) {
            const int64_t owner = (i0 + e) / a.shard;
            const int64_t next = (owner + 1) * a.shard - i0;
            const int64_t end = next < cnt ? next : cnt;
            bulk_load(st + 2 * e, a.gsrc[owner] + i0 + e, (unsigned)(2 * (end - e)), &ring.full[s], policy);
            e = end;
          }
        }
        unsigned char* stt = st + 2 * kTile;
        bulk_load(stt, a.master + e0, (unsigned)(4 * cnt), &ring.full[s], policy);
        bulk_load(stt + 4 * kTile, a.m + e0, (unsigned)(4 * cnt), &ring.full[s], policy);
        bulk_load(stt + 8 * kTile, a.v + e0, (unsigned)(4 * cnt), &ring.full[s], policy);
        ring.last_k[s] = (int)k;
      }
    }
  } else {
    const int j = (threadIdx.x - 32) * kVec;
    for (int it = 0;; ++it) {
      const int64_t tile = blockIdx.x + (int64_t)it * gridDim.x;
      if (tile >= n_tiles) break;
      const int s = it % stages;
      const unsigned k = (unsigned)(it / stages);
      if (!consume_stage(ring, s, k, a.error, lane, a.wait_ns)) break;
      const int64_t e0 = tile * kTile;
      const int64_t cnt = (n_elem - e0) < kTile ? (n_elem - e0) : kTile;
      const unsigned char* st = smem + (size_t)s * kBcastStageBytes;
      const bool active = j < cnt;
      float4 p0, p1, m0, m1, v0, v1;
      uint4 gw;
      if (active) {
        gw = *reinterpret_cast<const uint4*>(st + 2 * j);
        const float* stt = reinterpret_cast<const float*>(st + 2 * kTile);
        p0 = *reinterpret_cast<const float4*>(stt + j);
        p1 = *reinterpret_cast<const float4*>(stt + j + 4);
        m0 = *reinterpret_cast<const float4*>(stt + kTile + j);
        m1 = *reinterpret_cast<const float4*>(stt + kTile + j + 4);
        v0 = *reinterpret_cast<const float4*>(stt + 2 * kTile + j);
        v1 = *reinterpret_cast<const float4*>(stt + 2 * kTile + j + 4);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ring.empty[s]);
      if (active && skip) {
        const int64_t e = e0 + j;
        const uint4 pw = round8<F>(p0, p1);
        if (a.param_shard) st_out(a.param_shard + e, pw);
        for (int r = 0; r < a.n_out; ++r) st_out(a.out[r] + e, pw);
      } else if (active) {
        const int64_t e = e0 + j;
        float g[kVec] = {F::lo(gw.x), F::hi(gw.x), F::lo(gw.y), F::hi(gw.y),
                         F::lo(gw.z), F::hi(gw.z), F::lo(gw.w), F::hi(gw.w)};
        uint16_t p16[kVec];
        adam8<F>(g, p0, p1, m0, m1, v0, v1, sc, p16);  // loss-scale and clip factors via sc.flags
        st_out(a.master + e, p0);
        st_out(a.master + e + 4, p1);
        st_out(a.m + e, m0);
        st_out(a.m + e + 4, m1);
        st_out(a.v + e, v0);
        st_out(a.v + e + 4, v1);
        const uint4 pw = pack8(p16);
        if (a.param_shard) st_out(a.param_shard + e, pw);
        for (int r = 0; r < a.n_out; ++r) st_out(a.out[r] + e, pw);
      }
    }
  }
  ring_drain(ring, stages, a.error);
}

// ------------------------------------------------- pass 2, bulk stores --
//
// The same pass with the results leaving through the Tensor Memory
// Accelerator as in the fused bulk-store kernel (fused_bulk.cu): the
// consumers write the updated master/m/v back into the stage and the 16-bit
// parameters over the stage's gradient slice, fence the async proxy and
// arrive on `computed`; a storer warp's elected lane copies the stage out with
// bulk stores -- master/m/v (not on a skipped step, which leaves them
// unchanged), the parameter shard at stage 3 and the N destinations -- then
// waits until the copies have read the stage and releases it.  A consumer
// lane issues no global store.  Tiles of T elements, W consumer warps.
constexpr int kBulkBcastTile = 1024;
constexpr int kBulkBcastWarps = 8;
constexpr int kBulkBcastThreads = 32 * (kBulkBcastWarps + 2);
constexpr unsigned kBulkBcastStageBytes = kBulkBcastTile * 14;  // [g 2T][master 4T][m 4T][v 4T]

inline size_t bulk_bcast_smem_bytes(int stages) {
  return (size_t)stages * kBulkBcastStageBytes + 3 * (size_t)stages * sizeof(uint64_t) + 4 * (size_t)(stages + 1);
}

template <class F>
__global__ void __launch_bounds__(kBulkBcastThreads, 1)
    adam_bcast_bulk_kernel(const __grid_constant__ AdamBcastArgs a, int stages, int uniform, int store_hint) {
  constexpr int T = kBulkBcastTile;
  constexpr int W = kBulkBcastWarps;
  constexpr int EPT = T / (32 * W);
  static_assert(EPT == 4, "four elements per consumer lane");
  extern __shared__ __align__(128) unsigned char smem[];
  const unsigned sb = kBulkBcastStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)stages * sb);
  uint64_t* computed = full + stages;
  uint64_t* empty = computed + stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + stages);
  volatile int* last_k = abort_flag + 1;
  AdamScalars sc = a.sc_dev ? *a.sc_dev : a.sc;
  const bool skip = apply_decision(a.dec, sc);  // a skipped step writes the unchanged parameters only
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_elem = a.n_vec * kVec;
  const int64_t n_tiles = (n_elem + T - 1) / T;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&computed[s], W);
      mbar_init(&empty[s], 1);
      last_k[s] = -1;
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      const uint64_t policy = evict_first_policy();
      for (int it = 0;; ++it) {
        const int64_t tile = blockIdx.x + (int64_t)it * gridDim.x;
        if (tile >= n_tiles || *abort_flag) break;
        const int s = it % stages;
        const unsigned k = (unsigned)(it / stages);
        if (k > 0) {
          const int w = mbar_wait_or_abort(&empty[s], (k - 1) & 1u, abort_flag, a.wait_ns);
          if (w != 0) {
            if (w == 1) atomicOr(a.error, 1u);
            *abort_flag = 1;
            break;
          }
        }
        fence_proxy_async_smem();  // the stage's last reads (consumers, stores) before the refill
        const int64_t e0 = tile * T;
        const int64_t cnt = (n_elem - e0) < T ? (n_elem - e0) : T;
        unsigned char* st = smem + (size_t)s * sb;
        mbar_expect_tx(&full[s], (unsigned)(cnt * 14));
        const int64_t i0 = a.lo + e0;  // flat index of the tile's first element
        if (uniform) {
          bulk_load(st, a.gsrc[0] + i0, (unsigned)(2 * cnt), &full[s], policy);
        } else {
          // one copy per owner: owners change every `shard` elements (a multiple of 8)
          for (int64_t e = 0; e < cnt;) {
            const int64_t owner = (i0 + e) / a.shard;
            const int64_t next = (owner + 1) * a.shard - i0;
            const int64_t end = next < cnt ? next : cnt;
            bulk_load(st + 2 * e, a.gsrc[owner] + i0 + e, (unsigned)(2 * (end - e)), &full[s], policy);
            e = end;
          }
        }
        bulk_load(st + 2 * T, a.master + e0, (unsigned)(4 * cnt), &full[s], policy);
        bulk_load(st + 6 * T, a.m + e0, (unsigned)(4 * cnt), &full[s], policy);
        bulk_load(st + 10 * T, a.v + e0, (unsigned)(4 * cnt), &full[s], policy);
        last_k[s] = (int)k;
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------- storer --
    if (lane == 0) {
      const uint64_t spol = evict_first_policy();
      auto put = [&](void* dst, const void* src, unsigned bytes) {
        if (store_hint) bulk_store(dst, src, bytes, spol);
        else bulk_store(dst, src, bytes);
      };
      for (int it = 0;; ++it) {
        const int64_t tile = blockIdx.x + (int64_t)it * gridDim.x;
        if (tile >= n_tiles) break;
        const int s = it % stages;
        const unsigned k = (unsigned)(it / stages);
        const int w = mbar_wait_or_abort(&computed[s], k & 1u, abort_flag, a.wait_ns);
        if (w != 0) {
          if (w == 1) atomicOr(a.error, 8u);
          *abort_flag = 1;
          break;
        }
        const int64_t e0 = tile * T;
        const unsigned cnt = (unsigned)((n_elem - e0) < T ? (n_elem - e0) : T);
        const unsigned char* st = smem + (size_t)s * sb;
        if (!skip) {
          put(a.master + e0, st + 2 * T, 4 * cnt);
          put(a.m + e0, st + 6 * T, 4 * cnt);
          put(a.v + e0, st + 10 * T, 4 * cnt);
        }
        if (a.param_shard) put(a.param_shard + e0, st, 2 * cnt);
        for (int r = 0; r < a.n_out; ++r) put(a.out[r] + e0, st, 2 * cnt);
        bulk_commit();
        bulk_wait_read<0>();  // the copies have read the stage: hand it back to the producer
        mbar_arrive(&empty[s]);
      }
      bulk_wait<0>();  // every store of this CTA performed before the CTA ends
    }
  } else {
    // ----------------------------------------------------------- consumers --
    const int j = (threadIdx.x - 64) * EPT;
    for (int it = 0;; ++it) {
      const int64_t tile = blockIdx.x + (int64_t)it * gridDim.x;
      if (tile >= n_tiles) break;
      const int s = it % stages;
      const unsigned k = (unsigned)(it / stages);
      const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(&full[s], k & 1u, a.wait_ns));
      if (!ok) {
        if (lane == 0) atomicOr(a.error, 2u);
        *abort_flag = 1;
        break;
      }
      if (__any_sync(0xFFFFFFFFu, *abort_flag != 0)) break;
      const int64_t e0 = tile * T;
      const int64_t cnt = (n_elem - e0) < T ? (n_elem - e0) : T;
      unsigned char* st = smem + (size_t)s * sb;
      if (j < cnt) {  // cnt is a multiple of 8, so a lane's four elements are whole
        float4 p = *reinterpret_cast<const float4*>(st + 2 * T + 4 * j);
        float4 m = *reinterpret_cast<const float4*>(st + 6 * T + 4 * j);
        float4 v = *reinterpret_cast<const float4*>(st + 10 * T + 4 * j);
        uint2 pw;
        if (skip) {
          pw = make_uint2(pack2(F::rn(p.x), F::rn(p.y)), pack2(F::rn(p.z), F::rn(p.w)));
        } else {
          const uint2 gw = *reinterpret_cast<const uint2*>(st + 2 * j);
          const uint16_t h0 = F::rn(adam1(F::lo(gw.x), p.x, m.x, v.x, sc));  // loss-scale and clip factors via sc.flags
          const uint16_t h1 = F::rn(adam1(F::hi(gw.x), p.y, m.y, v.y, sc));
          const uint16_t h2 = F::rn(adam1(F::lo(gw.y), p.z, m.z, v.z, sc));
          const uint16_t h3 = F::rn(adam1(F::hi(gw.y), p.w, m.w, v.w, sc));
          pw = make_uint2(pack2(h0, h1), pack2(h2, h3));
          *reinterpret_cast<float4*>(st + 2 * T + 4 * j) = p;
          *reinterpret_cast<float4*>(st + 6 * T + 4 * j) = m;
          *reinterpret_cast<float4*>(st + 10 * T + 4 * j) = v;
        }
        *reinterpret_cast<uint2*>(st + 2 * j) = pw;  // over the gradient, which this lane alone read here
      }
      fence_proxy_async_smem();  // this lane's stage writes before the storer's bulk copies read them
      __syncwarp();
      if (lane == 0) mbar_arrive(&computed[s]);
    }
  }
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    // drain the bulk loads already issued before the CTA's memory goes away
    for (int s = 0; s < stages; ++s)
      if (last_k[s] >= 0 && !mbar_wait(&full[s], (unsigned)last_k[s] & 1u)) atomicOr(a.error, 4u);
  }
}

// The same pass over every layer of a stage-3 step in one cooperative launch
// (layered_walk.cuh): `a`'s sources, states and shard at flat element 0
// (a.lo = 0), its N destinations at the temporary layer buffers' start; a
// layer's stores into those buffers follow every CTA's stores of the layers
// before it.  A kernel of its own, so that the one-interval kernel above
// keeps its measured code.
template <class F>
__global__ void __launch_bounds__(kBulkBcastThreads, 1)
    adam_bcast_bulk_layered_kernel(const __grid_constant__ AdamBcastArgs a, int stages, int uniform, int store_hint,
                                   const __grid_constant__ SegTable g) {
  constexpr int T = kBulkBcastTile;
  constexpr int W = kBulkBcastWarps;
  constexpr int EPT = T / (32 * W);
  static_assert(EPT == 4, "four elements per consumer lane");
  extern __shared__ __align__(128) unsigned char smem[];
  const unsigned sb = kBulkBcastStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)stages * sb);
  uint64_t* computed = full + stages;
  uint64_t* empty = computed + stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + stages);
  volatile int* last_k = abort_flag + 1;
  AdamScalars sc = a.sc_dev ? *a.sc_dev : a.sc;
  const bool skip = apply_decision(a.dec, sc);  // a skipped step writes the unchanged parameters only
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&computed[s], W);
      mbar_init(&empty[s], 1);
      last_k[s] = -1;
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      const uint64_t policy = evict_first_policy();
      TileCursor cur;
      for (int it = 0;; ++it) {
        long long e0, ed;
        unsigned cnt;
        if (!cursor_next<T, true>(cur, g, 0, 0, e0, ed, cnt) || *abort_flag) break;
        const int s = it % stages;
        const unsigned k = (unsigned)(it / stages);
        if (k > 0) {
          const int w = mbar_wait_or_abort(&empty[s], (k - 1) & 1u, abort_flag, a.wait_ns);
          if (w != 0) {
            if (w == 1) atomicOr(a.error, 1u);
            *abort_flag = 1;
            break;
          }
        }
        fence_proxy_async_smem();  // the stage's last reads (consumers, stores) before the refill
        unsigned char* st = smem + (size_t)s * sb;
        mbar_expect_tx(&full[s], cnt * 14u);
        const int64_t i0 = e0;  // flat index of the tile's first element
        if (uniform) {
          bulk_load(st, a.gsrc[0] + i0, (unsigned)(2 * cnt), &full[s], policy);
        } else {
          // one copy per owner: owners change every `shard` elements (a multiple of 8)
          for (int64_t e = 0; e < (int64_t)cnt;) {
            const int64_t owner = (i0 + e) / a.shard;
            const int64_t next = (owner + 1) * a.shard - i0;
            const int64_t end = next < (int64_t)cnt ? next : (int64_t)cnt;
            bulk_load(st + 2 * e, a.gsrc[owner] + i0 + e, (unsigned)(2 * (end - e)), &full[s], policy);
            e = end;
          }
        }
        bulk_load(st + 2 * T, a.master + e0, (unsigned)(4 * cnt), &full[s], policy);
        bulk_load(st + 6 * T, a.m + e0, (unsigned)(4 * cnt), &full[s], policy);
        bulk_load(st + 10 * T, a.v + e0, (unsigned)(4 * cnt), &full[s], policy);
        last_k[s] = (int)k;
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------- storer --
    if (lane == 0) {
      const uint64_t spol = evict_first_policy();
      auto put = [&](void* dst, const void* src, unsigned bytes) {
        if (store_hint) bulk_store(dst, src, bytes, spol);
        else bulk_store(dst, src, bytes);
      };
      TileCursor cur;
      int arrived = 0;  // layers this storer has finished and arrived for
      for (int it = 0;; ++it) {
        long long e0, ed;
        unsigned cnt;
        if (!cursor_next<T, true>(cur, g, 0, 0, e0, ed, cnt)) break;
        const int s = it % stages;
        const unsigned k = (unsigned)(it / stages);
        const int w = mbar_wait_or_abort(&computed[s], k & 1u, abort_flag, a.wait_ns);
        if (w != 0) {
          if (w == 1) atomicOr(a.error, 8u);
          *abort_flag = 1;
          break;
        }
        if (cur.seg > arrived) {  // a new layer: every CTA's stores of the layers before it first
          while (arrived < cur.seg) {
            segment_arrive(g.counter);
            ++arrived;
          }
          if (!segment_wait(g.counter, gridDim.x * (unsigned)cur.seg, abort_flag, a.wait_ns)) {
            atomicOr(a.error, 16u);
            *abort_flag = 1;
            break;
          }
        }
        const unsigned char* st = smem + (size_t)s * sb;
        if (!skip) {
          put(a.master + e0, st + 2 * T, 4 * cnt);
          put(a.m + e0, st + 6 * T, 4 * cnt);
          put(a.v + e0, st + 10 * T, 4 * cnt);
        }
        if (a.param_shard) put(a.param_shard + e0, st, 2 * cnt);
        for (int r = 0; r < a.n_out; ++r) put(a.out[r] + ed, st, 2 * cnt);
        bulk_commit();
        bulk_wait_read<0>();  // the copies have read the stage: hand it back to the producer
        mbar_arrive(&empty[s]);
      }
      // arrive for the layers left (also after an abort: the other CTAs'
      // waits then end; the step has failed)
      for (; arrived < g.n; ++arrived) segment_arrive(g.counter);
      bulk_wait<0>();  // every store of this CTA performed before the CTA ends
    }
  } else {
    // ----------------------------------------------------------- consumers --
    const int j = (threadIdx.x - 64) * EPT;
    TileCursor cur;
    for (int it = 0;; ++it) {
      long long e0, ed;
      unsigned cnt;
      if (!cursor_next<T, true>(cur, g, 0, 0, e0, ed, cnt)) break;
      const int s = it % stages;
      const unsigned k = (unsigned)(it / stages);
      const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(&full[s], k & 1u, a.wait_ns));
      if (!ok) {
        if (lane == 0) atomicOr(a.error, 2u);
        *abort_flag = 1;
        break;
      }
      if (__any_sync(0xFFFFFFFFu, *abort_flag != 0)) break;
      unsigned char* st = smem + (size_t)s * sb;
      if (j < (int)cnt) {  // cnt is a multiple of 8, so a lane's four elements are whole
        float4 p = *reinterpret_cast<const float4*>(st + 2 * T + 4 * j);
        float4 m = *reinterpret_cast<const float4*>(st + 6 * T + 4 * j);
        float4 v = *reinterpret_cast<const float4*>(st + 10 * T + 4 * j);
        uint2 pw;
        if (skip) {
          pw = make_uint2(pack2(F::rn(p.x), F::rn(p.y)), pack2(F::rn(p.z), F::rn(p.w)));
        } else {
          const uint2 gw = *reinterpret_cast<const uint2*>(st + 2 * j);
          const uint16_t h0 = F::rn(adam1(F::lo(gw.x), p.x, m.x, v.x, sc));  // loss-scale and clip factors via sc.flags
          const uint16_t h1 = F::rn(adam1(F::hi(gw.x), p.y, m.y, v.y, sc));
          const uint16_t h2 = F::rn(adam1(F::lo(gw.y), p.z, m.z, v.z, sc));
          const uint16_t h3 = F::rn(adam1(F::hi(gw.y), p.w, m.w, v.w, sc));
          pw = make_uint2(pack2(h0, h1), pack2(h2, h3));
          *reinterpret_cast<float4*>(st + 2 * T + 4 * j) = p;
          *reinterpret_cast<float4*>(st + 6 * T + 4 * j) = m;
          *reinterpret_cast<float4*>(st + 10 * T + 4 * j) = v;
        }
        *reinterpret_cast<uint2*>(st + 2 * j) = pw;  // over the gradient, which this lane alone read here
      }
      fence_proxy_async_smem();  // this lane's stage writes before the storer's bulk copies read them
      __syncwarp();
      if (lane == 0) mbar_arrive(&computed[s]);
    }
  }
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    // drain the bulk loads already issued before the CTA's memory goes away
    for (int s = 0; s < stages; ++s)
      if (last_k[s] >= 0 && !mbar_wait(&full[s], (unsigned)last_k[s] & 1u)) atomicOr(a.error, 4u);
  }
}

template <class K>
cudaError_t opt_in(K kernel) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTmaMaxSmem);
}

int reduce_stages(int n_ranks) {
  int stages = kTpStages;
  while (stages > 2 && tp_smem_bytes(reduce_stage_bytes(n_ranks), stages) > (size_t)kTmaMaxSmem) --stages;
  return stages;
}

}  // namespace

cudaError_t two_pass_configure() {
  cudaError_t e = cudaSuccess;
  if (e == cudaSuccess) e = opt_in(reduce_tma_kernel<false, Bf16>);
  if (e == cudaSuccess) e = opt_in(reduce_tma_kernel<true, Bf16>);
  if (e == cudaSuccess) e = opt_in(reduce_tma_kernel<false, F16>);
  if (e == cudaSuccess) e = opt_in(reduce_tma_kernel<true, F16>);
  if (e == cudaSuccess) e = opt_in(reduce_chunked_tma_kernel<false, Bf16>);
  if (e == cudaSuccess) e = opt_in(reduce_chunked_tma_kernel<true, Bf16>);
  if (e == cudaSuccess) e = opt_in(reduce_chunked_tma_kernel<false, F16>);
  if (e == cudaSuccess) e = opt_in(reduce_chunked_tma_kernel<true, F16>);
  if (e == cudaSuccess) e = opt_in(adam_bcast_tma_kernel<Bf16>);
  if (e == cudaSuccess) e = opt_in(adam_bcast_tma_kernel<F16>);
  if (e == cudaSuccess) e = opt_in(adam_bcast_bulk_kernel<Bf16>);
  if (e == cudaSuccess) e = opt_in(adam_bcast_bulk_kernel<F16>);
  if (e == cudaSuccess) e = opt_in(adam_bcast_bulk_layered_kernel<Bf16>);
  if (e == cudaSuccess) e = opt_in(adam_bcast_bulk_layered_kernel<F16>);
  if (e == cudaSuccess) e = opt_in(reduce_bulk_kernel<false, Bf16>);
  if (e == cudaSuccess) e = opt_in(reduce_bulk_kernel<true, Bf16>);
  if (e == cudaSuccess) e = opt_in(reduce_bulk_kernel<false, F16>);
  if (e == cudaSuccess) e = opt_in(reduce_bulk_kernel<true, F16>);
  return e;
}

cudaError_t launch_reduce_tma(const ReduceArgs& a, int grid, cudaStream_t s) {
  if (a.n_ranks < 1 || a.n_ranks > kMaxRanks) return cudaErrorInvalidValue;
  if (a.n_ranks > kTmaMaxRanks) {
    const size_t bytes = tp_smem_bytes(kChunkStageBytes, kTpStages);
    if (a.fmt == kFmtF16) {
      if (a.write_back) reduce_chunked_tma_kernel<true, F16><<<grid, kTpThreads, bytes, s>>>(a, kTpStages);
      else reduce_chunked_tma_kernel<false, F16><<<grid, kTpThreads, bytes, s>>>(a, kTpStages);
    } else {
      if (a.write_back) reduce_chunked_tma_kernel<true, Bf16><<<grid, kTpThreads, bytes, s>>>(a, kTpStages);
      else reduce_chunked_tma_kernel<false, Bf16><<<grid, kTpThreads, bytes, s>>>(a, kTpStages);
    }
    return cudaGetLastError();
  }
  const int stages = reduce_stages(a.n_ranks);
  const size_t bytes = tp_smem_bytes(reduce_stage_bytes(a.n_ranks), stages);
  if (a.fmt == kFmtF16) {
    if (a.write_back) reduce_tma_kernel<true, F16><<<grid, kTpThreads, bytes, s>>>(a, stages);
    else reduce_tma_kernel<false, F16><<<grid, kTpThreads, bytes, s>>>(a, stages);
  } else {
    if (a.write_back) reduce_tma_kernel<true, Bf16><<<grid, kTpThreads, bytes, s>>>(a, stages);
    else reduce_tma_kernel<false, Bf16><<<grid, kTpThreads, bytes, s>>>(a, stages);
  }
  return cudaGetLastError();
}

cudaError_t launch_adam_bcast_tma(const AdamBcastArgs& a, int grid, bool uniform, cudaStream_t s) {
  const size_t bytes = tp_smem_bytes(kBcastStageBytes, kTpStages);
  if (a.fmt == kFmtF16)
    adam_bcast_tma_kernel<F16><<<grid, kTpThreads, bytes, s>>>(a, kTpStages, uniform ? 1 : 0);
  else
    adam_bcast_tma_kernel<Bf16><<<grid, kTpThreads, bytes, s>>>(a, kTpStages, uniform ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_adam_bcast_bulk(const AdamBcastArgs& a, int grid, bool uniform, int stages, int store_hint,
                                   cudaStream_t s) {
  if (stages < 2) stages = 2;
  if (stages > kTmaMaxStages) stages = kTmaMaxStages;
  while (stages > 2 && bulk_bcast_smem_bytes(stages) > (size_t)kTmaMaxSmem) --stages;
  const size_t bytes = bulk_bcast_smem_bytes(stages);
  if (a.fmt == kFmtF16)
    adam_bcast_bulk_kernel<F16><<<grid, kBulkBcastThreads, bytes, s>>>(a, stages, uniform ? 1 : 0, store_hint);
  else
    adam_bcast_bulk_kernel<Bf16><<<grid, kBulkBcastThreads, bytes, s>>>(a, stages, uniform ? 1 : 0, store_hint);
  return cudaGetLastError();
}

cudaError_t launch_adam_bcast_bulk_layered(const AdamBcastArgs& a, const SegTable& g, int grid, bool uniform,
                                           int stages, int store_hint, cudaStream_t s) {
  if (g.n < 1 || g.n > kMaxSegments || !g.counter || a.lo != 0) return cudaErrorInvalidValue;
  if (stages < 2) stages = 2;
  if (stages > kTmaMaxStages) stages = kTmaMaxStages;
  while (stages > 2 && bulk_bcast_smem_bytes(stages) > (size_t)kTmaMaxSmem) --stages;
  // at least 116 KB, so that an SM holds one CTA: tiles are dealt by CTA index
  const size_t bytes = std::max<size_t>(bulk_bcast_smem_bytes(stages), 116 * 1024);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)kBulkBcastThreads);
  cfg.dynamicSmemBytes = bytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const int un = uniform ? 1 : 0;
  if (a.fmt == kFmtF16)
    return cudaLaunchKernelEx(&cfg, adam_bcast_bulk_layered_kernel<F16>, a, stages, un, store_hint, g);
  return cudaLaunchKernelEx(&cfg, adam_bcast_bulk_layered_kernel<Bf16>, a, stages, un, store_hint, g);
}

cudaError_t launch_reduce_bulk(const ReduceArgs& a, int grid, int stages, int store_hint, cudaStream_t s) {
  if (a.n_ranks < 1 || a.n_ranks > kTmaMaxRanks) return cudaErrorInvalidValue;
  if (stages < 2) stages = 2;
  if (stages > kTmaMaxStages) stages = kTmaMaxStages;
  while (stages > 2 && bulk_reduce_smem_bytes(a.n_ranks, stages) > (size_t)kTmaMaxSmem) --stages;
  const size_t bytes = bulk_reduce_smem_bytes(a.n_ranks, stages);
  if (a.fmt == kFmtF16) {
    if (a.write_back) reduce_bulk_kernel<true, F16><<<grid, kBulkRedThreads, bytes, s>>>(a, stages, store_hint);
    else reduce_bulk_kernel<false, F16><<<grid, kBulkRedThreads, bytes, s>>>(a, stages, store_hint);
  } else {
    if (a.write_back) reduce_bulk_kernel<true, Bf16><<<grid, kBulkRedThreads, bytes, s>>>(a, stages, store_hint);
    else reduce_bulk_kernel<false, Bf16><<<grid, kBulkRedThreads, bytes, s>>>(a, stages, store_hint);
  }
  return cudaGetLastError();
}

int64_t two_pass_tile() { return kTile; }
int64_t bulk_bcast_tile() { return kBulkBcastTile; }

}  // namespace zsm
