// Fused ZeRO step kernel with the inputs staged through shared memory by the
// Tensor Memory Accelerator (sm_100a).
//
// Same arithmetic and outputs as the register-path fused kernel (kernels.cu),
// different data movement: one persistent CTA per SM; warp 0 is a producer
// whose elected lane streams each tile's N gradient slices and its fp32
// master/m/v slices from HBM into a ring of shared-memory stages with 1-D
// bulk copies (cp.async.bulk, completion counted in bytes on an mbarrier);
// two groups of eight consumer warps take alternate tiles, reduce, update
// and store from shared memory, then release the stage.  Group g owns stages
// g, g+2, ... (the stage count is even), so each group meets the phases of
// its stages in order.  With four 56 KB stages per SM (N = 8) up to 224 KB of
// loads are in flight per SM without holding them in registers.  The bulk copies
// read only this GPU's memory into the CTA's own shared memory; no cluster
// multicast is used.
//
// Every wait on an mbarrier is bounded (kWaitNs of wall time).  A wait that
// runs out records an error code in the scratch arena, stops the producer,
// drains the copies already issued (again bounded) and ends the CTA, so the
// host sees ZERO_ECUDA instead of a hung GPU.
#include <cuda_runtime.h>

#include <algorithm>

#include "device_math.cuh"
#include "kernels.cuh"
#include "tma_pipe.cuh"

namespace zsm {
namespace {

using namespace dev;
using namespace pipe;


__host__ __device__ inline unsigned tma_stage_bytes(int n_ranks) {
  return (unsigned)(kTile * (2 * n_ranks + 12));
}

// Shared memory: [stages x stage_bytes][full[stages]][empty[stages]][abort][last_k[stages]]
//
// Warps 0..G-1 are producers (lane 0 works), warps G + 8g .. G + 8g + 7 form
// consumer group g.  Tile number `it` of this CTA (tile = blockIdx.x + it *
// gridDim.x) belongs to group it % G and lives in stage it % stages; the
// stage count is a multiple of G, so every stage belongs to one group and
// each group's producer and consumers meet its stages' phases in order.
template <int MODE, int G, class F>
__global__ void __launch_bounds__(tma_threads<G>(), 1)
    fused_step_tma_kernel(const __grid_constant__ FusedArgs a, int stages) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int N = a.n_ranks;
  const unsigned stage_bytes = tma_stage_bytes(N);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)stages * stage_bytes);
  uint64_t* empty = full + stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + stages);
  volatile int* last_k = abort_flag + 1;  // last phase issued on each stage, -1 = none
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_elem = a.n_vec * kVec;
  const int64_t n_tiles = (n_elem + kTile - 1) / kTile;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
      last_k[s] = -1;
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (a.pdl == kPdlWaitFirst) pdl_wait();

  double sq = 0.0;
  unsigned long long nf = 0;
  bool waited = false;  // this thread has waited for the grid before (kPdlEarlyLoads)
  const AdamScalars sc = a.sc_dev ? *a.sc_dev : a.sc;

  if (warp < G) {
    // ---------------------------------------------------------- producer --
    if (lane == 0) {
      const int g = warp;
      const uint64_t policy = evict_first_policy();
      for (int it = g;; it += G) {
        const int64_t tile = blockIdx.x + (int64_t)it * gridDim.x;
        if (tile >= n_tiles) break;
        const int s = it % stages;
        const unsigned k = (unsigned)(it / stages);
        if (*abort_flag) break;
        if (k > 0 && !mbar_wait(&empty[s], (k - 1) & 1u, a.ns.wait_ns)) {
          atomicOr(a.ns.error, 1u);
          *abort_flag = 1;
          break;
        }
        fence_proxy_async_smem();  // the consumers' reads of this stage before the copies refill it
        const int64_t e0 = tile * kTile;
        const int64_t cnt = (n_elem - e0) < kTile ? (n_elem - e0) : kTile;
        unsigned char* st = smem + (size_t)s * stage_bytes;
        mbar_expect_tx(&full[s], (unsigned)(cnt * (2 * N + 12)));
        for (int r = 0; r < N; ++r)
          bulk_load(st + (size_t)r * 2 * kTile, a.grad[r] + e0, (unsigned)(2 * cnt), &full[s], policy);
        unsigned char* stt = st + (size_t)N * 2 * kTile;
        bulk_load(stt, a.master + e0, (unsigned)(4 * cnt), &full[s], policy);
        bulk_load(stt + 4 * kTile, a.m + e0, (unsigned)(4 * cnt), &full[s], policy);
        bulk_load(stt + 8 * kTile, a.v + e0, (unsigned)(4 * cnt), &full[s], policy);
        last_k[s] = (int)k;
      }
      pdl_trigger();  // no more loads to issue: the next fused launch may start
    }
  } else {
    // --------------------------------------------------------- consumers --
    const int g = (warp - G) / kConsumerWarps;
    const int c = (threadIdx.x - 32 * G) % kConsumers;  // 0..255
    for (int it = g;; it += G) {
      const int64_t tile = blockIdx.x + (int64_t)it * gridDim.x;
      if (tile >= n_tiles) break;
      const int s = it % stages;
      const unsigned k = (unsigned)(it / stages);
      // warp-uniform decisions, so that no lane is left waiting at __syncwarp
      const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(&full[s], k & 1u, a.ns.wait_ns));
      if (!ok) {
        if (lane == 0) atomicOr(a.ns.error, 2u);
        *abort_flag = 1;
        break;
      }
      if (__any_sync(0xFFFFFFFFu, *abort_flag != 0)) break;
      const int64_t e0 = tile * kTile;
      const int64_t cnt = (n_elem - e0) < kTile ? (n_elem - e0) : kTile;
      const unsigned char* st = smem + (size_t)s * stage_bytes;
      const int j = c * kVec;
      const bool active = j < cnt;  // the last tile may be ragged
      float4 p0, p1, m0, m1, v0, v1;
      float acc[kVec];
      if (active) {
        const float* stt = reinterpret_cast<const float*>(st + (size_t)N * 2 * kTile);
        p0 = *reinterpret_cast<const float4*>(stt + j);
        p1 = *reinterpret_cast<const float4*>(stt + j + 4);
        m0 = *reinterpret_cast<const float4*>(stt + kTile + j);
        m1 = *reinterpret_cast<const float4*>(stt + kTile + j + 4);
        v0 = *reinterpret_cast<const float4*>(stt + 2 * kTile + j);
        v1 = *reinterpret_cast<const float4*>(stt + 2 * kTile + j + 4);
#pragma unroll
        for (int q = 0; q < kVec; ++q) acc[q] = 0.0f;
        for (int r = 0; r < N; ++r)
          add8<F>(acc, *reinterpret_cast<const uint4*>(st + (size_t)r * 2 * kTile + 2 * j));
      }
      // every lane of the warp is done reading this stage: release it
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (active) {
        const int64_t e = e0 + j;
        if (a.pdl == kPdlEarlyLoads && !waited) {  // the first store waits for the grid before
          pdl_wait();
          waited = true;
        }
        uint16_t g16[kVec];
        float gv[kVec];
        mean_bf16<F>(acc, a.inv_n, g16, gv, sq, nf);
        if (MODE == kFusedZ1) {
          const uint4 gw = pack8(g16);
          for (int r = 0; r < N; ++r) st_out(const_cast<uint16_t*>(a.grad[r]) + e, gw);
        }
        if (a.grad_shard) st_out(a.grad_shard + e, pack8(g16));
        uint16_t p16[kVec];
        adam8<F>(gv, p0, p1, m0, m1, v0, v1, sc, p16);
        st_out(a.master + e, p0);
        st_out(a.master + e + 4, p1);
        st_out(a.m + e, m0);
        st_out(a.m + e + 4, m1);
        st_out(a.v + e, v0);
        st_out(a.v + e + 4, v1);
        const uint4 pw = pack8(p16);
        if (MODE == kFusedZ3) st_out(a.param_shard + e, pw);
        for (int r = 0; r < N; ++r) st_out(a.out[r] + e, pw);
      }
    }
  }
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    // drain the bulk copies already issued before the CTA's memory goes away
    for (int s = 0; s < stages; ++s)
      if (last_k[s] >= 0 && !mbar_wait(&full[s], (unsigned)last_k[s] & 1u)) atomicOr(a.ns.error, 4u);
  }
  if (a.pdl == kPdlEarly || a.pdl == kPdlEarlyLoads) pdl_wait();  // the norm scratch is shared with the grid before
  norm_epilogue<tma_threads<G>()>(a.ns, sq, nf, a.accumulate);
}

// ------------------------------------------- 16 consumer warps variant --
//
// The same tile (2048 elements) and ring as fused_step_tma_kernel<MODE, 1>,
// consumed by sixteen warps of four elements each instead of eight warps of
// eight: twice the warps to hide the latency of the Adam arithmetic, with one
// producer and one in-order pipeline.
constexpr int kWideWarps = 16;
constexpr int kWideThreads = 32 + kWideWarps * 32;  // 544

template <class F>
__device__ __forceinline__ void add4(float (&acc)[4], uint2 w) {
  acc[0] = __fadd_rn(acc[0], F::lo(w.x));
  acc[1] = __fadd_rn(acc[1], F::hi(w.x));
  acc[2] = __fadd_rn(acc[2], F::lo(w.y));
  acc[3] = __fadd_rn(acc[3], F::hi(w.y));
}


template <int MODE, class F>
__global__ void __launch_bounds__(kWideThreads, 1)
    fused_step_tma_wide_kernel(const __grid_constant__ FusedArgs a, int stages) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int N = a.n_ranks;
  const unsigned stage_bytes = tma_stage_bytes(N);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)stages * stage_bytes);
  uint64_t* empty = full + stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + stages);
  volatile int* last_k = abort_flag + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_elem = a.n_vec * kVec;
  const int64_t n_tiles = (n_elem + kTile - 1) / kTile;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kWideWarps);
      last_k[s] = -1;
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (a.pdl == kPdlWaitFirst) pdl_wait();

  double sq = 0.0;
  unsigned long long nf = 0;
  bool waited = false;  // this thread has waited for the grid before (kPdlEarlyLoads)
  const AdamScalars sc = a.sc_dev ? *a.sc_dev : a.sc;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t policy = evict_first_policy();
      for (int it = 0;; ++it) {
        const int64_t tile = blockIdx.x + (int64_t)it * gridDim.x;
        if (tile >= n_tiles || *abort_flag) break;
        const int s = it % stages;
        const unsigned k = (unsigned)(it / stages);
        if (k > 0 && !mbar_wait(&empty[s], (k - 1) & 1u, a.ns.wait_ns)) {
          atomicOr(a.ns.error, 1u);
          *abort_flag = 1;
          break;
        }
        fence_proxy_async_smem();  // the consumers' reads of this stage before the copies refill it
        const int64_t e0 = tile * kTile;
        const int64_t cnt = (n_elem - e0) < kTile ? (n_elem - e0) : kTile;
        unsigned char* st = smem + (size_t)s * stage_bytes;
        mbar_expect_tx(&full[s], (unsigned)(cnt * (2 * N + 12)));
        for (int r = 0; r < N; ++r)
          bulk_load(st + (size_t)r * 2 * kTile, a.grad[r] + e0, (unsigned)(2 * cnt), &full[s], policy);
        unsigned char* stt = st + (size_t)N * 2 * kTile;
        bulk_load(stt, a.master + e0, (unsigned)(4 * cnt), &full[s], policy);
        bulk_load(stt + 4 * kTile, a.m + e0, (unsigned)(4 * cnt), &full[s], policy);
        bulk_load(stt + 8 * kTile, a.v + e0, (unsigned)(4 * cnt), &full[s], policy);
        last_k[s] = (int)k;
      }
      pdl_trigger();  // no more loads to issue: the next fused launch may start
    }
  } else {
    const int c = threadIdx.x - 32;  // 0..511
    const int j = c * 4;
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
      const int64_t e0 = tile * kTile;
      const int64_t cnt = (n_elem - e0) < kTile ? (n_elem - e0) : kTile;
      const unsigned char* st = smem + (size_t)s * stage_bytes;
      const bool active = j < cnt;  // cnt is a multiple of 8, so 4-element groups are whole
      float4 p, m, v;
      float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      if (active) {
        const float* stt = reinterpret_cast<const float*>(st + (size_t)N * 2 * kTile);
        p = *reinterpret_cast<const float4*>(stt + j);
        m = *reinterpret_cast<const float4*>(stt + kTile + j);
        v = *reinterpret_cast<const float4*>(stt + 2 * kTile + j);
        for (int r = 0; r < N; ++r) add4<F>(acc, *reinterpret_cast<const uint2*>(st + (size_t)r * 2 * kTile + 2 * j));
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (active) {
        const int64_t e = e0 + j;
        if (a.pdl == kPdlEarlyLoads && !waited) {  // the first store waits for the grid before
          pdl_wait();
          waited = true;
        }
        uint16_t g16[4];
        float gv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          g16[q] = F::rn(__fmul_rn(acc[q], a.inv_n));
          gv[q] = F::f32(g16[q]);
          const double d = (double)gv[q];
          sq = __dadd_rn(sq, __dmul_rn(d, d));
          nf += isfinite(gv[q]) ? 0ull : 1ull;
        }
        const uint2 gw = make_uint2(pack2(g16[0], g16[1]), pack2(g16[2], g16[3]));
        if (MODE == kFusedZ1)
          for (int r = 0; r < N; ++r) st_out(const_cast<uint16_t*>(a.grad[r]) + e, gw);
        if (a.grad_shard) st_out(a.grad_shard + e, gw);
        const uint16_t h0 = F::rn(adam1(gv[0], p.x, m.x, v.x, sc));
        const uint16_t h1 = F::rn(adam1(gv[1], p.y, m.y, v.y, sc));
        const uint16_t h2 = F::rn(adam1(gv[2], p.z, m.z, v.z, sc));
        const uint16_t h3 = F::rn(adam1(gv[3], p.w, m.w, v.w, sc));
        st_out(a.master + e, p);
        st_out(a.m + e, m);
        st_out(a.v + e, v);
        const uint2 pw = make_uint2(pack2(h0, h1), pack2(h2, h3));
        if (MODE == kFusedZ3) st_out(a.param_shard + e, pw);
        for (int r = 0; r < N; ++r) st_out(a.out[r] + e, pw);
      }
    }
  }
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s)
      if (last_k[s] >= 0 && !mbar_wait(&full[s], (unsigned)last_k[s] & 1u)) atomicOr(a.ns.error, 4u);
  }
  if (a.pdl == kPdlEarly || a.pdl == kPdlEarlyLoads) pdl_wait();  // the norm scratch is shared with the grid before
  norm_epilogue<kWideThreads>(a.ns, sq, nf, a.accumulate);
}

// ------------------------------------------------ rank-chunked variant --
//
// For N > 16 a stage holding all N slices of a tile no longer fits, so the
// replicas travel in chunks of kChunkRanks ranks.  Two rings:
//   chunk ring (cstages x 32 KB): the producer streams, tile by tile, the
//                                 rank chunks 0, 1, ... of the tile;
//   state ring (sstages x 24 KB): the tile's master/m/v slices.
// The consumers fold every chunk into their fp32 accumulators in rank order
// (chunk c holds ranks 8c..8c+7), release it, and after the last chunk read the
// states, update and store.  Phases advance in the same order on both sides
// (chunk index = tile iteration x chunks per tile + chunk), so the parity of
// every wait is that of its running index.  One producer, one consumer group.
constexpr int kChunkRanks = 8;
constexpr unsigned kChunkBytes = kChunkRanks * 2 * kTile;   // 32 KB
constexpr unsigned kStateBytes = 12 * kTile;                // 24 KB

__host__ __device__ inline size_t chunked_smem_bytes(int cstages, int sstages) {
  return (size_t)cstages * kChunkBytes + (size_t)sstages * kStateBytes +
         2 * (size_t)(cstages + sstages) * sizeof(uint64_t) + 4 * (size_t)(1 + cstages + sstages);
}

template <int MODE, class F>
__global__ void __launch_bounds__(tma_threads<1>(), 1)
    fused_step_chunked_kernel(const __grid_constant__ FusedArgs a, int cstages, int sstages) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int N = a.n_ranks;
  const int n_chunks = (N + kChunkRanks - 1) / kChunkRanks;
  unsigned char* chunk_base = smem;
  unsigned char* state_base = smem + (size_t)cstages * kChunkBytes;
  uint64_t* cfull = reinterpret_cast<uint64_t*>(state_base + (size_t)sstages * kStateBytes);
  uint64_t* cempty = cfull + cstages;
  uint64_t* sfull = cempty + cstages;
  uint64_t* sempty = sfull + sstages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sempty + sstages);
  volatile int* last_ck = abort_flag + 1;        // last phase issued per chunk stage
  volatile int* last_sk = last_ck + cstages;     // last phase issued per state stage
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_elem = a.n_vec * kVec;
  const int64_t n_tiles = (n_elem + kTile - 1) / kTile;

  if (threadIdx.x == 0) {
    for (int s = 0; s < cstages; ++s) {
      mbar_init(&cfull[s], 1);
      mbar_init(&cempty[s], kConsumerWarps);
      last_ck[s] = -1;
    }
    for (int s = 0; s < sstages; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], kConsumerWarps);
      last_sk[s] = -1;
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (a.pdl == kPdlWaitFirst) pdl_wait();

  double sq = 0.0;
  unsigned long long nf = 0;
  bool waited = false;  // this thread has waited for the grid before (kPdlEarlyLoads)
  const AdamScalars sc = a.sc_dev ? *a.sc_dev : a.sc;

  if (warp == 0) {
    // ---------------------------------------------------------- producer --
    if (lane == 0) {
      const uint64_t policy = evict_first_policy();
      for (int it = 0;; ++it) {
        const int64_t tile = blockIdx.x + (int64_t)it * gridDim.x;
        if (tile >= n_tiles || *abort_flag) break;
        const int64_t e0 = tile * kTile;
        const int64_t cnt = (n_elem - e0) < kTile ? (n_elem - e0) : kTile;
        // the tile's optimizer state
        const int ss = it % sstages;
        const unsigned sk = (unsigned)(it / sstages);
        if (sk > 0 && !mbar_wait(&sempty[ss], (sk - 1) & 1u, a.ns.wait_ns)) {
          atomicOr(a.ns.error, 1u);
          *abort_flag = 1;
          break;
        }
        fence_proxy_async_smem();
        unsigned char* stt = state_base + (size_t)ss * kStateBytes;
        mbar_expect_tx(&sfull[ss], (unsigned)(12 * cnt));
        bulk_load(stt, a.master + e0, (unsigned)(4 * cnt), &sfull[ss], policy);
        bulk_load(stt + 4 * kTile, a.m + e0, (unsigned)(4 * cnt), &sfull[ss], policy);
        bulk_load(stt + 8 * kTile, a.v + e0, (unsigned)(4 * cnt), &sfull[ss], policy);
        last_sk[ss] = (int)sk;
        // the tile's rank chunks
        bool stop = false;
        for (int c = 0; c < n_chunks; ++c) {
          const int ci = it * n_chunks + c;
          const int cs = ci % cstages;
          const unsigned ck = (unsigned)(ci / cstages);
          if (ck > 0 && !mbar_wait(&cempty[cs], (ck - 1) & 1u, a.ns.wait_ns)) {
            atomicOr(a.ns.error, 1u);
            *abort_flag = 1;
            stop = true;
            break;
          }
          fence_proxy_async_smem();
          const int r0 = c * kChunkRanks;
          const int r1 = (r0 + kChunkRanks) < N ? (r0 + kChunkRanks) : N;
          unsigned char* st = chunk_base + (size_t)cs * kChunkBytes;
          mbar_expect_tx(&cfull[cs], (unsigned)((r1 - r0) * 2 * cnt));
          for (int r = r0; r < r1; ++r)
            bulk_load(st + (size_t)(r - r0) * 2 * kTile, a.grad[r] + e0, (unsigned)(2 * cnt), &cfull[cs], policy);
          last_ck[cs] = (int)ck;
        }
        if (stop) break;
      }
      pdl_trigger();  // no more loads to issue: the next fused launch may start
    }
  } else {
    // --------------------------------------------------------- consumers --
    const int c_id = threadIdx.x - 32;  // 0..255
    const int j = c_id * kVec;
    bool aborted = false;
    for (int it = 0; !aborted; ++it) {
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
        const int cs = ci % cstages;
        const unsigned ck = (unsigned)(ci / cstages);
        const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(&cfull[cs], ck & 1u, a.ns.wait_ns));
        if (!ok || __any_sync(0xFFFFFFFFu, *abort_flag != 0)) {
          if (!ok && lane == 0) atomicOr(a.ns.error, 2u);
          *abort_flag = 1;
          aborted = true;
          break;
        }
        const int r0 = c * kChunkRanks;
        const int r1 = (r0 + kChunkRanks) < N ? (r0 + kChunkRanks) : N;
        const unsigned char* st = chunk_base + (size_t)cs * kChunkBytes;
        if (active)
          for (int r = r0; r < r1; ++r)
            add8<F>(acc, *reinterpret_cast<const uint4*>(st + (size_t)(r - r0) * 2 * kTile + 2 * j));
        __syncwarp();
        if (lane == 0) mbar_arrive(&cempty[cs]);
      }
      if (aborted) break;
      const int ss = it % sstages;
      const unsigned sk = (unsigned)(it / sstages);
      const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sfull[ss], sk & 1u, a.ns.wait_ns));
      if (!ok) {
        if (lane == 0) atomicOr(a.ns.error, 2u);
        *abort_flag = 1;
        break;
      }
      float4 p0, p1, m0, m1, v0, v1;
      if (active) {
        const float* stt = reinterpret_cast<const float*>(state_base + (size_t)ss * kStateBytes);
        p0 = *reinterpret_cast<const float4*>(stt + j);
        p1 = *reinterpret_cast<const float4*>(stt + j + 4);
        m0 = *reinterpret_cast<const float4*>(stt + kTile + j);
        m1 = *reinterpret_cast<const float4*>(stt + kTile + j + 4);
        v0 = *reinterpret_cast<const float4*>(stt + 2 * kTile + j);
        v1 = *reinterpret_cast<const float4*>(stt + 2 * kTile + j + 4);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sempty[ss]);
      if (active) {
        const int64_t e = e0 + j;
        if (a.pdl == kPdlEarlyLoads && !waited) {  // the first store waits for the grid before
          pdl_wait();
          waited = true;
        }
        uint16_t g16[kVec];
        float gv[kVec];
        mean_bf16<F>(acc, a.inv_n, g16, gv, sq, nf);
        if (MODE == kFusedZ1) {
          const uint4 gw = pack8(g16);
          for (int r = 0; r < N; ++r) st_out(const_cast<uint16_t*>(a.grad[r]) + e, gw);
        }
        if (a.grad_shard) st_out(a.grad_shard + e, pack8(g16));
        uint16_t p16[kVec];
        adam8<F>(gv, p0, p1, m0, m1, v0, v1, sc, p16);
        st_out(a.master + e, p0);
        st_out(a.master + e + 4, p1);
        st_out(a.m + e, m0);
        st_out(a.m + e + 4, m1);
        st_out(a.v + e, v0);
        st_out(a.v + e + 4, v1);
        const uint4 pw = pack8(p16);
        if (MODE == kFusedZ3) st_out(a.param_shard + e, pw);
        for (int r = 0; r < N; ++r) st_out(a.out[r] + e, pw);
      }
    }
  }
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    // drain the bulk copies already issued before the CTA's memory goes away
    for (int s = 0; s < cstages; ++s)
      if (last_ck[s] >= 0 && !mbar_wait(&cfull[s], (unsigned)last_ck[s] & 1u)) atomicOr(a.ns.error, 4u);
    for (int s = 0; s < sstages; ++s)
      if (last_sk[s] >= 0 && !mbar_wait(&sfull[s], (unsigned)last_sk[s] & 1u)) atomicOr(a.ns.error, 4u);
  }
  if (a.pdl == kPdlEarly || a.pdl == kPdlEarlyLoads) pdl_wait();  // the norm scratch is shared with the grid before
  norm_epilogue<tma_threads<1>()>(a.ns, sq, nf, a.accumulate);
}

// A programmatic dependent launch may place its CTAs while the grid before
// it still runs.  These kernels are persistent -- one CTA per SM, tiles dealt
// out by CTA index -- so an SM must never take two CTAs of one grid: with the
// attribute the launch asks for at least this much shared memory, more than
// half of an SM's 228 KB once the 1 KB each block reserves is counted, and a
// dependent grid's CTAs then land only on SMs the grid before has left.
constexpr size_t kPdlSoloSmem = 116 * 1024;

size_t pdl_smem(const FusedArgs& a, size_t bytes) {
  return a.pdl != kPdlNone && bytes < kPdlSoloSmem ? kPdlSoloSmem : bytes;
}

template <int MODE>
cudaError_t launch_chunked_mode(const FusedArgs& a, int grid, int cstages, int sstages, cudaStream_t s) {
  const size_t bytes = pdl_smem(a, chunked_smem_bytes(cstages, sstages));
  const bool pdl = a.pdl != kPdlNone;
  if (a.fmt == kFmtF16)
    return launch_kernel(fused_step_chunked_kernel<MODE, F16>, grid, tma_threads<1>(), bytes, s, pdl, a, cstages,
                         sstages);
  return launch_kernel(fused_step_chunked_kernel<MODE, Bf16>, grid, tma_threads<1>(), bytes, s, pdl, a, cstages,
                       sstages);
}

size_t tma_smem_bytes(int n_ranks, int stages) {
  return (size_t)stages * tma_stage_bytes(n_ranks) + 2 * stages * sizeof(uint64_t) + 4 * (stages + 1);
}

template <int MODE, class F>
cudaError_t launch_tma_fmt(const FusedArgs& a, int grid, int stages, int groups, size_t bytes, cudaStream_t s) {
  const bool pdl = a.pdl != kPdlNone;
  if (groups == kWideGroup)
    return launch_kernel(fused_step_tma_wide_kernel<MODE, F>, grid, kWideThreads, bytes, s, pdl, a, stages);
  if (groups == 2)
    return launch_kernel(fused_step_tma_kernel<MODE, 2, F>, grid, tma_threads<2>(), bytes, s, pdl, a, stages);
  return launch_kernel(fused_step_tma_kernel<MODE, 1, F>, grid, tma_threads<1>(), bytes, s, pdl, a, stages);
}

template <int MODE>
cudaError_t launch_tma_mode(const FusedArgs& a, int grid, int stages, int groups, cudaStream_t s) {
  const size_t bytes = pdl_smem(a, tma_smem_bytes(a.n_ranks, stages));
  if (a.fmt == kFmtF16) return launch_tma_fmt<MODE, F16>(a, grid, stages, groups, bytes, s);
  return launch_tma_fmt<MODE, Bf16>(a, grid, stages, groups, bytes, s);
}

}  // namespace

template <class K>
static cudaError_t opt_in(K kernel) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTmaMaxSmem);
}

template <class F>
cudaError_t tma_configure_fmt() {
  cudaError_t e = cudaSuccess;
  if (e == cudaSuccess) e = opt_in(fused_step_tma_kernel<kFusedZ1, 1, F>);
  if (e == cudaSuccess) e = opt_in(fused_step_tma_kernel<kFusedZ2, 1, F>);
  if (e == cudaSuccess) e = opt_in(fused_step_tma_kernel<kFusedZ3, 1, F>);
  if (e == cudaSuccess) e = opt_in(fused_step_tma_kernel<kFusedZ1, 2, F>);
  if (e == cudaSuccess) e = opt_in(fused_step_tma_kernel<kFusedZ2, 2, F>);
  if (e == cudaSuccess) e = opt_in(fused_step_tma_kernel<kFusedZ3, 2, F>);
  if (e == cudaSuccess) e = opt_in(fused_step_tma_wide_kernel<kFusedZ1, F>);
  if (e == cudaSuccess) e = opt_in(fused_step_tma_wide_kernel<kFusedZ2, F>);
  if (e == cudaSuccess) e = opt_in(fused_step_tma_wide_kernel<kFusedZ3, F>);
  if (e == cudaSuccess) e = opt_in(fused_step_chunked_kernel<kFusedZ1, F>);
  if (e == cudaSuccess) e = opt_in(fused_step_chunked_kernel<kFusedZ2, F>);
  if (e == cudaSuccess) e = opt_in(fused_step_chunked_kernel<kFusedZ3, F>);
  return e;
}

cudaError_t tma_configure() {
  cudaError_t e = tma_configure_fmt<Bf16>();
  return e == cudaSuccess ? tma_configure_fmt<F16>() : e;
}

cudaError_t launch_fused_chunked(int mode, const FusedArgs& a, int grid, int cstages, cudaStream_t s) {
  const int sstages = 2;
  if (cstages < 2) cstages = 2;
  while (cstages > 2 && chunked_smem_bytes(cstages, sstages) > (size_t)kTmaMaxSmem) --cstages;
  switch (mode) {
    case kFusedZ1: return launch_chunked_mode<kFusedZ1>(a, grid, cstages, sstages, s);
    case kFusedZ2: return launch_chunked_mode<kFusedZ2>(a, grid, cstages, sstages, s);
    case kFusedZ3: return launch_chunked_mode<kFusedZ3>(a, grid, cstages, sstages, s);
    default: return cudaErrorInvalidValue;
  }
}

int tma_stages_for(int n_ranks, int groups, int max_stages) {
  if (n_ranks < 1 || n_ranks > kTmaMaxRanks || (groups != 1 && groups != 2 && groups != kWideGroup)) return 0;
  if (groups == kWideGroup) groups = 1;  // one pipeline
  int stages = max_stages > 0 ? std::min(max_stages, kTmaMaxStages) : kTmaDefaultStages;
  while (stages > 0 && tma_smem_bytes(n_ranks, stages) > (size_t)kTmaMaxSmem) --stages;
  stages -= stages % groups;  // every stage belongs to one consumer group
  return stages >= 2 ? stages : 0;
}

int tma_ctas_per_sm(int n_ranks, int groups, int max_stages) {
  const int stages = tma_stages_for(n_ranks, groups, max_stages);
  if (stages == 0) return 0;
  const size_t bytes = tma_smem_bytes(n_ranks, stages);
  int b = 0;
  cudaError_t e = groups == kWideGroup
                      ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, fused_step_tma_wide_kernel<kFusedZ2, Bf16>,
                                                                      kWideThreads, bytes)
                  : groups == 2
                      ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, fused_step_tma_kernel<kFusedZ2, 2, Bf16>,
                                                                      tma_threads<2>(), bytes)
                      : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, fused_step_tma_kernel<kFusedZ2, 1, Bf16>,
                                                                      tma_threads<1>(), bytes);
  return e == cudaSuccess ? b : 0;
}

cudaError_t launch_fused_tma(int mode, const FusedArgs& a, int grid, int groups, int max_stages,
                             cudaStream_t s) {
  const int stages = tma_stages_for(a.n_ranks, groups, max_stages);
  if (stages == 0) return cudaErrorInvalidValue;
  switch (mode) {
    case kFusedZ1: return launch_tma_mode<kFusedZ1>(a, grid, stages, groups, s);
    case kFusedZ2: return launch_tma_mode<kFusedZ2>(a, grid, stages, groups, s);
    case kFusedZ3: return launch_tma_mode<kFusedZ3>(a, grid, stages, groups, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace zsm
