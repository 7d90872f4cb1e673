// Fused ZeRO step kernel whose loads AND stores are bulk copies (sm_100a).
//
// The same arithmetic and outputs as the other fused kernels (reduce in rank
// order, mean, Adam, broadcast of the 16-bit parameters -- "ZERO训练技术",
// sections "ZeRO-1"/"ZeRO-2"/"ZeRO-3", parts "2. 反向" and "3. 更新"), with
// both directions of data movement handed to the Tensor Memory Accelerator:
//
//   warp 0 (producer)  its elected lane streams tile after tile -- the N
//                      gradient slices and the fp32 master/m/v slices of T
//                      elements -- into a ring of shared-memory stages
//                      (cp.async.bulk, completion counted in bytes on the
//                      stage's `full` mbarrier);
//   warps 2..W+1       (consumers) reduce, update, and write every result
//                      back into the same stage: master/m/v in place, the
//                      16-bit parameters over rank 0's gradient slice, the
//                      averaged gradient (stage 1 write-back or the reduced
//                      shard) into a slice of its own; then fence the async
//                      proxy and arrive on the stage's `computed` mbarrier;
//   warp 1 (storer)    its elected lane waits for `computed`, issues the
//                      stage's bulk stores (shared -> global: master, m, v,
//                      the N parameter replicas, the ZeRO-3 shard, the
//                      ZeRO-1 write-back), waits until they have read the
//                      stage and releases it to the producer (`empty`).
//
// A lane of the consumers therefore issues no global store at all: the 2N + 6
// sixteen-byte stores per lane per tile of the register-store kernels become
// N + 3 (+ N at ZeRO-1) bulk copies per tile from one thread.  Every copy
// reads or writes only this GPU's memory and this CTA's shared memory; no
// cluster multicast.
//
// Every mbarrier wait is bounded (kWaitNs); a role whose wait runs out sets an
// error bit in the scratch arena and the CTA's abort flag, the other roles
// leave their loops, the copies already issued are drained (loads: bounded
// wait on their barriers; stores: the issuing thread's bulk-group wait, which
// depends on no other thread) and the CTA ends.
//
// kMove builds the movement-only twin used to measure what this exact pattern
// of streams can move on the device: identical copies and shared-memory
// traffic, the arithmetic replaced by an XOR fold of the gradients and the
// 16-bit rounding of the unchanged master weights (so a twin pass leaves a
// context's master/m/v and parameters as they were).  No step entry point
// launches it.
#include <cuda_runtime.h>

#include <algorithm>

#include "device_math.cuh"
#include "kernels.cuh"
#include "tma_pipe.cuh"
#include "layered_walk.cuh"

namespace zsm {
namespace {

using namespace dev;
using namespace pipe;

// ------------------------------------------------ per-thread smem vectors --

template <int EPT>
struct H16 {  // EPT 16-bit values, two per word
  uint32_t w[EPT / 2];
};
template <int EPT>
struct V32 {  // EPT fp32 values
  float f[EPT];
};

template <int EPT>
__device__ __forceinline__ H16<EPT> lds16(const unsigned char* p);
template <>
__device__ __forceinline__ H16<8> lds16<8>(const unsigned char* p) {
  const uint4 v = *reinterpret_cast<const uint4*>(p);
  return {{v.x, v.y, v.z, v.w}};
}
template <>
__device__ __forceinline__ H16<4> lds16<4>(const unsigned char* p) {
  const uint2 v = *reinterpret_cast<const uint2*>(p);
  return {{v.x, v.y}};
}
template <>
__device__ __forceinline__ H16<2> lds16<2>(const unsigned char* p) {
  return {{*reinterpret_cast<const uint32_t*>(p)}};
}

template <int EPT>
__device__ __forceinline__ void sts16(unsigned char* p, const H16<EPT>& h);
template <>
__device__ __forceinline__ void sts16<8>(unsigned char* p, const H16<8>& h) {
  *reinterpret_cast<uint4*>(p) = make_uint4(h.w[0], h.w[1], h.w[2], h.w[3]);
}
template <>
__device__ __forceinline__ void sts16<4>(unsigned char* p, const H16<4>& h) {
  *reinterpret_cast<uint2*>(p) = make_uint2(h.w[0], h.w[1]);
}
template <>
__device__ __forceinline__ void sts16<2>(unsigned char* p, const H16<2>& h) {
  *reinterpret_cast<uint32_t*>(p) = h.w[0];
}

template <int EPT>
__device__ __forceinline__ V32<EPT> ldsf(const unsigned char* p) {
  V32<EPT> r;
#pragma unroll
  for (int q = 0; q < EPT; q += 4) {
    if constexpr (EPT >= 4) {
      const float4 v = *reinterpret_cast<const float4*>(p + 4 * q);
      r.f[q] = v.x;
      r.f[q + 1] = v.y;
      r.f[q + 2] = v.z;
      r.f[q + 3] = v.w;
    } else {
      const float2 v = *reinterpret_cast<const float2*>(p + 4 * q);
      r.f[q] = v.x;
      r.f[q + 1] = v.y;
    }
  }
  return r;
}

template <int EPT>
__device__ __forceinline__ void stsf(unsigned char* p, const V32<EPT>& r) {
#pragma unroll
  for (int q = 0; q < EPT; q += 4) {
    if constexpr (EPT >= 4) {
      *reinterpret_cast<float4*>(p + 4 * q) = make_float4(r.f[q], r.f[q + 1], r.f[q + 2], r.f[q + 3]);
    } else {
      *reinterpret_cast<float2*>(p + 4 * q) = make_float2(r.f[q], r.f[q + 1]);
    }
  }
}

// ------------------------------------------------------------ stage layout --
//
// One stage of T elements: [N gradient slices, 2T bytes each][master 4T][m 4T]
// [v 4T][averaged gradient 2T, only when stored].  Consumers overwrite the
// state slices in place and rank 0's gradient slice with the parameters.
__host__ __device__ inline unsigned bulk_stage_bytes(int n_ranks, int tile, bool need_g) {
  return (unsigned)tile * (unsigned)(2 * n_ranks + 12 + (need_g ? 2 : 0));
}

__host__ __device__ inline size_t bulk_smem_bytes(int n_ranks, int tile, bool need_g, int stages) {
  return (size_t)stages * bulk_stage_bytes(n_ranks, tile, need_g) + 3 * (size_t)stages * sizeof(uint64_t) +
         4 * (size_t)(stages + 1);
}

template <int MODE, class F, int T, int W, bool kMove>
__global__ void __launch_bounds__(32 * (W + 2), 1)
    fused_bulk_kernel(const __grid_constant__ FusedArgs a, int stages, uint32_t opaque) {
  constexpr int EPT = T / (32 * W);
  static_assert(EPT == 2 || EPT == 4 || EPT == 8, "2, 4 or 8 elements per consumer lane");
  constexpr int NT = 32 * (W + 2);
  extern __shared__ __align__(128) unsigned char smem[];
  const int N = a.n_ranks;
  const bool need_g = MODE == kFusedZ1 || a.grad_shard != nullptr;
  const unsigned sb = bulk_stage_bytes(N, T, need_g);
  const unsigned off_state = 2u * (unsigned)N * T;  // master; m at +4T, v at +8T
  const unsigned off_g = off_state + 12u * T;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)stages * sb);
  uint64_t* computed = full + stages;
  uint64_t* empty = computed + stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + stages);
  volatile int* last_k = abort_flag + 1;  // last phase of `full` issued per stage, -1 = none
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
  if (a.pdl == kPdlWaitFirst) pdl_wait();

  double sq = 0.0;
  unsigned nf32 = 0;  // non-finite count of this lane (well below 2^32 elements a lane)
  const AdamScalars sc = a.sc_dev ? *a.sc_dev : a.sc;

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
        fence_proxy_async_smem();  // the stage's last reads (consumers, stores) before the refill
        const int64_t e0 = tile * T;
        const int64_t cnt = (n_elem - e0) < T ? (n_elem - e0) : T;
        unsigned char* st = smem + (size_t)s * sb;
        mbar_expect_tx(&full[s], (unsigned)(cnt * (2 * N + 12)));
        for (int r = 0; r < N; ++r)
          bulk_load(st + (size_t)r * 2 * T, a.grad[r] + e0, (unsigned)(2 * cnt), &full[s], policy);
        bulk_load(st + off_state, a.master + e0, (unsigned)(4 * cnt), &full[s], policy);
        bulk_load(st + off_state + 4 * T, a.m + e0, (unsigned)(4 * cnt), &full[s], policy);
        bulk_load(st + off_state + 8 * T, a.v + e0, (unsigned)(4 * cnt), &full[s], policy);
        last_k[s] = (int)k;
      }
      pdl_trigger();  // no more loads to issue: the next fused launch may start
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------- storer --
    if (lane == 0) {
      bool waited = false;
      const uint64_t spol = evict_first_policy();
      const bool hint = a.store_hint != 0;
      auto put = [&](void* dst, const void* src, unsigned bytes) {
        if (hint) bulk_store(dst, src, bytes, spol);
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
        if (a.pdl == kPdlEarlyLoads && !waited) {  // the first store waits for the grid before
          pdl_wait();
          waited = true;
        }
        const int64_t e0 = tile * T;
        const unsigned cnt = (unsigned)((n_elem - e0) < T ? (n_elem - e0) : T);
        const unsigned char* st = smem + (size_t)s * sb;
        put(a.master + e0, st + off_state, 4 * cnt);
        put(a.m + e0, st + off_state + 4 * T, 4 * cnt);
        put(a.v + e0, st + off_state + 8 * T, 4 * cnt);
        if (MODE == kFusedZ3) put(a.param_shard + e0, st, 2 * cnt);
        for (int r = 0; r < N; ++r) put(a.out[r] + e0, st, 2 * cnt);
        if (MODE == kFusedZ1)
          for (int r = 0; r < N; ++r) put(const_cast<uint16_t*>(a.grad[r]) + e0, st + off_g, 2 * cnt);
        if (a.grad_shard) put(a.grad_shard + e0, st + off_g, 2 * cnt);
        bulk_commit();
        bulk_wait_read<0>();  // the copies have read the stage: hand it back to the producer
        mbar_arrive(&empty[s]);
      }
      bulk_wait<0>();  // every store of this CTA performed before the CTA ends
    }
  } else {
    // ----------------------------------------------------------- consumers --
    const int c = threadIdx.x - 64;  // 0 .. 32W-1
    const int j = c * EPT;
    for (int it = 0;; ++it) {
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
      const int64_t e0 = tile * T;
      const int64_t cnt = (n_elem - e0) < T ? (n_elem - e0) : T;
      unsigned char* st = smem + (size_t)s * sb;
      if (j < cnt) {  // cnt is a multiple of 8, so a lane's EPT elements are whole
        V32<EPT> p = ldsf<EPT>(st + off_state + 4 * j);
        V32<EPT> m = ldsf<EPT>(st + off_state + 4 * T + 4 * j);
        V32<EPT> v = ldsf<EPT>(st + off_state + 8 * T + 4 * j);
        H16<EPT> par, gout;
        if constexpr (kMove) {
          // movement only: every slice read, nothing computed but a fold
          uint32_t fold[EPT / 2];
#pragma unroll
          for (int q = 0; q < EPT / 2; ++q) fold[q] = 0u;
          for (int r = 0; r < N; ++r) {
            const H16<EPT> h = lds16<EPT>(st + (size_t)r * 2 * T + 2 * j);
#pragma unroll
            for (int q = 0; q < EPT / 2; ++q) fold[q] ^= h.w[q];
          }
#pragma unroll
          for (int q = 0; q < EPT / 2; ++q) {
            par.w[q] = pack2(F::rn(p.f[2 * q]), F::rn(p.f[2 * q + 1])) ^ (fold[q] & opaque);
            gout.w[q] = fold[q];
          }
        } else {
          float acc[EPT];
#pragma unroll
          for (int q = 0; q < EPT; ++q) acc[q] = 0.0f;
          for (int r = 0; r < N; ++r) {
            const H16<EPT> h = lds16<EPT>(st + (size_t)r * 2 * T + 2 * j);
#pragma unroll
            for (int q = 0; q < EPT / 2; ++q) {
              acc[2 * q] = __fadd_rn(acc[2 * q], F::lo(h.w[q]));
              acc[2 * q + 1] = __fadd_rn(acc[2 * q + 1], F::hi(h.w[q]));
            }
          }
          uint16_t g16[EPT], p16[EPT];
#pragma unroll
          for (int q = 0; q < EPT; ++q) {
            g16[q] = F::rn(__fmul_rn(acc[q], a.inv_n));
            const float g = F::f32(g16[q]);
            const double d = (double)g;
            // the square is exact (at most 11-bit significands, in range), so the
            // fused multiply-add rounds once, as the add after an exact product
            sq = __fma_rn(d, d, sq);
            nf32 += isfinite(g) ? 0u : 1u;
            p16[q] = F::rn(adam1(g, p.f[q], m.f[q], v.f[q], sc));
          }
#pragma unroll
          for (int q = 0; q < EPT / 2; ++q) {
            par.w[q] = pack2(p16[2 * q], p16[2 * q + 1]);
            gout.w[q] = pack2(g16[2 * q], g16[2 * q + 1]);
          }
        }
        stsf<EPT>(st + off_state + 4 * j, p);
        stsf<EPT>(st + off_state + 4 * T + 4 * j, m);
        stsf<EPT>(st + off_state + 8 * T + 4 * j, v);
        sts16<EPT>(st + 2 * j, par);  // over rank 0's slice, which this lane alone read here
        if (need_g) sts16<EPT>(st + off_g + 2 * j, gout);
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
      if (last_k[s] >= 0 && !mbar_wait(&full[s], (unsigned)last_k[s] & 1u)) atomicOr(a.ns.error, 4u);
  }
  if (a.pdl == kPdlEarly || a.pdl == kPdlEarlyLoads) pdl_wait();  // the norm scratch is shared with the grid before
  norm_epilogue<NT>(a.ns, sq, (unsigned long long)nf32, a.accumulate);
}

// The layered stage-3 launch: the kernel above with the tile walk through
// the segments of `g` and the storers' ordering between segments.  A kernel
// of its own: sharing the walk with the one-interval kernel (a template flag)
// made that kernel's stage-1 and stage-2 launches 1.5-6 % slower on B200.
template <class F, int T, int W, bool kMove>
__global__ void __launch_bounds__(32 * (W + 2), 1)
    fused_bulk_layered_kernel(const __grid_constant__ FusedArgs a, int stages, const __grid_constant__ SegTable g) {
  constexpr int MODE = kFusedZ3;
  constexpr bool kLayered = true;
  constexpr uint32_t opaque = 0u;
  constexpr int EPT = T / (32 * W);
  static_assert(EPT == 2 || EPT == 4 || EPT == 8, "2, 4 or 8 elements per consumer lane");
  constexpr int NT = 32 * (W + 2);
  extern __shared__ __align__(128) unsigned char smem[];
  const int N = a.n_ranks;
  const bool need_g = MODE == kFusedZ1 || a.grad_shard != nullptr;
  const unsigned sb = bulk_stage_bytes(N, T, need_g);
  const unsigned off_state = 2u * (unsigned)N * T;  // master; m at +4T, v at +8T
  const unsigned off_g = off_state + 12u * T;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)stages * sb);
  uint64_t* computed = full + stages;
  uint64_t* empty = computed + stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + stages);
  volatile int* last_k = abort_flag + 1;  // last phase of `full` issued per stage, -1 = none
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
  if (a.pdl == kPdlWaitFirst) pdl_wait();

  double sq = 0.0;
  unsigned nf32 = 0;  // non-finite count of this lane (well below 2^32 elements a lane)
  const AdamScalars sc = a.sc_dev ? *a.sc_dev : a.sc;

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      const uint64_t policy = evict_first_policy();
      TileCursor cur;
      for (int it = 0;; ++it) {
        long long e0, ed;
        unsigned cnt;
        if (!cursor_next<T, kLayered>(cur, g, n_tiles, n_elem, e0, ed, cnt) || *abort_flag) break;
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
        fence_proxy_async_smem();  // the stage's last reads (consumers, stores) before the refill
        unsigned char* st = smem + (size_t)s * sb;
        mbar_expect_tx(&full[s], cnt * (unsigned)(2 * N + 12));
        for (int r = 0; r < N; ++r)
          bulk_load(st + (size_t)r * 2 * T, a.grad[r] + e0, (unsigned)(2 * cnt), &full[s], policy);
        bulk_load(st + off_state, a.master + e0, (unsigned)(4 * cnt), &full[s], policy);
        bulk_load(st + off_state + 4 * T, a.m + e0, (unsigned)(4 * cnt), &full[s], policy);
        bulk_load(st + off_state + 8 * T, a.v + e0, (unsigned)(4 * cnt), &full[s], policy);
        last_k[s] = (int)k;
      }
      pdl_trigger();  // no more loads to issue: the next fused launch may start
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------- storer --
    if (lane == 0) {
      bool waited = false;
      const uint64_t spol = evict_first_policy();
      const bool hint = a.store_hint != 0;
      auto put = [&](void* dst, const void* src, unsigned bytes) {
        if (hint) bulk_store(dst, src, bytes, spol);
        else bulk_store(dst, src, bytes);
      };
      TileCursor cur;
      int arrived = 0;  // layered: segments this storer has finished and arrived for
      for (int it = 0;; ++it) {
        long long e0, ed;
        unsigned cnt;
        if (!cursor_next<T, kLayered>(cur, g, n_tiles, n_elem, e0, ed, cnt)) break;
        const int s = it % stages;
        const unsigned k = (unsigned)(it / stages);
        const int w = mbar_wait_or_abort(&computed[s], k & 1u, abort_flag, a.ns.wait_ns);
        if (w != 0) {
          if (w == 1) atomicOr(a.ns.error, 8u);
          *abort_flag = 1;
          break;
        }
        if (a.pdl == kPdlEarlyLoads && !waited) {  // the first store waits for the grid before
          pdl_wait();
          waited = true;
        }
        if constexpr (kLayered) {
          // a new layer: every CTA's stores of the layers before it first
          if (cur.seg > arrived) {
            while (arrived < cur.seg) {
              segment_arrive(g.counter);
              ++arrived;
            }
            if (!segment_wait(g.counter, gridDim.x * (unsigned)cur.seg, abort_flag, a.ns.wait_ns)) {
              atomicOr(a.ns.error, 16u);
              *abort_flag = 1;
              break;
            }
          }
        }
        const unsigned char* st = smem + (size_t)s * sb;
        put(a.master + e0, st + off_state, 4 * cnt);
        put(a.m + e0, st + off_state + 4 * T, 4 * cnt);
        put(a.v + e0, st + off_state + 8 * T, 4 * cnt);
        if (MODE == kFusedZ3) put(a.param_shard + e0, st, 2 * cnt);
        for (int r = 0; r < N; ++r) put(a.out[r] + ed, st, 2 * cnt);
        if (MODE == kFusedZ1)
          for (int r = 0; r < N; ++r) put(const_cast<uint16_t*>(a.grad[r]) + e0, st + off_g, 2 * cnt);
        if (a.grad_shard) put(a.grad_shard + e0, st + off_g, 2 * cnt);
        bulk_commit();
        bulk_wait_read<0>();  // the copies have read the stage: hand it back to the producer
        mbar_arrive(&empty[s]);
      }
      if constexpr (kLayered) {
        // arrive for the layers left (also after an abort: the other CTAs
        // then end without waiting out their limit; the step has failed)
        for (; arrived < g.n; ++arrived) segment_arrive(g.counter);
      }
      bulk_wait<0>();  // every store of this CTA performed before the CTA ends
    }
  } else {
    // ----------------------------------------------------------- consumers --
    const int c = threadIdx.x - 64;  // 0 .. 32W-1
    const int j = c * EPT;
    TileCursor cur;
    for (int it = 0;; ++it) {
      long long e0, ed;
      unsigned cnt;
      if (!cursor_next<T, kLayered>(cur, g, n_tiles, n_elem, e0, ed, cnt)) break;
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
      unsigned char* st = smem + (size_t)s * sb;
      if (j < (int)cnt) {  // cnt is a multiple of 8, so a lane's EPT elements are whole
        V32<EPT> p = ldsf<EPT>(st + off_state + 4 * j);
        V32<EPT> m = ldsf<EPT>(st + off_state + 4 * T + 4 * j);
        V32<EPT> v = ldsf<EPT>(st + off_state + 8 * T + 4 * j);
        H16<EPT> par, gout;
        if constexpr (kMove) {
          // movement only: every slice read, nothing computed but a fold
          uint32_t fold[EPT / 2];
#pragma unroll
          for (int q = 0; q < EPT / 2; ++q) fold[q] = 0u;
          for (int r = 0; r < N; ++r) {
            const H16<EPT> h = lds16<EPT>(st + (size_t)r * 2 * T + 2 * j);
#pragma unroll
            for (int q = 0; q < EPT / 2; ++q) fold[q] ^= h.w[q];
          }
#pragma unroll
          for (int q = 0; q < EPT / 2; ++q) {
            par.w[q] = pack2(F::rn(p.f[2 * q]), F::rn(p.f[2 * q + 1])) ^ (fold[q] & opaque);
            gout.w[q] = fold[q];
          }
        } else {
          float acc[EPT];
#pragma unroll
          for (int q = 0; q < EPT; ++q) acc[q] = 0.0f;
          for (int r = 0; r < N; ++r) {
            const H16<EPT> h = lds16<EPT>(st + (size_t)r * 2 * T + 2 * j);
#pragma unroll
            for (int q = 0; q < EPT / 2; ++q) {
              acc[2 * q] = __fadd_rn(acc[2 * q], F::lo(h.w[q]));
              acc[2 * q + 1] = __fadd_rn(acc[2 * q + 1], F::hi(h.w[q]));
            }
          }
          uint16_t g16[EPT], p16[EPT];
#pragma unroll
          for (int q = 0; q < EPT; ++q) {
            g16[q] = F::rn(__fmul_rn(acc[q], a.inv_n));
            const float g = F::f32(g16[q]);
            const double d = (double)g;
            // the square is exact (at most 11-bit significands, in range), so the
            // fused multiply-add rounds once, as the add after an exact product
            sq = __fma_rn(d, d, sq);
            nf32 += isfinite(g) ? 0u : 1u;
            p16[q] = F::rn(adam1(g, p.f[q], m.f[q], v.f[q], sc));
          }
#pragma unroll
          for (int q = 0; q < EPT / 2; ++q) {
            par.w[q] = pack2(p16[2 * q], p16[2 * q + 1]);
            gout.w[q] = pack2(g16[2 * q], g16[2 * q + 1]);
          }
        }
        stsf<EPT>(st + off_state + 4 * j, p);
        stsf<EPT>(st + off_state + 4 * T + 4 * j, m);
        stsf<EPT>(st + off_state + 8 * T + 4 * j, v);
        sts16<EPT>(st + 2 * j, par);  // over rank 0's slice, which this lane alone read here
        if (need_g) sts16<EPT>(st + off_g + 2 * j, gout);
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
      if (last_k[s] >= 0 && !mbar_wait(&full[s], (unsigned)last_k[s] & 1u)) atomicOr(a.ns.error, 4u);
  }
  if (a.pdl == kPdlEarly || a.pdl == kPdlEarlyLoads) pdl_wait();  // the norm scratch is shared with the grid before
  norm_epilogue<NT>(a.ns, sq, (unsigned long long)nf32, a.accumulate);
}

// --------------------------------------- rank-chunked bulk-store variant --
//
// For N > 16 the N slices of a tile do not fit one stage, so the producer
// streams them through a chunk ring, 8 ranks a chunk stage, and the tile's
// master/m/v through a state ring.  The consumers fold every chunk into their
// fp32 accumulators in rank order (the same additions as the one-stage
// kernel) and release it; after the last chunk they take the tile's state
// stage, update, and write every result back into that stage (master/m/v in
// place, the 16-bit parameters and the averaged gradient into slices of their
// own), which the storer then copies out with bulk stores and releases.
constexpr int kBulkChunkRanks = 8;

__host__ __device__ inline unsigned bulk_chunk_bytes(int tile) { return (unsigned)(kBulkChunkRanks * 2 * tile); }

// [master 4T][m 4T][v 4T][parameters 2T][averaged gradient 2T, when stored]
__host__ __device__ inline unsigned bulk_state_bytes(int tile, bool need_g) {
  return (unsigned)tile * (unsigned)(14 + (need_g ? 2 : 0));
}

__host__ __device__ inline size_t bulk_chunked_smem_bytes(int tile, bool need_g, int cstages, int sstages) {
  return (size_t)cstages * bulk_chunk_bytes(tile) + (size_t)sstages * bulk_state_bytes(tile, need_g) +
         sizeof(uint64_t) * (size_t)(2 * cstages + 3 * sstages) + 4 * (size_t)(1 + cstages + sstages);
}

template <int MODE, class F, int T, int W, bool kMove>
__global__ void __launch_bounds__(32 * (W + 2), 1)
    fused_bulk_chunked_kernel(const __grid_constant__ FusedArgs a, int cstages, int sstages, uint32_t opaque) {
  constexpr int EPT = T / (32 * W);
  static_assert(EPT == 2 || EPT == 4 || EPT == 8, "2, 4 or 8 elements per consumer lane");
  constexpr int NT = 32 * (W + 2);
  extern __shared__ __align__(128) unsigned char smem[];
  const int N = a.n_ranks;
  const int n_chunks = (N + kBulkChunkRanks - 1) / kBulkChunkRanks;
  const bool need_g = MODE == kFusedZ1 || a.grad_shard != nullptr;
  const unsigned cb = bulk_chunk_bytes(T), sb = bulk_state_bytes(T, need_g);
  const unsigned off_par = 12u * T, off_g = 14u * T;
  unsigned char* chunk_base = smem;
  unsigned char* state_base = smem + (size_t)cstages * cb;
  uint64_t* cfull = reinterpret_cast<uint64_t*>(state_base + (size_t)sstages * sb);
  uint64_t* cempty = cfull + cstages;
  uint64_t* sfull = cempty + cstages;
  uint64_t* scomputed = sfull + sstages;
  uint64_t* sempty = scomputed + sstages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sempty + sstages);
  volatile int* last_ck = abort_flag + 1;     // last phase issued per chunk stage, -1 = none
  volatile int* last_sk = last_ck + cstages;  // last phase issued per state stage
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_elem = a.n_vec * kVec;
  const int64_t n_tiles = (n_elem + T - 1) / T;

  if (threadIdx.x == 0) {
    for (int s = 0; s < cstages; ++s) {
      mbar_init(&cfull[s], 1);
      mbar_init(&cempty[s], W);
      last_ck[s] = -1;
    }
    for (int s = 0; s < sstages; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&scomputed[s], W);
      mbar_init(&sempty[s], 1);
      last_sk[s] = -1;
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (a.pdl == kPdlWaitFirst) pdl_wait();

  double sq = 0.0;
  unsigned nf32 = 0;  // non-finite count of this lane (well below 2^32 elements a lane)
  const AdamScalars sc = a.sc_dev ? *a.sc_dev : a.sc;

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      const uint64_t policy = evict_first_policy();
      for (int it = 0;; ++it) {
        const int64_t tile = blockIdx.x + (int64_t)it * gridDim.x;
        if (tile >= n_tiles || *abort_flag) break;
        const int64_t e0 = tile * T;
        const int64_t cnt = (n_elem - e0) < T ? (n_elem - e0) : T;
        const int ss = it % sstages;
        const unsigned sk = (unsigned)(it / sstages);
        if (sk > 0) {
          const int w = mbar_wait_or_abort(&sempty[ss], (sk - 1) & 1u, abort_flag, a.ns.wait_ns);
          if (w != 0) {
            if (w == 1) atomicOr(a.ns.error, 1u);
            *abort_flag = 1;
            break;
          }
        }
        fence_proxy_async_smem();
        unsigned char* stt = state_base + (size_t)ss * sb;
        mbar_expect_tx(&sfull[ss], (unsigned)(12 * cnt));
        bulk_load(stt, a.master + e0, (unsigned)(4 * cnt), &sfull[ss], policy);
        bulk_load(stt + 4 * T, a.m + e0, (unsigned)(4 * cnt), &sfull[ss], policy);
        bulk_load(stt + 8 * T, a.v + e0, (unsigned)(4 * cnt), &sfull[ss], policy);
        last_sk[ss] = (int)sk;
        bool stop = false;
        for (int c = 0; c < n_chunks; ++c) {
          const int ci = it * n_chunks + c;
          const int cs = ci % cstages;
          const unsigned ck = (unsigned)(ci / cstages);
          if (ck > 0) {
            const int w = mbar_wait_or_abort(&cempty[cs], (ck - 1) & 1u, abort_flag, a.ns.wait_ns);
            if (w != 0) {
              if (w == 1) atomicOr(a.ns.error, 1u);
              *abort_flag = 1;
              stop = true;
              break;
            }
          }
          fence_proxy_async_smem();
          const int r0 = c * kBulkChunkRanks;
          const int r1 = (r0 + kBulkChunkRanks) < N ? (r0 + kBulkChunkRanks) : N;
          unsigned char* st = chunk_base + (size_t)cs * cb;
          mbar_expect_tx(&cfull[cs], (unsigned)((r1 - r0) * 2 * cnt));
          for (int r = r0; r < r1; ++r)
            bulk_load(st + (size_t)(r - r0) * 2 * T, a.grad[r] + e0, (unsigned)(2 * cnt), &cfull[cs], policy);
          last_ck[cs] = (int)ck;
        }
        if (stop) break;
      }
      pdl_trigger();  // no more loads to issue: the next fused launch may start
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------- storer --
    if (lane == 0) {
      bool waited = false;
      const uint64_t spol = evict_first_policy();
      const bool hint = a.store_hint != 0;
      auto put = [&](void* dst, const void* src, unsigned bytes) {
        if (hint) bulk_store(dst, src, bytes, spol);
        else bulk_store(dst, src, bytes);
      };
      for (int it = 0;; ++it) {
        const int64_t tile = blockIdx.x + (int64_t)it * gridDim.x;
        if (tile >= n_tiles) break;
        const int ss = it % sstages;
        const unsigned sk = (unsigned)(it / sstages);
        const int w = mbar_wait_or_abort(&scomputed[ss], sk & 1u, abort_flag, a.ns.wait_ns);
        if (w != 0) {
          if (w == 1) atomicOr(a.ns.error, 8u);
          *abort_flag = 1;
          break;
        }
        if (a.pdl == kPdlEarlyLoads && !waited) {  // the first store waits for the grid before
          pdl_wait();
          waited = true;
        }
        const int64_t e0 = tile * T;
        const unsigned cnt = (unsigned)((n_elem - e0) < T ? (n_elem - e0) : T);
        const unsigned char* stt = state_base + (size_t)ss * sb;
        put(a.master + e0, stt, 4 * cnt);
        put(a.m + e0, stt + 4 * T, 4 * cnt);
        put(a.v + e0, stt + 8 * T, 4 * cnt);
        if (MODE == kFusedZ3) put(a.param_shard + e0, stt + off_par, 2 * cnt);
        for (int r = 0; r < N; ++r) put(a.out[r] + e0, stt + off_par, 2 * cnt);
        if (MODE == kFusedZ1)
          for (int r = 0; r < N; ++r) put(const_cast<uint16_t*>(a.grad[r]) + e0, stt + off_g, 2 * cnt);
        if (a.grad_shard) put(a.grad_shard + e0, stt + off_g, 2 * cnt);
        bulk_commit();
        bulk_wait_read<0>();  // the copies have read the stage: hand it back to the producer
        mbar_arrive(&sempty[ss]);
      }
      bulk_wait<0>();  // every store of this CTA performed before the CTA ends
    }
  } else {
    // ----------------------------------------------------------- consumers --
    const int c_id = threadIdx.x - 64;
    const int j = c_id * EPT;
    bool aborted = false;
    for (int it = 0; !aborted; ++it) {
      const int64_t tile = blockIdx.x + (int64_t)it * gridDim.x;
      if (tile >= n_tiles) break;
      const int64_t e0 = tile * T;
      const int64_t cnt = (n_elem - e0) < T ? (n_elem - e0) : T;
      const bool active = j < cnt;  // cnt is a multiple of 8, so a lane's EPT elements are whole
      float acc[EPT];
      uint32_t fold[EPT / 2];
#pragma unroll
      for (int q = 0; q < EPT; ++q) acc[q] = 0.0f;
#pragma unroll
      for (int q = 0; q < EPT / 2; ++q) fold[q] = 0u;
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
        const int r0 = c * kBulkChunkRanks;
        const int r1 = (r0 + kBulkChunkRanks) < N ? (r0 + kBulkChunkRanks) : N;
        const unsigned char* st = chunk_base + (size_t)cs * cb;
        if (active) {
          for (int r = r0; r < r1; ++r) {
            const H16<EPT> h = lds16<EPT>(st + (size_t)(r - r0) * 2 * T + 2 * j);
#pragma unroll
            for (int q = 0; q < EPT / 2; ++q) {
              if constexpr (kMove) {
                fold[q] ^= h.w[q];
              } else {
                acc[2 * q] = __fadd_rn(acc[2 * q], F::lo(h.w[q]));
                acc[2 * q + 1] = __fadd_rn(acc[2 * q + 1], F::hi(h.w[q]));
              }
            }
          }
        }
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
      unsigned char* stt = state_base + (size_t)ss * sb;
      if (active) {
        V32<EPT> p = ldsf<EPT>(stt + 4 * j);
        V32<EPT> m = ldsf<EPT>(stt + 4 * T + 4 * j);
        V32<EPT> v = ldsf<EPT>(stt + 8 * T + 4 * j);
        H16<EPT> par, gout;
        if constexpr (kMove) {
#pragma unroll
          for (int q = 0; q < EPT / 2; ++q) {
            par.w[q] = pack2(F::rn(p.f[2 * q]), F::rn(p.f[2 * q + 1])) ^ (fold[q] & opaque);
            gout.w[q] = fold[q];
          }
        } else {
          uint16_t g16[EPT], p16[EPT];
#pragma unroll
          for (int q = 0; q < EPT; ++q) {
            g16[q] = F::rn(__fmul_rn(acc[q], a.inv_n));
            const float g = F::f32(g16[q]);
            const double d = (double)g;
            // the square is exact (at most 11-bit significands, in range), so the
            // fused multiply-add rounds once, as the add after an exact product
            sq = __fma_rn(d, d, sq);
            nf32 += isfinite(g) ? 0u : 1u;
            p16[q] = F::rn(adam1(g, p.f[q], m.f[q], v.f[q], sc));
          }
#pragma unroll
          for (int q = 0; q < EPT / 2; ++q) {
            par.w[q] = pack2(p16[2 * q], p16[2 * q + 1]);
            gout.w[q] = pack2(g16[2 * q], g16[2 * q + 1]);
          }
        }
        stsf<EPT>(stt + 4 * j, p);
        stsf<EPT>(stt + 4 * T + 4 * j, m);
        stsf<EPT>(stt + 8 * T + 4 * j, v);
        sts16<EPT>(stt + off_par + 2 * j, par);
        if (need_g) sts16<EPT>(stt + off_g + 2 * j, gout);
      }
      fence_proxy_async_smem();  // this lane's stage writes before the storer's bulk copies read them
      __syncwarp();
      if (lane == 0) mbar_arrive(&scomputed[ss]);
    }
  }
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    // drain the bulk loads already issued before the CTA's memory goes away
    for (int s = 0; s < cstages; ++s)
      if (last_ck[s] >= 0 && !mbar_wait(&cfull[s], (unsigned)last_ck[s] & 1u)) atomicOr(a.ns.error, 4u);
    for (int s = 0; s < sstages; ++s)
      if (last_sk[s] >= 0 && !mbar_wait(&sfull[s], (unsigned)last_sk[s] & 1u)) atomicOr(a.ns.error, 4u);
  }
  if (a.pdl == kPdlEarly || a.pdl == kPdlEarlyLoads) pdl_wait();  // the norm scratch is shared with the grid before
  norm_epilogue<NT>(a.ns, sq, (unsigned long long)nf32, a.accumulate);
}

// A programmatic dependent launch may place its CTAs while the grid before it
// still runs; these kernels are persistent (tiles dealt by CTA index), so a
// launch with the attribute asks for more than half an SM's shared memory and
// a dependent grid's CTAs land only on SMs the grid before has left.
constexpr size_t kPdlSoloSmemBulk = 116 * 1024;

template <int MODE, class F, int T, int W, bool kMove>
cudaError_t launch_cfg(const FusedArgs& a, int grid, int stages, int sstages, size_t bytes, uint32_t opaque,
                       cudaStream_t s) {
  (void)sstages;
  return launch_kernel(fused_bulk_kernel<MODE, F, T, W, kMove>, grid, 32 * (W + 2), bytes, s, a.pdl != kPdlNone,
                       a, stages, opaque);
}

// The layered stage-3 launch: cooperative, so that every CTA is resident at
// once (its storers wait on one another's progress), and one CTA per SM.
template <class F, int T, int W, bool kMove>
cudaError_t launch_layered_cfg(const FusedArgs& a, const SegTable& g, int grid, int stages, size_t bytes,
                               cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)(32 * (W + 2)));
  cfg.dynamicSmemBytes = bytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fused_bulk_layered_kernel<F, T, W, kMove>, a, stages, g);
}

template <int MODE, class F, int T, int W, bool kMove>
cudaError_t launch_chunked_cfg(const FusedArgs& a, int grid, int cstages, int sstages, size_t bytes,
                               uint32_t opaque, cudaStream_t s) {
  return launch_kernel(fused_bulk_chunked_kernel<MODE, F, T, W, kMove>, grid, 32 * (W + 2), bytes, s,
                       a.pdl != kPdlNone, a, cstages, sstages, opaque);
}

// The (tile, consumer warps) configurations built.  One-stage kernel (N <=
// 16): 2048 x 8 and 1024 x 4 (8 elements a lane), 2048 x 16 and 1024 x 8 (4
// a lane), 1024 x 16 (2).  Rank-chunked kernel (N > 16): 2048 x 8, 1024 x 8.
#define ZSM_BULK_CONFIGS(X) X(2048, 8) X(2048, 16) X(1024, 4) X(1024, 8) X(1024, 16)
#define ZSM_BULK_CHUNKED_CONFIGS(X) X(2048, 8) X(1024, 8)

template <int MODE, class F, bool kMove>
cudaError_t launch_mode_fmt(const FusedArgs& a, int grid, int tile, int warps, int stages, int sstages,
                            size_t bytes, uint32_t opaque, cudaStream_t s) {
  if (a.n_ranks > kTmaMaxRanks) {
#define ZSM_BULK_CASE(TT, WW)                                                                        \
  if (tile == TT && warps == WW)                                                                     \
    return launch_chunked_cfg<MODE, F, TT, WW, kMove>(a, grid, stages, sstages, bytes, opaque, s);
    ZSM_BULK_CHUNKED_CONFIGS(ZSM_BULK_CASE)
#undef ZSM_BULK_CASE
    return cudaErrorInvalidValue;
  }
#define ZSM_BULK_CASE(TT, WW) \
  if (tile == TT && warps == WW) return launch_cfg<MODE, F, TT, WW, kMove>(a, grid, stages, sstages, bytes, opaque, s);
  ZSM_BULK_CONFIGS(ZSM_BULK_CASE)
#undef ZSM_BULK_CASE
  return cudaErrorInvalidValue;
}

template <int MODE>
cudaError_t launch_mode(const FusedArgs& a, int grid, int tile, int warps, int stages, int sstages, size_t bytes,
                        bool move, uint32_t opaque, cudaStream_t s) {
  if (move) return launch_mode_fmt<MODE, Bf16, true>(a, grid, tile, warps, stages, sstages, bytes, opaque, s);
  if (a.fmt == kFmtF16)
    return launch_mode_fmt<MODE, F16, false>(a, grid, tile, warps, stages, sstages, bytes, opaque, s);
  return launch_mode_fmt<MODE, Bf16, false>(a, grid, tile, warps, stages, sstages, bytes, opaque, s);
}

template <class K>
cudaError_t opt_in(K kernel) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTmaMaxSmem);
}

template <int MODE, class F, bool kMove>
cudaError_t configure_mode_fmt() {
  cudaError_t e = cudaSuccess;
#define ZSM_BULK_OPT(TT, WW)                                                          \
  if (e == cudaSuccess) e = opt_in(fused_bulk_kernel<MODE, F, TT, WW, kMove>);        \
  if (MODE == kFusedZ3 && e == cudaSuccess) e = opt_in(fused_bulk_layered_kernel<F, TT, WW, kMove>);
  ZSM_BULK_CONFIGS(ZSM_BULK_OPT)
#undef ZSM_BULK_OPT
#define ZSM_BULK_OPT(TT, WW) \
  if (e == cudaSuccess) e = opt_in(fused_bulk_chunked_kernel<MODE, F, TT, WW, kMove>);
  ZSM_BULK_CHUNKED_CONFIGS(ZSM_BULK_OPT)
#undef ZSM_BULK_OPT
  return e;
}

template <int MODE>
cudaError_t configure_mode() {
  cudaError_t e = configure_mode_fmt<MODE, Bf16, false>();
  if (e == cudaSuccess) e = configure_mode_fmt<MODE, F16, false>();
  if (e == cudaSuccess) e = configure_mode_fmt<MODE, Bf16, true>();
  return e;
}

// Ring depths of the rank-chunked kernel: chunk stages (at most max_cstages
// when given) and state stages, the most that fit; false when nothing fits.
bool chunked_rings(int tile, bool need_g, int max_cstages, int* cstages, int* sstages) {
  int cs = max_cstages > 0 ? std::min(max_cstages, kTmaMaxStages) : (tile >= 2048 ? 3 : 6);
  int ss = tile >= 2048 ? 2 : 3;
  while (cs > 2 && bulk_chunked_smem_bytes(tile, need_g, cs, ss) > (size_t)kTmaMaxSmem) --cs;
  while (ss > 2 && bulk_chunked_smem_bytes(tile, need_g, cs, ss) > (size_t)kTmaMaxSmem) --ss;
  if (bulk_chunked_smem_bytes(tile, need_g, cs, ss) > (size_t)kTmaMaxSmem) return false;
  *cstages = cs;
  *sstages = ss;
  return true;
}

}  // namespace

bool bulk_config_valid(int n_ranks, int tile, int warps) {
  if (n_ranks > kTmaMaxRanks) {
#define ZSM_BULK_VALID(TT, WW) \
  if (tile == TT && warps == WW) return true;
    ZSM_BULK_CHUNKED_CONFIGS(ZSM_BULK_VALID)
#undef ZSM_BULK_VALID
    return false;
  }
#define ZSM_BULK_VALID(TT, WW) \
  if (tile == TT && warps == WW) return true;
  ZSM_BULK_CONFIGS(ZSM_BULK_VALID)
#undef ZSM_BULK_VALID
  return false;
}

int bulk_stages_for(int n_ranks, int tile, bool need_g, int max_stages) {
  if (n_ranks < 1 || n_ranks > kMaxRanks) return 0;
  if (n_ranks > kTmaMaxRanks) {
    int cs = 0, ss = 0;
    return chunked_rings(tile, need_g, max_stages, &cs, &ss) ? cs : 0;
  }
  int stages = max_stages > 0 ? std::min(max_stages, kTmaMaxStages) : kTmaMaxStages;
  while (stages > 0 && bulk_smem_bytes(n_ranks, tile, need_g, stages) > (size_t)kTmaMaxSmem) --stages;
  return stages >= 2 ? stages : 0;
}

cudaError_t bulk_configure() {
  cudaError_t e = configure_mode<kFusedZ1>();
  if (e == cudaSuccess) e = configure_mode<kFusedZ2>();
  if (e == cudaSuccess) e = configure_mode<kFusedZ3>();
  return e;
}

cudaError_t launch_fused_bulk(int mode, const FusedArgs& a, int grid, int tile, int warps, int max_stages, bool move,
                              uint32_t opaque, cudaStream_t s) {
  const bool need_g = mode == kFusedZ1 || a.grad_shard != nullptr;
  if (!bulk_config_valid(a.n_ranks, tile, warps)) return cudaErrorInvalidValue;
  int stages = 0, sstages = 0;
  size_t bytes = 0;
  if (a.n_ranks > kTmaMaxRanks) {
    if (!chunked_rings(tile, need_g, max_stages, &stages, &sstages)) return cudaErrorInvalidValue;
    bytes = bulk_chunked_smem_bytes(tile, need_g, stages, sstages);
  } else {
    stages = bulk_stages_for(a.n_ranks, tile, need_g, max_stages);
    if (stages == 0) return cudaErrorInvalidValue;
    bytes = bulk_smem_bytes(a.n_ranks, tile, need_g, stages);
  }
  if (a.pdl != kPdlNone && bytes < kPdlSoloSmemBulk) bytes = kPdlSoloSmemBulk;
  switch (mode) {
    case kFusedZ1: return launch_mode<kFusedZ1>(a, grid, tile, warps, stages, sstages, bytes, move, opaque, s);
    case kFusedZ2: return launch_mode<kFusedZ2>(a, grid, tile, warps, stages, sstages, bytes, move, opaque, s);
    case kFusedZ3: return launch_mode<kFusedZ3>(a, grid, tile, warps, stages, sstages, bytes, move, opaque, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_fused_bulk_layered(const FusedArgs& a, const SegTable& g, int grid, int tile, int warps,
                                      int max_stages, bool move, cudaStream_t s) {
  if (a.n_ranks < 1 || a.n_ranks > kTmaMaxRanks || g.n < 1 || g.n > kMaxSegments || !g.counter ||
      a.pdl != kPdlNone)
    return cudaErrorInvalidValue;
  const bool need_g = a.grad_shard != nullptr;
  const int stages = bulk_stages_for(a.n_ranks, tile, need_g, max_stages);
  if (stages == 0) return cudaErrorInvalidValue;
  size_t bytes = bulk_smem_bytes(a.n_ranks, tile, need_g, stages);
  if (bytes < kPdlSoloSmemBulk) bytes = kPdlSoloSmemBulk;  // one CTA per SM: tiles are dealt by CTA index
#define ZSM_BULK_CASE(TT, WW)                                                                   \
  if (tile == TT && warps == WW) {                                                              \
    if (move) return launch_layered_cfg<Bf16, TT, WW, true>(a, g, grid, stages, bytes, s);      \
    if (a.fmt == kFmtF16) return launch_layered_cfg<F16, TT, WW, false>(a, g, grid, stages, bytes, s); \
    return launch_layered_cfg<Bf16, TT, WW, false>(a, g, grid, stages, bytes, s);               \
  }
  ZSM_BULK_CONFIGS(ZSM_BULK_CASE)
#undef ZSM_BULK_CASE
  return cudaErrorInvalidValue;
}

}  // namespace zsm
