// Device helpers shared by the ZeRO step kernels: streaming accesses, bf16
// packing, the rank-order reduction, the Adam update and the per-launch
// gradient-norm epilogue.
//
// Numerics (identical on every path): the averaged gradient of element i is
//   acc = +0;  for r = 0..N-1: acc = acc + f32(g_r[i])      (binary32, RN)
//   g_i = bf16_rn(acc * fp32(1/N))
// and Adam runs with one correctly rounded binary32 operation per step of
//   p = p*decay; m = b1*m + omb1*g; v = b2*v + omb2*(g*g);
//   p = p - lr*((m/bc1) / (sqrt(v/bc2) + eps))
// (bias-corrected Adam with decoupled weight decay; the ZeRO pages -- "ZERO训练
// 技术" sections "ZeRO-1"/"ZeRO-2"/"ZeRO-3" -- name Adam on the owned shard
// without printing its equations).  The __f*_rn intrinsics keep every operation
// separately rounded: no multiply-add contraction, no flush to zero.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "kernels.cuh"

namespace zsm {
namespace dev {

// ------------------------------------------------------------ memory access --

// Streaming 16-byte accesses: every byte of the step is touched exactly once,
// so loads and stores are marked evict-first and nothing is kept in L1.
__device__ __forceinline__ uint4 ld_stream(const uint16_t* p) {
  return __ldcs(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ float4 ld_stream(const float* p) {
  return __ldcs(reinterpret_cast<const float4*>(p));
}
__device__ __forceinline__ void st_stream(uint16_t* p, uint4 v) {
  __stcs(reinterpret_cast<uint4*>(p), v);
}
__device__ __forceinline__ void st_stream(float* p, float4 v) {
  __stcs(reinterpret_cast<float4*>(p), v);
}

// ------------------------------------------------------------- bf16 helpers --

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint16_t to_bf16(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// The two 16-bit storage formats: decode the low / high half of a 32-bit word
// (exact), decode one value, round a binary32 to the format (nearest even).
struct Bf16 {
  static __device__ __forceinline__ float lo(uint32_t w) { return __uint_as_float(w << 16); }
  static __device__ __forceinline__ float hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
  static __device__ __forceinline__ float f32(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }
  static __device__ __forceinline__ uint16_t rn(float x) { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }
};

struct F16 {
  static __device__ __forceinline__ float lo(uint32_t w) {
    return __half2float(__ushort_as_half((unsigned short)(w & 0xFFFFu)));
  }
  static __device__ __forceinline__ float hi(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w >> 16))); }
  static __device__ __forceinline__ float f32(uint16_t h) { return __half2float(__ushort_as_half(h)); }
  static __device__ __forceinline__ uint16_t rn(float x) { return __half_as_ushort(__float2half_rn(x)); }
};

__device__ __forceinline__ uint32_t pack2(uint16_t lo, uint16_t hi) {
  return (uint32_t)lo | ((uint32_t)hi << 16);
}

__device__ __forceinline__ uint4 pack8(const uint16_t (&h)[kVec]) {
  return make_uint4(pack2(h[0], h[1]), pack2(h[2], h[3]), pack2(h[4], h[5]), pack2(h[6], h[7]));
}

template <class F = Bf16>
__device__ __forceinline__ void add8(float (&acc)[kVec], uint4 w) {
  acc[0] = __fadd_rn(acc[0], F::lo(w.x));
  acc[1] = __fadd_rn(acc[1], F::hi(w.x));
  acc[2] = __fadd_rn(acc[2], F::lo(w.y));
  acc[3] = __fadd_rn(acc[3], F::hi(w.y));
  acc[4] = __fadd_rn(acc[4], F::lo(w.z));
  acc[5] = __fadd_rn(acc[5], F::hi(w.z));
  acc[6] = __fadd_rn(acc[6], F::lo(w.w));
  acc[7] = __fadd_rn(acc[7], F::hi(w.w));
}

// ------------------------------------------ programmatic dependent launch --

// Waits until the grids this one depends on have completed and their memory
// operations are visible; returns at once for a launch without the
// programmatic attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Lets the dependent grid launch once every CTA of this grid has issued this
// or exited (later calls in the same CTA have no further effect).
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------- rank-order reduce --

// acc[j] = sum over r = 0..n-1 of grad[r][e + j], in rank order.  Ranks are
// loaded in groups of 8 (eight 16-byte loads in flight per lane).  With more
// than 8 ranks (kMulti) the next group's loads are issued before the current
// group is added, which costs a second 8-vector buffer of registers.
template <bool kMulti, class F = Bf16, class PtrArray>
__device__ __forceinline__ void reduce_ranks(const PtrArray& grad, int n, int64_t e,
                                             float (&acc)[kVec]) {
#pragma unroll
  for (int j = 0; j < kVec; ++j) acc[j] = 0.0f;
  uint4 cur[8];
#pragma unroll
  for (int k = 0; k < 8; ++k)
    if (k < n) cur[k] = ld_stream(grad[k] + e);
  if constexpr (!kMulti) {
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (k < n) add8<F>(acc, cur[k]);
  } else {
    uint4 nxt[8];
    for (int r0 = 0; r0 < n; r0 += 8) {
      const int r1 = r0 + 8;
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (r1 + k < n) nxt[k] = ld_stream(grad[r1 + k] + e);
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (r0 + k < n) add8<F>(acc, cur[k]);
#pragma unroll
      for (int k = 0; k < 8; ++k) cur[k] = nxt[k];
    }
  }
}

// Mean, rounding to the 16-bit format, and the norm / non-finite tallies of
// one vector (of the stored, still loss-scaled, averaged gradient).
template <class F = Bf16>
__device__ __forceinline__ void mean_bf16(const float (&acc)[kVec], float inv_n,
                                          uint16_t (&g16)[kVec], float (&g)[kVec], double& sq,
                                          unsigned long long& nf) {
#pragma unroll
  for (int j = 0; j < kVec; ++j) {
    g16[j] = F::rn(__fmul_rn(acc[j], inv_n));
    g[j] = F::f32(g16[j]);
    const double d = (double)g[j];
    sq = __dadd_rn(sq, __dmul_rn(d, d));  // each square exact (at most 11-bit significands)
    nf += isfinite(g[j]) ? 0ull : 1ull;
  }
}

// ------------------------------------------------------------------- Adam --

// The 16-bit rounding of 8 fp32 values (the parameters of unchanged masters).
template <class F>
__device__ __forceinline__ uint4 round8(const float4& p0, const float4& p1) {
  return make_uint4((uint32_t)F::rn(p0.x) | ((uint32_t)F::rn(p0.y) << 16),
                    (uint32_t)F::rn(p0.z) | ((uint32_t)F::rn(p0.w) << 16),
                    (uint32_t)F::rn(p1.x) | ((uint32_t)F::rn(p1.y) << 16),
                    (uint32_t)F::rn(p1.z) | ((uint32_t)F::rn(p1.w) << 16));
}

// Folds the clipped step's decision into the scalars: the coefficient when
// below 1; returns whether the step is skipped.  `dec` may be null.
__device__ __forceinline__ bool apply_decision(const ClipDecision* dec, AdamScalars& sc) {
  if (!dec) return false;
  const float coef = dec->coef;
  if (coef < 1.0f) {
    sc.coef = coef;
    sc.flags |= kClip;
  }
  return dec->skip != 0;
}

__device__ __forceinline__ float adam1(float g, float& p, float& m, float& v,
                                       const AdamScalars& s) {
  if (s.flags & kUnscale) g = __fmul_rn(g, s.inv_scale);  // loss scale first,
  if (s.flags & kClip) g = __fmul_rn(g, s.coef);          // then the clipping coefficient
  p = __fmul_rn(p, s.decay);
  m = __fadd_rn(__fmul_rn(s.b1, m), __fmul_rn(s.omb1, g));
  v = __fadd_rn(__fmul_rn(s.b2, v), __fmul_rn(s.omb2, __fmul_rn(g, g)));
  const float mh = __fdiv_rn(m, s.bc1);
  const float vh = __fdiv_rn(v, s.bc2);
  const float den = __fadd_rn(__fsqrt_rn(vh), s.eps);
  p = __fsub_rn(p, __fmul_rn(s.lr, __fdiv_rn(mh, den)));
  return p;
}

// Adam on 8 consecutive elements: state vectors in, 16-bit params out.
template <class F = Bf16>
__device__ __forceinline__ void adam8(const float (&g)[kVec], float4& p0, float4& p1, float4& m0,
                                      float4& m1, float4& v0, float4& v1, const AdamScalars& s,
                                      uint16_t (&out)[kVec]) {
  out[0] = F::rn(adam1(g[0], p0.x, m0.x, v0.x, s));
  out[1] = F::rn(adam1(g[1], p0.y, m0.y, v0.y, s));
  out[2] = F::rn(adam1(g[2], p0.z, m0.z, v0.z, s));
  out[3] = F::rn(adam1(g[3], p0.w, m0.w, v0.w, s));
  out[4] = F::rn(adam1(g[4], p1.x, m1.x, v1.x, s));
  out[5] = F::rn(adam1(g[5], p1.y, m1.y, v1.y, s));
  out[6] = F::rn(adam1(g[6], p1.z, m1.z, v1.z, s));
  out[7] = F::rn(adam1(g[7], p1.w, m1.w, v1.w, s));
}

// ------------------------------------------------------- norm epilogue --

// Per-CTA partials, then the last CTA to finish sums them in index order and
// folds the result into the step accumulator (written on a step's first
// launch, added on later ones).  Deterministic for a fixed grid; no waits.
// NT is the block size; every thread of the block must call it.
template <int NT>
__device__ __forceinline__ void norm_epilogue(const NormScratch& ns, double sq, unsigned long long nf,
                                              int accumulate) {
  constexpr int kWarps = NT / 32;
  __shared__ double s_sq[kWarps];
  __shared__ unsigned long long s_nf[kWarps];
  __shared__ int s_last;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sq = __dadd_rn(sq, __shfl_xor_sync(0xFFFFFFFFu, sq, o));
    nf += __shfl_xor_sync(0xFFFFFFFFu, nf, o);
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) {
    s_sq[warp] = sq;
    s_nf[warp] = nf;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double b = 0.0;
    unsigned long long c = 0;
    for (int w = 0; w < kWarps; ++w) {
      b = __dadd_rn(b, s_sq[w]);
      c += s_nf[w];
    }
    ns.partial_sq[blockIdx.x] = b;
    ns.partial_nf[blockIdx.x] = c;
    __threadfence();
    const unsigned int prev = atomicAdd(ns.done, 1u);
    s_last = (prev == gridDim.x - 1) ? 1 : 0;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  double b = 0.0;
  unsigned long long c = 0;
  for (int i = threadIdx.x; i < (int)gridDim.x; i += NT) {
    b = __dadd_rn(b, __ldcg(ns.partial_sq + i));
    c += __ldcg(ns.partial_nf + i);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    b = __dadd_rn(b, __shfl_xor_sync(0xFFFFFFFFu, b, o));
    c += __shfl_xor_sync(0xFFFFFFFFu, c, o);
  }
  __syncthreads();
  if (lane == 0) {
    s_sq[warp] = b;
    s_nf[warp] = c;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double tb = 0.0;
    unsigned long long tc = 0;
    for (int w = 0; w < kWarps; ++w) {
      tb = __dadd_rn(tb, s_sq[w]);
      tc += s_nf[w];
    }
    if (accumulate) {
      *ns.step_sq = __dadd_rn(*ns.step_sq, tb);
      *ns.step_nf += tc;
    } else {
      *ns.step_sq = tb;
      *ns.step_nf = tc;
    }
    *ns.done = 0u;
    __threadfence();
  }
}

}  // namespace dev
}  // namespace zsm
