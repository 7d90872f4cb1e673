// Register-path kernels of the ZeRO optimizer step (sm_100a): the fused step
// for any N (loads straight into registers), the unfused reduce-scatter /
// all-reduce, Adam, all-gather and the state initialisation.  Arithmetic and
// helpers are in device_math.cuh.
//
// What each computes follows "ZERO训练技术": the all-reduce of section
// "ZeRO-1" (part "2. 反向") and the reduce-scatter of section "ZeRO-2"
// (the N ranks' gradients summed and averaged, each owner keeping its
// shard), the owner's Adam update of its shard (sections "ZeRO-1" to
// "ZeRO-3", part "3. 更新") and the all-gather of the updated 16-bit
// parameters into every rank's copy (section "ZeRO-1", part "all-gather 是
// 什么"; section "ZeRO-3" for the temporary full-layer buffers).  The fused
// kernel does the three in one pass per element, since the N ranks are
// buffers of one GPU.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "device_math.cuh"
#include "kernels.cuh"

namespace zsm {
namespace {

using namespace dev;

// ------------------------------------------------------------ fused step --

// One pass over [lo, hi): read the N gradient replicas once, reduce in rank
// order, run Adam in registers, write master/m/v once, and write the bf16
// parameters to every rank's destination.
//   kFusedZ1: also writes the averaged gradient back to the N replicas (the
//             all-reduce result every rank keeps under ZeRO-1).
//   kFusedZ2: parameters to the N replicas (reduce-scatter + update +
//             all-gather).
//   kFusedZ3: parameters to the owner's shard and the N temporary layer
//             buffers.
template <int MODE, bool kMulti, class F>
__global__ void __launch_bounds__(kThreads) fused_step_kernel(const __grid_constant__ FusedArgs a) {
  double sq = 0.0;
  unsigned long long nf = 0;
  if (a.pdl == kPdlWaitFirst) pdl_wait();  // before any global access, the step's scalars included
  const AdamScalars sc = a.sc_dev ? *a.sc_dev : a.sc;
  bool waited = false;
  // every CTA is resident from the start (the grid is sized to the SM count),
  // so the next fused launch may be scheduled as soon as CTAs exit
  pdl_trigger();
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  for (int64_t vi = (int64_t)blockIdx.x * kThreads + threadIdx.x; vi < a.n_vec; vi += stride) {
    const int64_t e = vi * kVec;
    float4 p0 = ld_stream(a.master + e), p1 = ld_stream(a.master + e + 4);
    float4 m0 = ld_stream(a.m + e), m1 = ld_stream(a.m + e + 4);
    float4 v0 = ld_stream(a.v + e), v1 = ld_stream(a.v + e + 4);
    float acc[kVec];
    reduce_ranks<kMulti, F>(a.grad, a.n_ranks, e, acc);
    uint16_t g16[kVec];
    float g[kVec];
    mean_bf16<F>(acc, a.inv_n, g16, g, sq, nf);
    if (a.pdl == kPdlEarlyLoads && !waited) {  // the first store waits for the grid before
      pdl_wait();
      waited = true;
    }
    if (MODE == kFusedZ1) {
      const uint4 gw = pack8(g16);
      for (int r = 0; r < a.n_ranks; ++r) st_stream(const_cast<uint16_t*>(a.grad[r]) + e, gw);
    }
    if (a.grad_shard) st_stream(a.grad_shard + e, pack8(g16));
    uint16_t p16[kVec];
    adam8<F>(g, p0, p1, m0, m1, v0, v1, sc, p16);
    st_stream(a.master + e, p0);
    st_stream(a.master + e + 4, p1);
    st_stream(a.m + e, m0);
    st_stream(a.m + e + 4, m1);
    st_stream(a.v + e, v0);
    st_stream(a.v + e + 4, v1);
    const uint4 pw = pack8(p16);
    if (MODE == kFusedZ3) st_stream(a.param_shard + e, pw);
    for (int r = 0; r < a.n_ranks; ++r) st_stream(a.out[r] + e, pw);
  }
  if (a.pdl == kPdlEarly || a.pdl == kPdlEarlyLoads) pdl_wait();  // the norm scratch is shared with the grid before
  norm_epilogue<kThreads>(a.ns, sq, nf, a.accumulate);
}

// ------------------------------------------------------ unfused kernels --

template <bool kMulti, class F>
__global__ void __launch_bounds__(kThreads) reduce_kernel(const __grid_constant__ ReduceArgs a) {
  double sq = 0.0;
  unsigned long long nf = 0;
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  for (int64_t vi = (int64_t)blockIdx.x * kThreads + threadIdx.x; vi < a.n_vec; vi += stride) {
    const int64_t e = vi * kVec;
    float acc[kVec];
    reduce_ranks<kMulti, F>(a.grad, a.n_ranks, e, acc);
    uint16_t g16[kVec];
    float g[kVec];
    mean_bf16<F>(acc, a.inv_n, g16, g, sq, nf);
    const uint4 gw = pack8(g16);
    if (a.shard_out) st_stream(a.shard_out + e, gw);
    if (a.write_back)
      for (int r = 0; r < a.n_ranks; ++r) st_stream(const_cast<uint16_t*>(a.grad[r]) + e, gw);
  }
  norm_epilogue<kThreads>(a.ns, sq, nf, a.accumulate);
}

template <class F>
__global__ void __launch_bounds__(kThreads) adam_kernel(const __grid_constant__ AdamArgs a) {
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  for (int64_t vi = (int64_t)blockIdx.x * kThreads + threadIdx.x; vi < a.n_vec; vi += stride) {
    const int64_t e = vi * kVec;
    float4 p0 = ld_stream(a.master + e), p1 = ld_stream(a.master + e + 4);
    float4 m0 = ld_stream(a.m + e), m1 = ld_stream(a.m + e + 4);
    float4 v0 = ld_stream(a.v + e), v1 = ld_stream(a.v + e + 4);
    const uint4 gw = ld_stream(a.grad + e);
    float g[kVec] = {F::lo(gw.x), F::hi(gw.x), F::lo(gw.y), F::hi(gw.y),
                     F::lo(gw.z), F::hi(gw.z), F::lo(gw.w), F::hi(gw.w)};
    uint16_t p16[kVec];
    adam8<F>(g, p0, p1, m0, m1, v0, v1, a.sc, p16);
    st_stream(a.master + e, p0);
    st_stream(a.master + e + 4, p1);
    st_stream(a.m + e, m0);
    st_stream(a.m + e + 4, m1);
    st_stream(a.v + e, v0);
    st_stream(a.v + e + 4, v1);
    st_stream(a.out + e, pack8(p16));
  }
}

template <class F>
__global__ void __launch_bounds__(kThreads) adam_bcast_kernel(const __grid_constant__ AdamBcastArgs a) {
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  AdamScalars sc = a.sc_dev ? *a.sc_dev : a.sc;
  const bool skip = apply_decision(a.dec, sc);
  for (int64_t vi = (int64_t)blockIdx.x * kThreads + threadIdx.x; vi < a.n_vec; vi += stride) {
    const int64_t e = vi * kVec;
    const int64_t i = a.lo + e;  // flat index; the 8 elements share one owner (S % 8 == 0)
    float4 p0 = ld_stream(a.master + e), p1 = ld_stream(a.master + e + 4);
    if (skip) {  // a skipped step: the unchanged parameters, no state written
      const uint4 pw = round8<F>(p0, p1);
      if (a.param_shard) st_stream(a.param_shard + e, pw);
      for (int r = 0; r < a.n_out; ++r) st_stream(a.out[r] + e, pw);
      continue;
    }
    float4 m0 = ld_stream(a.m + e), m1 = ld_stream(a.m + e + 4);
    float4 v0 = ld_stream(a.v + e), v1 = ld_stream(a.v + e + 4);
    const uint4 gw = ld_stream(a.gsrc[i / a.shard] + i);
    float g[kVec] = {F::lo(gw.x), F::hi(gw.x), F::lo(gw.y), F::hi(gw.y),
                     F::lo(gw.z), F::hi(gw.z), F::lo(gw.w), F::hi(gw.w)};
    uint16_t p16[kVec];
    adam8<F>(g, p0, p1, m0, m1, v0, v1, sc, p16);  // unscale and clip via sc.flags
    st_stream(a.master + e, p0);
    st_stream(a.master + e + 4, p1);
    st_stream(a.m + e, m0);
    st_stream(a.m + e + 4, m1);
    st_stream(a.v + e, v0);
    st_stream(a.v + e + 4, v1);
    const uint4 pw = pack8(p16);
    if (a.param_shard) st_stream(a.param_shard + e, pw);
    for (int r = 0; r < a.n_out; ++r) st_stream(a.out[r] + e, pw);
  }
}

// A step's first kernel, one thread: the powers beta^(t+1) as one more
// binary64 product each, and the step's binary32 scalars from them -- each
// derived scalar rounded once from binary64, as the host computes them.
__global__ void step_begin_kernel(StepState* st, const StepHparams hp, ClipDecision* dec) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  const double q1 = __dmul_rn(st->p1, hp.beta1);
  const double q2 = __dmul_rn(st->p2, hp.beta2);
  AdamScalars s;
  s.b1 = __double2float_rn(hp.beta1);
  s.b2 = __double2float_rn(hp.beta2);
  s.omb1 = __double2float_rn(__dsub_rn(1.0, hp.beta1));
  s.omb2 = __double2float_rn(__dsub_rn(1.0, hp.beta2));
  s.bc1 = __double2float_rn(__dsub_rn(1.0, q1));
  s.bc2 = __double2float_rn(__dsub_rn(1.0, q2));
  s.decay = __double2float_rn(__dsub_rn(1.0, __dmul_rn(hp.lr, hp.weight_decay)));
  s.lr = __double2float_rn(hp.lr);
  s.eps = __double2float_rn(hp.eps);
  s.inv_scale = __double2float_rn(__ddiv_rn(1.0, hp.loss_scale));
  s.coef = 1.0f;
  s.flags = s.inv_scale != 1.0f ? kUnscale : 0;
  st->sc = s;
  st->t_next = st->t + 1;
  st->p1_next = q1;
  st->p2_next = q2;
  if (dec) {
    dec->coef = 1.0f;
    dec->skip = 0;
  }
}

// A completed (fused) step: t and the powers advance.
__global__ void step_commit_kernel(StepState* st) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  st->t = st->t_next;
  st->p1 = st->p1_next;
  st->p2 = st->p2_next;
}

// The clipped step's decision (ClipDecision), one thread, from the step's
// sums; commits the step state unless the step is skipped.
__global__ void clip_decide_kernel(const NormScratch ns, const ClipParams p, ClipDecision* out, StepState* st) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  ClipDecision d;
  d.nonfinite = *ns.step_nf;
  d.norm = __ddiv_rn(__dsqrt_rn(*ns.step_sq), p.loss_scale);
  d.skip = (p.skip_nonfinite && d.nonfinite > 0) ? 1 : 0;
  d.coef = 1.0f;
  if (!d.skip && p.max_norm > 0.0) {
    const float c = __double2float_rn(__ddiv_rn(p.max_norm, __dadd_rn(d.norm, 1e-6)));
    if (c < 1.0f) d.coef = c;  // false for a NaN norm: no clipping
  }
  *out = d;
  if (!d.skip) {
    st->t = st->t_next;
    st->p1 = st->p1_next;
    st->p2 = st->p2_next;
  }
}

__global__ void __launch_bounds__(kThreads) gather_kernel(const __grid_constant__ GatherArgs a) {
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  for (int64_t vi = (int64_t)blockIdx.x * kThreads + threadIdx.x; vi < a.n_vec; vi += stride) {
    const int64_t e = vi * kVec;
    const uint4 w = ld_stream(a.src + e);
    for (int r = 0; r < a.n_out; ++r) st_stream(a.out[r] + e, w);
  }
}

// Optimizer state from sources (fresh master weights with m = v = 0, or a
// checkpoint's master/m/v), zeros past the sources, bf16(master) to every
// parameter destination, reduced-gradient shards cleared.
template <class F>
__global__ void __launch_bounds__(kThreads) init_kernel(const __grid_constant__ InitArgs a) {
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int64_t vi = (int64_t)blockIdx.x * kThreads + threadIdx.x; vi < a.n_vec; vi += stride) {
    const int64_t e = vi * kVec;
    const bool src = vi < a.n_src_vec;
    const float4 p0 = src ? ld_stream(a.master_src + e) : z, p1 = src ? ld_stream(a.master_src + e + 4) : z;
    const float4 m0 = src && a.m_src ? ld_stream(a.m_src + e) : z, m1 = src && a.m_src ? ld_stream(a.m_src + e + 4) : z;
    const float4 v0 = src && a.v_src ? ld_stream(a.v_src + e) : z, v1 = src && a.v_src ? ld_stream(a.v_src + e + 4) : z;
    st_stream(a.master + e, p0);
    st_stream(a.master + e + 4, p1);
    st_stream(a.m + e, m0);
    st_stream(a.m + e + 4, m1);
    st_stream(a.v + e, v0);
    st_stream(a.v + e + 4, v1);
    const uint16_t h[kVec] = {F::rn(p0.x), F::rn(p0.y), F::rn(p0.z), F::rn(p0.w),
                              F::rn(p1.x), F::rn(p1.y), F::rn(p1.z), F::rn(p1.w)};
    const uint4 w = pack8(h);
    for (int r = 0; r < a.n_out; ++r) st_stream(a.out[r] + e, w);
    if (a.grad_shard) st_stream(a.grad_shard + e, make_uint4(0u, 0u, 0u, 0u));
  }
}

}  // namespace

// --------------------------------------------------------------- launchers --

template <int MODE, class F>
cudaError_t launch_fused_mode(const FusedArgs& a, int grid, cudaStream_t s) {
  const bool pdl = a.pdl != kPdlNone;
  if (a.n_ranks <= 8) return launch_kernel(fused_step_kernel<MODE, false, F>, grid, kThreads, 0, s, pdl, a);
  return launch_kernel(fused_step_kernel<MODE, true, F>, grid, kThreads, 0, s, pdl, a);
}

template <class F>
cudaError_t launch_fused_fmt(int mode, const FusedArgs& a, int grid, cudaStream_t s) {
  switch (mode) {
    case kFusedZ1: return launch_fused_mode<kFusedZ1, F>(a, grid, s);
    case kFusedZ2: return launch_fused_mode<kFusedZ2, F>(a, grid, s);
    case kFusedZ3: return launch_fused_mode<kFusedZ3, F>(a, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_fused(int mode, const FusedArgs& a, int grid, cudaStream_t s) {
  return a.fmt == kFmtF16 ? launch_fused_fmt<F16>(mode, a, grid, s) : launch_fused_fmt<Bf16>(mode, a, grid, s);
}

template <class F>
void launch_reduce_fmt(const ReduceArgs& a, int grid, cudaStream_t s) {
  if (a.n_ranks <= 8)
    reduce_kernel<false, F><<<grid, kThreads, 0, s>>>(a);
  else
    reduce_kernel<true, F><<<grid, kThreads, 0, s>>>(a);
}

cudaError_t launch_reduce(const ReduceArgs& a, int grid, cudaStream_t s) {
  if (a.fmt == kFmtF16) launch_reduce_fmt<F16>(a, grid, s);
  else launch_reduce_fmt<Bf16>(a, grid, s);
  return cudaGetLastError();
}

cudaError_t launch_adam(const AdamArgs& a, int grid, cudaStream_t s) {
  if (a.fmt == kFmtF16) adam_kernel<F16><<<grid, kThreads, 0, s>>>(a);
  else adam_kernel<Bf16><<<grid, kThreads, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_gather(const GatherArgs& a, int grid, cudaStream_t s) {
  gather_kernel<<<grid, kThreads, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_adam_bcast(const AdamBcastArgs& a, int grid, cudaStream_t s) {
  if (a.fmt == kFmtF16) adam_bcast_kernel<F16><<<grid, kThreads, 0, s>>>(a);
  else adam_bcast_kernel<Bf16><<<grid, kThreads, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_clip_decide(const NormScratch& ns, const ClipParams& p, ClipDecision* out, StepState* state,
                               cudaStream_t s) {
  clip_decide_kernel<<<1, 32, 0, s>>>(ns, p, out, state);
  return cudaGetLastError();
}

cudaError_t launch_step_begin(StepState* state, const StepHparams& hp, ClipDecision* dec, cudaStream_t s) {
  step_begin_kernel<<<1, 32, 0, s>>>(state, hp, dec);
  return cudaGetLastError();
}

cudaError_t launch_step_commit(StepState* state, cudaStream_t s) {
  step_commit_kernel<<<1, 32, 0, s>>>(state);
  return cudaGetLastError();
}

cudaError_t launch_init(const InitArgs& a, int grid, cudaStream_t s) {
  if (a.fmt == kFmtF16) init_kernel<F16><<<grid, kThreads, 0, s>>>(a);
  else init_kernel<Bf16><<<grid, kThreads, 0, s>>>(a);
  return cudaGetLastError();
}

template <class K>
int blocks_of(K kernel, cudaError_t* e) {
  int b = 0;
  if (*e == cudaSuccess) *e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kernel, kThreads, 0);
  return b;
}

cudaError_t occupancy(int mode, int n_ranks, int* fused_blocks, int* simple_blocks) {
  cudaError_t e = cudaSuccess;
  const bool multi = n_ranks > 8;
  switch (mode) {
    case kFusedZ1:
      *fused_blocks = multi ? blocks_of(fused_step_kernel<kFusedZ1, true, Bf16>, &e) : blocks_of(fused_step_kernel<kFusedZ1, false, Bf16>, &e);
      break;
    case kFusedZ2:
      *fused_blocks = multi ? blocks_of(fused_step_kernel<kFusedZ2, true, Bf16>, &e) : blocks_of(fused_step_kernel<kFusedZ2, false, Bf16>, &e);
      break;
    case kFusedZ3:
      *fused_blocks = multi ? blocks_of(fused_step_kernel<kFusedZ3, true, Bf16>, &e) : blocks_of(fused_step_kernel<kFusedZ3, false, Bf16>, &e);
      break;
    default: return cudaErrorInvalidValue;
  }
  int mn = multi ? blocks_of(reduce_kernel<true, Bf16>, &e) : blocks_of(reduce_kernel<false, Bf16>, &e);
  mn = std::min(mn, blocks_of(adam_kernel<Bf16>, &e));
  mn = std::min(mn, blocks_of(gather_kernel, &e));
  mn = std::min(mn, blocks_of(adam_bcast_kernel<Bf16>, &e));
  mn = std::min(mn, blocks_of(init_kernel<Bf16>, &e));
  *simple_blocks = mn;
  return e;
}

}  // namespace zsm
