// zero_fused_step_static: one fused ZeRO-2 step over a caller-described
// interval that allocates nothing ("ZERO训练技术" section "ZeRO-2":
// reduce-scatter, update of the owned shard, all-gather, fused into one pass).
//
// Why it exists: the context-based entry points need the caller to allocate
// and lend a scratch arena (zero_buffer_sizes / zero_bind).  Some callers
// cannot allocate device memory at the point where they run an optimizer
// step: a framework whose caching allocator already owns the whole device (a
// cudaMalloc of its own would fail or fragment that pool), a latency-critical
// loop where cudaMalloc/cudaFree may synchronise the device, or a one-off
// caller with no long-lived context object to keep a scratch buffer in.  This
// entry point takes only the step's inputs and outputs; the few words of
// scratch the kernel needs (per-CTA gradient-norm partials, an arrival counter
// and the step's sums) live in a file-scope __device__ array instead.
//
// The array is a fixed 32 KiB + 64 B (room for the partials of 2048 CTAs; a
// launch never takes more CTAs than that, and the kernel's grid-stride loop
// covers any interval), held on every GPU that loads the library until the
// process exits.  Every call on a device shares it and it keeps the last
// call's contents, so calls that overlap on the GPU (different streams, no
// ordering between them) race on it; calls ordered on one stream do not.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "device_math.cuh"
#include "kernels.cuh"
#include "zero_sm.h"

namespace {

using namespace zsm;
using namespace zsm::dev;

constexpr int kStaticMaxCtas = 2048;
constexpr size_t kOffSq = 0;                                   // double[kStaticMaxCtas]
constexpr size_t kOffNf = 8 * (size_t)kStaticMaxCtas;          // u64[kStaticMaxCtas]
constexpr size_t kOffStep = 16 * (size_t)kStaticMaxCtas;       // double sum, u64 count
constexpr size_t kOffDone = kOffStep + 16;                     // u32 arrivals, u32 error
constexpr size_t kStaticScratchBytes = kOffStep + 64;

}  // namespace

// The scratch.  In host code `g_static_scratch` is only a host-side stand-in
// for the symbol, not a device address: the kernel gets the address that
// cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

namespace {

constexpr int kMaxDevices = 64;

struct DeviceSetup {
  bool ready = false;
  unsigned char* scratch = nullptr;  // device address of g_static_scratch on that device
  int grid_cap = 0;                  // SMs x resident CTAs per SM
};

std::mutex g_setup_mu;
DeviceSetup g_setup[kMaxDevices];

template <bool kMulti>
__global__ void __launch_bounds__(kThreads) static_fused_step_kernel(const __grid_constant__ FusedArgs a) {
  double sq = 0.0;
  unsigned long long nf = 0;
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  for (int64_t vi = (int64_t)blockIdx.x * kThreads + threadIdx.x; vi < a.n_vec; vi += stride) {
    const int64_t e = vi * kVec;
    float4 p0 = ld_stream(a.master + e), p1 = ld_stream(a.master + e + 4);
    float4 m0 = ld_stream(a.m + e), m1 = ld_stream(a.m + e + 4);
    float4 v0 = ld_stream(a.v + e), v1 = ld_stream(a.v + e + 4);
    float acc[kVec];
    reduce_ranks<kMulti>(a.grad, a.n_ranks, e, acc);
    uint16_t g16[kVec];
    float g[kVec];
    mean_bf16(acc, a.inv_n, g16, g, sq, nf);
    uint16_t p16[kVec];
    adam8(g, p0, p1, m0, m1, v0, v1, a.sc, p16);
    st_stream(a.master + e, p0);
    st_stream(a.master + e + 4, p1);
    st_stream(a.m + e, m0);
    st_stream(a.m + e + 4, m1);
    st_stream(a.v + e, v0);
    st_stream(a.v + e + 4, v1);
    const uint4 pw = pack8(p16);
    for (int r = 0; r < a.n_ranks; ++r) st_stream(a.out[r] + e, pw);
  }
  norm_epilogue<kThreads>(a.ns, sq, nf, a.accumulate);
}

// Once per device, with that device current: the symbol's device address and
// the launch cap.  Returns the setup or nullptr (status in *st).
const DeviceSetup* setup_device(zero_status* st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *st = ZERO_ECUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_setup_mu);
  DeviceSetup& d = g_setup[dev];
  if (d.ready) return &d;
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess || ptr == nullptr) {
    *st = ZERO_ECUDA;
    return nullptr;
  }
  int sms = 0, b1 = 0, b2 = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b1, static_fused_step_kernel<false>, kThreads, 0) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b2, static_fused_step_kernel<true>, kThreads, 0) != cudaSuccess) {
    *st = ZERO_ECUDA;
    return nullptr;
  }
  d.scratch = static_cast<unsigned char*>(ptr);
  d.grid_cap = sms * std::max(1, std::min(b1, b2));
  d.ready = true;
  return &d;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" zero_status zero_fused_step_static(int32_t n_ranks, int64_t n, const void* const* rank_grads,
                                              float* master, float* exp_avg, float* exp_avg_sq,
                                              void* const* rank_params, const zero_adam_hparams* hp,
                                              int64_t t, void* stats_out, void* stream) {
  if (n_ranks < 1 || n_ranks > ZERO_MAX_RANKS || n < 0 || n % kVec != 0 || t < 1 || !hp || !rank_grads ||
      !rank_params)
    return ZERO_EINVAL;
  if (!aligned16(master) || !aligned16(exp_avg) || !aligned16(exp_avg_sq)) return ZERO_EINVAL;
  if (stats_out && (reinterpret_cast<uintptr_t>(stats_out) & 7u)) return ZERO_EINVAL;
  if (!(hp->lr >= 0.0) || !(hp->beta1 >= 0.0 && hp->beta1 < 1.0) || !(hp->beta2 >= 0.0 && hp->beta2 < 1.0) ||
      !(hp->eps >= 0.0) || !(hp->weight_decay >= 0.0))
    return ZERO_EINVAL;
  FusedArgs a;
  std::memset(&a, 0, sizeof a);
  for (int r = 0; r < n_ranks; ++r) {
    if (!aligned16(rank_grads[r]) || !aligned16(rank_params[r])) return ZERO_EINVAL;
    a.grad[r] = static_cast<const uint16_t*>(rank_grads[r]);
    a.out[r] = static_cast<uint16_t*>(rank_params[r]);
  }
  zero_status st = ZERO_OK;
  const DeviceSetup* d = setup_device(&st);
  if (!d) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t n_vec = n / kVec;
  const int64_t want = std::max<int64_t>(1, (n_vec + kThreads - 1) / kThreads);
  // at most the CTAs the scratch has partials for (the loop is grid-stride)
  const int grid = (int)std::min<int64_t>(std::min<int64_t>(want, d->grid_cap), kStaticMaxCtas);
  // what must start at zero: the arrival counter and the error word
  if (cudaMemsetAsync(d->scratch + kOffDone, 0, 8, s) != cudaSuccess) return ZERO_ECUDA;
  if (n_vec > 0) {
    // binary32 scalars of step t, each rounded once from binary64; beta^t
    // is t successive binary64 products (no state survives between calls
    // to keep a running product in), left early once both have reached 0,
    // where every further product stays exactly 0
    double p1 = 1.0, p2 = 1.0;
    for (int64_t k = 0; k < t && (p1 != 0.0 || p2 != 0.0); ++k) {
      p1 *= hp->beta1;
      p2 *= hp->beta2;
    }
    a.sc.b1 = (float)hp->beta1;
    a.sc.b2 = (float)hp->beta2;
    a.sc.omb1 = (float)(1.0 - hp->beta1);
    a.sc.omb2 = (float)(1.0 - hp->beta2);
    a.sc.bc1 = (float)(1.0 - p1);
    a.sc.bc2 = (float)(1.0 - p2);
    a.sc.decay = (float)(1.0 - hp->lr * hp->weight_decay);
    a.sc.lr = (float)hp->lr;
    a.sc.eps = (float)hp->eps;
    a.master = master;
    a.m = exp_avg;
    a.v = exp_avg_sq;
    a.n_vec = n_vec;
    a.n_ranks = n_ranks;
    a.accumulate = 0;
    a.inv_n = (float)(1.0 / (double)n_ranks);
    a.ns.partial_sq = reinterpret_cast<double*>(d->scratch + kOffSq);
    a.ns.partial_nf = reinterpret_cast<unsigned long long*>(d->scratch + kOffNf);
    a.ns.step_sq = reinterpret_cast<double*>(d->scratch + kOffStep);
    a.ns.step_nf = reinterpret_cast<unsigned long long*>(d->scratch + kOffStep + 8);
    a.ns.done = reinterpret_cast<unsigned int*>(d->scratch + kOffDone);
    a.ns.error = reinterpret_cast<unsigned int*>(d->scratch + kOffDone + 4);
    if (n_ranks <= 8)
      static_fused_step_kernel<false><<<grid, kThreads, 0, s>>>(a);
    else
      static_fused_step_kernel<true><<<grid, kThreads, 0, s>>>(a);
    if (cudaGetLastError() != cudaSuccess) return ZERO_ECUDA;
  } else if (cudaMemsetAsync(d->scratch + kOffStep, 0, 16, s) != cudaSuccess) {
    return ZERO_ECUDA;
  }
  if (stats_out && cudaMemcpyAsync(stats_out, d->scratch + kOffStep, 16, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return ZERO_ECUDA;
  return ZERO_OK;
}
