/*
 * Device build of the seeded synthetic-input generator (definition in
 * synth_gen.h).  It writes gradient replicas and initial master weights
 * directly into HBM so that large workloads need no host staging.  It is
 * input generation only and is never part of a timed optimizer step.
 */
#include <cuda_runtime.h>
#include "synth_gen.h"

namespace {

// FMT: 0 = bf16 patterns, 1 = binary16 patterns, 2 = fp32 values
template <int FMT, typename T>
__global__ void synth_fill_kernel(uint64_t base, int64_t idx0, int64_t n, int kind, double scale,
                                  uint32_t zero_mod, T* __restrict__ out) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < n; j += stride) {
    if constexpr (FMT == 0) {
      out[j] = synth_value_bf16(base, idx0 + j, kind, scale, zero_mod);
    } else if constexpr (FMT == 1) {
      out[j] = synth_value_f16(base, idx0 + j, kind, scale, zero_mod);
    } else {
      out[j] = synth_value_f32(base, idx0 + j, kind, scale, zero_mod);
    }
  }
}

int grid_for(int64_t n) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t want = (n + 255) / 256;
  int64_t cap = (int64_t)sms * 8;
  return (int)(want < cap ? (want < 1 ? 1 : want) : cap);
}

}  // namespace

extern "C" {

uint64_t synth_dev_base(uint64_t seed, uint32_t stream, uint32_t step, uint32_t rank) {
  return synth_base(seed, stream, step, rank);
}

/* Returns the cudaError_t of the launch (0 on success). */
int synth_dev_fill_bf16(uint64_t base, int64_t idx0, int64_t n, int kind, double scale,
                        uint32_t zero_mod, void* out, void* stream) {
  if (n <= 0) return 0;
  synth_fill_kernel<0, uint16_t><<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(
      base, idx0, n, kind, scale, zero_mod, (uint16_t*)out);
  return (int)cudaGetLastError();
}

int synth_dev_fill_f16(uint64_t base, int64_t idx0, int64_t n, int kind, double scale,
                       uint32_t zero_mod, void* out, void* stream) {
  if (n <= 0) return 0;
  synth_fill_kernel<1, uint16_t><<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(
      base, idx0, n, kind, scale, zero_mod, (uint16_t*)out);
  return (int)cudaGetLastError();
}

int synth_dev_fill_f32(uint64_t base, int64_t idx0, int64_t n, int kind, double scale,
                       uint32_t zero_mod, void* out, void* stream) {
  if (n <= 0) return 0;
  synth_fill_kernel<2, float><<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(
      base, idx0, n, kind, scale, zero_mod, (float*)out);
  return (int)cudaGetLastError();
}

}  // extern "C"
