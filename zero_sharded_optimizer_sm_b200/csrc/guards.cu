// Guard bytes of the bound arenas (ZERO_OPT_GUARD).  No sanitizer runs
// these kernels' stores through a bounds check, so the library lays out,
// around the buffers it writes, bytes that nothing it does may touch:
// the unused end of every row of an arena (a rank replica, one of master /
// m / v, a gradient or layer buffer: the pitch's alignment slack and the
// replica pad) and a tail after each arena.  Filling them with one byte
// value and checking them after a step detects a store past the end of a
// buffer without any fault; the check records how many bytes changed and
// the first of them, and writes the value back.
#include <cuda_runtime.h>

#include "guards.cuh"

namespace zsm {
namespace {

// blockIdx.y: the arena; blockIdx.x strides over its rows and, after the
// last row, its tail.  Byte accesses: the rows' ends are not 16-byte
// aligned in general, and the check is a debugging aid, not a hot path.
__global__ void __launch_bounds__(256) guard_kernel(const __grid_constant__ GuardArgs a, int check) {
  const GuardSet& g = a.set[blockIdx.y];
  const long long spans = g.rows + (g.tail > 0 ? 1 : 0);
  for (long long r = blockIdx.x; r < spans; r += gridDim.x) {
    const long long lo = r < g.rows ? r * g.pitch + g.used : g.rows * g.pitch;
    const long long hi = r < g.rows ? (r + 1) * g.pitch : g.rows * g.pitch + g.tail;
    for (long long o = lo + threadIdx.x; o < hi; o += blockDim.x) {
      unsigned char* p = g.base + o;
      if (!check) {
        *p = kGuardByte;
      } else if (*p != kGuardByte) {
        atomicAdd(a.result, 1ull);
        atomicMin(a.result + 1, ((unsigned long long)blockIdx.y << 56) | (unsigned long long)o);
        *p = kGuardByte;
      }
    }
  }
}

}  // namespace

cudaError_t launch_guards(const GuardArgs& a, bool check, cudaStream_t s) {
  long long spans = 1;
  for (int k = 0; k < kGuardSets; ++k) spans = spans > a.set[k].rows + 1 ? spans : a.set[k].rows + 1;
  const dim3 grid((unsigned)(spans < 1024 ? spans : 1024), kGuardSets);
  guard_kernel<<<grid, 256, 0, s>>>(a, check ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace zsm
