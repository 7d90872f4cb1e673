// Guard bytes of the bound arenas (guards.cu, ZERO_OPT_GUARD): per arena,
// `rows` rows of `pitch` bytes from `base` whose bytes [used, pitch) are
// guards, then `tail` guard bytes after the last row (rows = tail = 0: no
// arena).  The check counts the guard bytes that differ from kGuardByte into
// result[0], the least (arena << 56 | byte offset) of them into result[1]
// (the caller sets 0 and ~0 first), and restores them.
#pragma once

#include <cuda_runtime.h>

namespace zsm {

constexpr int kGuardSets = 6;
constexpr unsigned char kGuardByte = 0xA5;
struct GuardSet {
  unsigned char* base;
  long long pitch, used, rows, tail;
};
struct GuardArgs {
  GuardSet set[kGuardSets];
  unsigned long long* result;
};
cudaError_t launch_guards(const GuardArgs& a, bool check, cudaStream_t s);

}  // namespace zsm
