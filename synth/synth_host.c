/*
 * Host build of the seeded synthetic-input generator (definition in
 * synth_gen.h).  Plain loops; used by the tests and the bench to produce the
 * same inputs the device build writes straight into HBM.
 */
#include "synth_gen.h"

uint64_t synth_host_base(uint64_t seed, uint32_t stream, uint32_t step, uint32_t rank) {
  return synth_base(seed, stream, step, rank);
}

void synth_host_fill_bf16(uint64_t base, int64_t idx0, int64_t n, int kind, double scale,
                          uint32_t zero_mod, uint16_t* out) {
  for (int64_t j = 0; j < n; ++j) out[j] = synth_value_bf16(base, idx0 + j, kind, scale, zero_mod);
}

void synth_host_fill_f32(uint64_t base, int64_t idx0, int64_t n, int kind, double scale,
                         uint32_t zero_mod, float* out) {
  for (int64_t j = 0; j < n; ++j) out[j] = synth_value_f32(base, idx0 + j, kind, scale, zero_mod);
}

void synth_host_gather_bf16(uint64_t base, const int64_t* idx, int64_t n, int kind, double scale,
                            uint32_t zero_mod, uint16_t* out) {
  for (int64_t j = 0; j < n; ++j) out[j] = synth_value_bf16(base, idx[j], kind, scale, zero_mod);
}

void synth_host_gather_f32(uint64_t base, const int64_t* idx, int64_t n, int kind, double scale,
                           uint32_t zero_mod, float* out) {
  for (int64_t j = 0; j < n; ++j) out[j] = synth_value_f32(base, idx[j], kind, scale, zero_mod);
}

void synth_host_fill_f16(uint64_t base, int64_t idx0, int64_t n, int kind, double scale,
                         uint32_t zero_mod, uint16_t* out) {
  for (int64_t j = 0; j < n; ++j) out[j] = synth_value_f16(base, idx0 + j, kind, scale, zero_mod);
}

void synth_host_gather_f16(uint64_t base, const int64_t* idx, int64_t n, int kind, double scale,
                           uint32_t zero_mod, uint16_t* out) {
  for (int64_t j = 0; j < n; ++j) out[j] = synth_value_f16(base, idx[j], kind, scale, zero_mod);
}
