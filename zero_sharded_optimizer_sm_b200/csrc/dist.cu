// ZeRO with one logical rank per GPU (one process per GPU).
//
// The same step as the single-device path ("ZERO训练技术", sections "ZeRO-1"
// and "ZeRO-2": reduce the ranks' gradients, update the owned shard, gather
// the updated parameters to every rank), with each rank's buffers in its own
// GPU's memory.  Rank r keeps its full 16-bit gradient replica and parameter
// replica and the fp32 master / m / v of the shard it owns, [rS, (r+1)S).  The
// other ranks' gradient and parameter replicas are mapped into this process
// with CUDA IPC handles, so that one kernel per rank
//   loads the N ranks' gradient slices of its shard -- the peers' over
//   NVLink / NVSwitch -- with plain 16-byte loads, sums them in rank order
//   0..N-1 (the same bits as the oracle and the single-device kernels),
//   runs Adam in registers, writes its fp32 states once, and stores the
//   16-bit result into every rank's parameter replica (ZeRO-1: also the
//   averaged gradient into every rank's gradient replica)
// -- the reduce-scatter, the update and the all-gather of the step in one
// pass, with no collective library call.  The kernel is the register-path
// fused kernel (kernels.cu): its loads and stores are ordinary ld/st.global,
// so no bulk copy and no multicast ever reads another GPU's memory.
//
// Ordering between ranks is the caller's (host barriers): every rank's
// gradient replica is complete before any rank's step kernel starts, and no
// rank uses its parameter replica, or refills its gradient replica, before
// every rank's step kernel has completed.  No kernel here waits on another
// rank.
#include <cuda.h>  // CUdeviceptr / CUresult types for the driver entry point
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "kernels.cuh"
#include "plan.hpp"
#include "zero_sm.h"

namespace {

constexpr int64_t kAlign = 256;
constexpr int64_t kDistScratch = 80 * 1024;
static_assert(16 * zsm::kMaxGrid + 64 <= kDistScratch, "norm partials and counters fit the scratch arena");

int64_t align_up(int64_t x, int64_t m) { return ((x + m - 1) / m) * m; }

// One exported arena: the IPC handle of the allocation that holds it, the
// arena's offset in that allocation and its length.
struct IpcEntry {
  cudaIpcMemHandle_t handle;
  int64_t offset;
  int64_t bytes;
};
constexpr int kExported = 3;  // GRAD, PARAM, GATHER (an empty arena's entry is zero)
constexpr int kExportedArena[kExported] = {ZERO_DIST_ARENA_GRAD, ZERO_DIST_ARENA_PARAM, ZERO_DIST_ARENA_GATHER};
static_assert(kExported * sizeof(IpcEntry) <= ZERO_DIST_HANDLE_BYTES, "the exported arenas fit a rank's record");

thread_local std::string g_dist_init_error;

}  // namespace

struct zero_dist {
  zsm::Plan plan;
  int world = 0, rank = 0, stage = 0;
  int64_t arena_bytes[ZERO_DIST_NUM_ARENAS] = {};
  int64_t state_pitch = 0;  // bytes between the shard's master, m and v
  char* arena[ZERO_DIST_NUM_ARENAS] = {};
  bool bound = false;
  bool peers_open = false;
  uint16_t* peer_grad[zsm::kMaxRanks] = {};    // every rank's gradient replica (stage 3: layer buffer), element 0
  uint16_t* peer_param[zsm::kMaxRanks] = {};   // every rank's parameter replica, element 0 (stage 1, 2)
  uint16_t* peer_gather[zsm::kMaxRanks] = {};  // every rank's temporary gathered-layer buffer (stage 3)
  std::vector<void*> mapped;                  // IPC mappings this context opened
  int sm_count = 0, grid = 0, grid_simple = 0;
  zero_adam_hparams hp{};
  bool have_hp = false;
  bool loaded = false;
  int64_t t = 0;            // completed steps
  int layers_in_step = 0;   // stage 3: layer launches of the step in progress
  double p1 = 1.0, p2 = 1.0;  // beta1^t, beta2^t: t binary64 multiplications, one per step
  std::string err;
  ~zero_dist() {
    for (void* p : mapped) cudaIpcCloseMemHandle(p);
  }
};

namespace {

zero_status dfail(zero_dist* d, zero_status s, const char* fmt, ...) {
  if (d) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    d->err = buf;
  }
  return s;
}

zero_status dcuda(zero_dist* d, cudaError_t e, const char* what) {
  return dfail(d, ZERO_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

float* master_of(zero_dist* d) { return reinterpret_cast<float*>(d->arena[ZERO_DIST_ARENA_STATES]); }
float* m_of(zero_dist* d) { return reinterpret_cast<float*>(d->arena[ZERO_DIST_ARENA_STATES] + d->state_pitch); }
float* v_of(zero_dist* d) {
  return reinterpret_cast<float*>(d->arena[ZERO_DIST_ARENA_STATES] + 2 * d->state_pitch);
}

zsm::NormScratch scratch_of(zero_dist* d) {
  char* s = d->arena[ZERO_DIST_ARENA_SCRATCH];
  zsm::NormScratch ns;
  ns.partial_sq = reinterpret_cast<double*>(s);
  ns.partial_nf = reinterpret_cast<unsigned long long*>(s + 8 * zsm::kMaxGrid);
  char* tail = s + 16 * zsm::kMaxGrid;
  ns.done = reinterpret_cast<unsigned int*>(tail);
  ns.error = reinterpret_cast<unsigned int*>(tail + 4);
  ns.step_sq = reinterpret_cast<double*>(tail + 8);
  ns.step_nf = reinterpret_cast<unsigned long long*>(tail + 16);
  ns.wait_ns = 2000000000ull;  // the register kernel it serves has no waits
  return ns;
}

// The binary32 scalars of step t from the running binary64 powers (the same
// sequence of roundings as t multiplications of beta): every derived scalar
// formed in binary64 and rounded once.
zsm::AdamScalars scalars_of(const zero_adam_hparams& hp, double p1, double p2) {
  zsm::AdamScalars s{};
  s.b1 = (float)hp.beta1;
  s.b2 = (float)hp.beta2;
  s.omb1 = (float)(1.0 - hp.beta1);
  s.omb2 = (float)(1.0 - hp.beta2);
  s.bc1 = (float)(1.0 - p1);
  s.bc2 = (float)(1.0 - p2);
  s.decay = (float)(1.0 - hp.lr * hp.weight_decay);
  s.lr = (float)hp.lr;
  s.eps = (float)hp.eps;
  s.inv_scale = 1.0f;
  s.coef = 1.0f;
  s.flags = 0;
  return s;
}

// Base and extent of the device allocation that holds `p` (driver call
// reached through the runtime's entry-point table, so the library links only
// the runtime).
cudaError_t allocation_of(const void* p, CUdeviceptr* base, size_t* size) {
  using RangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);
  static RangeFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &f, 12000, cudaEnableDefault, &q);
    if (e != cudaSuccess) return e;
    if (q != cudaDriverEntryPointSuccess || !f) return cudaErrorNotSupported;
    fn = reinterpret_cast<RangeFn>(f);
  }
  return fn(base, size, reinterpret_cast<CUdeviceptr>(p)) == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

zero_status check_ready(zero_dist* d) {
  if (!d) return ZERO_EINVAL;
  if (!d->bound) return dfail(d, ZERO_ESTATE, "arenas are not bound (zero_dist_bind)");
  if (!d->peers_open) return dfail(d, ZERO_ESTATE, "peers are not open (zero_dist_open_peers)");
  return ZERO_OK;
}

}  // namespace

extern "C" {

zero_status zero_dist_init(const zero_layout* layout, int32_t world, int32_t rank, int32_t stage, zero_dist** out) {
  if (!out || !layout) {
    g_dist_init_error = "layout and out must not be NULL";
    return ZERO_EINVAL;
  }
  *out = nullptr;
  if (world < 1 || world > zsm::kMaxRanks || rank < 0 || rank >= world) {
    g_dist_init_error = "need 1 <= world <= ZERO_MAX_RANKS and 0 <= rank < world";
    return ZERO_EINVAL;
  }
  if (stage == ZERO_STAGE_DP) {
    g_dist_init_error = "plain data parallelism exists only in the oracle";
    return ZERO_ENOTIMPL;
  }
  if (stage != ZERO_STAGE_1 && stage != ZERO_STAGE_2 && stage != ZERO_STAGE_3) {
    g_dist_init_error = "unknown stage";
    return ZERO_EINVAL;
  }
  zero_dist* d = new zero_dist;
  std::string err;
  if (!zsm::make_plan(layout->n_tensors, layout->numel, layout->layer_id, world, 0, &d->plan, &err)) {
    delete d;
    g_dist_init_error = err;
    return ZERO_EINVAL;
  }
  d->world = world;
  d->rank = rank;
  d->stage = stage;
  const int64_t S = d->plan.shard, P = d->plan.psi_pad, L = d->plan.max_layer;
  d->state_pitch = align_up(4 * S, kAlign);
  if (stage == ZERO_STAGE_3) {  // one layer's gradient, the parameter shard, one gathered layer
    d->arena_bytes[ZERO_DIST_ARENA_GRAD] = align_up(2 * std::max<int64_t>(L, 8), kAlign);
    d->arena_bytes[ZERO_DIST_ARENA_PARAM] = align_up(2 * S, kAlign);
    d->arena_bytes[ZERO_DIST_ARENA_GATHER] = align_up(2 * std::max<int64_t>(L, 8), kAlign);
  } else {
    d->arena_bytes[ZERO_DIST_ARENA_GRAD] = align_up(2 * P, kAlign);
    d->arena_bytes[ZERO_DIST_ARENA_PARAM] = align_up(2 * P, kAlign);
  }
  d->arena_bytes[ZERO_DIST_ARENA_STATES] = 3 * d->state_pitch;
  d->arena_bytes[ZERO_DIST_ARENA_SCRATCH] = kDistScratch;
  *out = d;
  return ZERO_OK;
}

zero_status zero_dist_sizes(const zero_dist* d, int64_t plan[3], int64_t arena_bytes[ZERO_DIST_NUM_ARENAS]) {
  if (!d) return ZERO_EINVAL;
  if (plan) {
    plan[0] = d->plan.psi;
    plan[1] = d->plan.psi_pad;
    plan[2] = d->plan.shard;
  }
  if (arena_bytes)
    for (int k = 0; k < ZERO_DIST_NUM_ARENAS; ++k) arena_bytes[k] = d->arena_bytes[k];
  return ZERO_OK;
}

zero_status zero_dist_tensor_offsets(const zero_dist* d, int64_t* out, int32_t cap) {
  if (!d || !out) return ZERO_EINVAL;
  if (cap < (int32_t)d->plan.start.size()) return ZERO_EINVAL;
  std::copy(d->plan.start.begin(), d->plan.start.end(), out);
  return ZERO_OK;
}

zero_status zero_dist_bind(zero_dist* d, void* const* arenas) {
  if (!d) return ZERO_EINVAL;
  if (d->bound) return dfail(d, ZERO_ESTATE, "arenas are already bound");
  if (!arenas) return dfail(d, ZERO_EINVAL, "arenas is NULL");
  for (int k = 0; k < ZERO_DIST_NUM_ARENAS; ++k) {
    if (d->arena_bytes[k] == 0) continue;
    if (!arenas[k]) return dfail(d, ZERO_EINVAL, "arena %d is NULL", k);
    if (reinterpret_cast<uintptr_t>(arenas[k]) % kAlign) return dfail(d, ZERO_EINVAL, "arena %d is not 256-byte aligned", k);
  }
  int dev = 0, fused = 0, simple = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&d->sm_count, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess)
    e = zsm::occupancy(d->stage == ZERO_STAGE_1 ? zsm::kFusedZ1 : d->stage == ZERO_STAGE_2 ? zsm::kFusedZ2 : zsm::kFusedZ3,
                       d->world, &fused, &simple);
  if (e != cudaSuccess) return dcuda(d, e, "device query");
  d->grid = std::max(1, std::min(zsm::kMaxGrid, d->sm_count * std::max(1, fused)));
  d->grid_simple = std::max(1, std::min(zsm::kMaxGrid, d->sm_count * std::max(1, simple)));
  for (int k = 0; k < ZERO_DIST_NUM_ARENAS; ++k) d->arena[k] = d->arena_bytes[k] ? static_cast<char*>(arenas[k]) : nullptr;
  d->peer_grad[d->rank] = reinterpret_cast<uint16_t*>(d->arena[ZERO_DIST_ARENA_GRAD]);
  d->peer_param[d->rank] = reinterpret_cast<uint16_t*>(d->arena[ZERO_DIST_ARENA_PARAM]);
  d->peer_gather[d->rank] = reinterpret_cast<uint16_t*>(d->arena[ZERO_DIST_ARENA_GATHER]);
  e = cudaMemset(d->arena[ZERO_DIST_ARENA_SCRATCH], 0, kDistScratch);
  if (e != cudaSuccess) return dcuda(d, e, "clearing the scratch arena");
  d->bound = true;
  if (d->world == 1) d->peers_open = true;
  return ZERO_OK;
}

zero_status zero_dist_export(zero_dist* d, void* record) {
  if (!d || !record) return ZERO_EINVAL;
  if (!d->bound) return dfail(d, ZERO_ESTATE, "arenas are not bound (zero_dist_bind)");
  IpcEntry ent[kExported];
  std::memset(ent, 0, sizeof ent);
  CUdeviceptr bases[kExported] = {};
  for (int k = 0; k < kExported; ++k) {
    const int which = kExportedArena[k];
    if (d->arena_bytes[which] == 0) continue;  // zero entry: nothing to map
    size_t size = 0;
    cudaError_t e = allocation_of(d->arena[which], &bases[k], &size);
    if (e != cudaSuccess) return dcuda(d, e, "finding the allocation of an exported arena");
    const CUdeviceptr base = bases[k];
    int same = -1;  // an earlier arena in the same allocation: one handle, opened once
    for (int q = 0; q < k; ++q)
      if (ent[q].bytes && bases[q] == base) same = q;
    if (same >= 0) {
      ent[k].handle = ent[same].handle;
    } else {
      e = cudaIpcGetMemHandle(&ent[k].handle, reinterpret_cast<void*>(base));
      if (e != cudaSuccess)
        return dcuda(d, e, "cudaIpcGetMemHandle (arenas must come from cudaMalloc-style allocations)");
    }
    ent[k].offset = (int64_t)(reinterpret_cast<uintptr_t>(d->arena[which]) - (uintptr_t)base);
    ent[k].bytes = d->arena_bytes[which];
  }
  std::memset(record, 0, ZERO_DIST_HANDLE_BYTES);
  std::memcpy(record, ent, sizeof ent);
  return ZERO_OK;
}

zero_status zero_dist_open_peers(zero_dist* d, const void* records) {
  if (!d || !records) return ZERO_EINVAL;
  if (!d->bound) return dfail(d, ZERO_ESTATE, "arenas are not bound (zero_dist_bind)");
  if (d->peers_open && d->world > 1) return dfail(d, ZERO_ESTATE, "peers are already open");
  const unsigned char* rec = static_cast<const unsigned char*>(records);
  // one mapping per distinct allocation (two arenas of a peer may share one)
  std::vector<std::pair<cudaIpcMemHandle_t, char*>> opened;
  for (int q = 0; q < d->world; ++q) {
    if (q == d->rank) continue;
    IpcEntry ent[kExported];
    std::memcpy(ent, rec + (size_t)q * ZERO_DIST_HANDLE_BYTES, sizeof ent);
    for (int k = 0; k < kExported; ++k) {
      const int which = kExportedArena[k];
      if (ent[k].bytes != d->arena_bytes[which] || ent[k].offset < 0 || ent[k].offset % kAlign)
        return dfail(d, ZERO_EINVAL, "rank %d's record does not describe this layout's arenas", q);
      if (ent[k].bytes == 0) continue;
      char* base = nullptr;
      for (auto& o : opened)
        if (std::memcmp(&o.first, &ent[k].handle, sizeof(cudaIpcMemHandle_t)) == 0) base = o.second;
      if (!base) {
        void* p = nullptr;
        cudaError_t e = cudaIpcOpenMemHandle(&p, ent[k].handle, cudaIpcMemLazyEnablePeerAccess);
        if (e != cudaSuccess) return dcuda(d, e, "cudaIpcOpenMemHandle");
        d->mapped.push_back(p);
        base = static_cast<char*>(p);
        opened.push_back({ent[k].handle, base});
      }
      uint16_t* arena = reinterpret_cast<uint16_t*>(base + ent[k].offset);
      if (which == ZERO_DIST_ARENA_GRAD) d->peer_grad[q] = arena;
      else if (which == ZERO_DIST_ARENA_PARAM) d->peer_param[q] = arena;
      else d->peer_gather[q] = arena;
    }
  }
  d->peers_open = true;
  return ZERO_OK;
}

zero_status zero_dist_set_hparams(zero_dist* d, const zero_adam_hparams* hp) {
  if (!d || !hp) return ZERO_EINVAL;
  if (!(hp->lr >= 0.0) || !(hp->beta1 >= 0.0 && hp->beta1 < 1.0) || !(hp->beta2 >= 0.0 && hp->beta2 < 1.0) ||
      !(hp->eps >= 0.0) || !(hp->weight_decay >= 0.0))
    return dfail(d, ZERO_EINVAL, "hyper-parameters out of range");
  d->hp = *hp;
  d->have_hp = true;
  return ZERO_OK;
}

zero_status zero_dist_load_master(zero_dist* d, const float* master_full, void* stream) {
  zero_status st = check_ready(d);
  if (st != ZERO_OK) return st;
  if (!master_full || reinterpret_cast<uintptr_t>(master_full) % 16)
    return dfail(d, ZERO_EINVAL, "master_full is NULL or not 16-byte aligned");
  const int64_t S = d->plan.shard, lo = d->rank * S;
  zsm::InitArgs a;
  std::memset(&a, 0, sizeof a);
  a.fmt = zsm::kFmtBf16;
  a.master_src = master_full + lo;
  a.n_src_vec = S / zsm::kVec;
  a.master = master_of(d);
  a.m = m_of(d);
  a.v = v_of(d);
  if (d->stage == ZERO_STAGE_3) {  // the rank's own parameter shard
    a.out[0] = d->peer_param[d->rank];
    a.n_out = 1;
  } else {
    for (int q = 0; q < d->world; ++q) a.out[q] = d->peer_param[q] + lo;
    a.n_out = d->world;
  }
  a.n_vec = S / zsm::kVec;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (a.n_vec > 0) {
    cudaError_t e = zsm::launch_init(a, d->grid_simple, s);
    if (e != cudaSuccess) return dcuda(d, e, "init kernel launch");
  }
  d->t = 0;
  d->p1 = d->p2 = 1.0;
  d->layers_in_step = 0;
  d->loaded = true;
  return ZERO_OK;
}

zero_status zero_dist_step(zero_dist* d, void* stream) {
  zero_status st = check_ready(d);
  if (st != ZERO_OK) return st;
  if (!d->have_hp) return dfail(d, ZERO_ESTATE, "hyper-parameters are not set (zero_dist_set_hparams)");
  if (!d->loaded) return dfail(d, ZERO_ESTATE, "state is not initialised (zero_dist_load_master)");
  if (d->stage == ZERO_STAGE_3) return dfail(d, ZERO_ESTATE, "stage 3 steps layer by layer (zero_dist_step_layer)");
  const int N = d->world;
  const int64_t S = d->plan.shard, lo = d->rank * S;
  const double p1 = d->p1 * d->hp.beta1, p2 = d->p2 * d->hp.beta2;
  zsm::FusedArgs a;
  std::memset(&a, 0, sizeof a);
  a.fmt = zsm::kFmtBf16;
  for (int q = 0; q < N; ++q) {
    a.grad[q] = d->peer_grad[q] + lo;
    a.out[q] = d->peer_param[q] + lo;
  }
  a.master = master_of(d);
  a.m = m_of(d);
  a.v = v_of(d);
  a.n_vec = S / zsm::kVec;
  a.n_ranks = N;
  a.inv_n = (float)(1.0 / (double)N);
  a.pdl = zsm::kPdlNone;
  a.sc = scalars_of(d->hp, p1, p2);
  a.ns = scratch_of(d);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t want = (a.n_vec + zsm::kThreads - 1) / zsm::kThreads;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(want, d->grid));
  cudaError_t e = zsm::launch_fused(d->stage == ZERO_STAGE_1 ? zsm::kFusedZ1 : zsm::kFusedZ2, a, grid, s);
  if (e != cudaSuccess) return dcuda(d, e, "fused step kernel launch");
  d->t += 1;
  d->p1 = p1;
  d->p2 = p2;
  return ZERO_OK;
}

zero_status zero_dist_step_layer(zero_dist* d, int32_t layer, int32_t last, void* stream) {
  zero_status st = check_ready(d);
  if (st != ZERO_OK) return st;
  if (!d->have_hp) return dfail(d, ZERO_ESTATE, "hyper-parameters are not set (zero_dist_set_hparams)");
  if (!d->loaded) return dfail(d, ZERO_ESTATE, "state is not initialised (zero_dist_load_master)");
  if (d->stage != ZERO_STAGE_3) return dfail(d, ZERO_ESTATE, "layer-by-layer steps are stage 3's (zero_dist_step)");
  if (layer < 0 || layer >= (int32_t)d->plan.layers.size())
    return dfail(d, ZERO_EINVAL, "layer %d out of range", layer);
  const int N = d->world;
  const int64_t S = d->plan.shard, own_lo = d->rank * S, own_hi = own_lo + S;
  const int64_t l_lo = d->plan.layers[layer].lo, l_hi = d->plan.layers[layer].hi;
  const int64_t lo = std::max(l_lo, own_lo), hi = std::min(l_hi, own_hi);  // the layer's part of this shard
  const double p1 = d->p1 * d->hp.beta1, p2 = d->p2 * d->hp.beta2;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (hi > lo) {
    zsm::FusedArgs a;
    std::memset(&a, 0, sizeof a);
    a.fmt = zsm::kFmtBf16;
    for (int q = 0; q < N; ++q) {
      a.grad[q] = d->peer_grad[q] + (lo - l_lo);   // every rank's layer gradient, at this part
      a.out[q] = d->peer_gather[q] + (lo - l_lo);  // every rank's gathered layer, at this part
    }
    a.param_shard = d->peer_param[d->rank] + (lo - own_lo);
    a.master = master_of(d) + (lo - own_lo);
    a.m = m_of(d) + (lo - own_lo);
    a.v = v_of(d) + (lo - own_lo);
    a.n_vec = (hi - lo) / zsm::kVec;
    a.n_ranks = N;
    a.accumulate = d->layers_in_step > 0 ? 1 : 0;
    a.inv_n = (float)(1.0 / (double)N);
    a.pdl = zsm::kPdlNone;
    a.sc = scalars_of(d->hp, p1, p2);
    a.ns = scratch_of(d);
    const int64_t want = (a.n_vec + zsm::kThreads - 1) / zsm::kThreads;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(want, d->grid));
    cudaError_t e = zsm::launch_fused(zsm::kFusedZ3, a, grid, s);
    if (e != cudaSuccess) return dcuda(d, e, "fused step kernel launch");
    d->layers_in_step += 1;
  }
  if (last) {
    if (d->layers_in_step == 0) {  // no part of any layer on this rank: the step's sums are zero
      const zsm::NormScratch ns = scratch_of(d);
      cudaError_t e = cudaMemsetAsync(ns.step_sq, 0, 16, s);
      if (e != cudaSuccess) return dcuda(d, e, "clearing the step's sums");
    }
    d->t += 1;
    d->p1 = p1;
    d->p2 = p2;
    d->layers_in_step = 0;
  }
  return ZERO_OK;
}

zero_status zero_dist_adam_shard(zero_dist* d, const void* grad_shard, void* stream) {
  zero_status st = check_ready(d);
  if (st != ZERO_OK) return st;
  if (!d->have_hp) return dfail(d, ZERO_ESTATE, "hyper-parameters are not set (zero_dist_set_hparams)");
  if (!d->loaded) return dfail(d, ZERO_ESTATE, "state is not initialised (zero_dist_load_master)");
  if (!grad_shard || reinterpret_cast<uintptr_t>(grad_shard) % 16)
    return dfail(d, ZERO_EINVAL, "grad_shard is NULL or not 16-byte aligned");
  const int64_t S = d->plan.shard, lo = d->rank * S;
  const double p1 = d->p1 * d->hp.beta1, p2 = d->p2 * d->hp.beta2;
  zsm::AdamArgs a;
  std::memset(&a, 0, sizeof a);
  a.fmt = zsm::kFmtBf16;
  a.grad = static_cast<const uint16_t*>(grad_shard);
  a.master = master_of(d);
  a.m = m_of(d);
  a.v = v_of(d);
  a.out = d->stage == ZERO_STAGE_3 ? d->peer_param[d->rank] : d->peer_param[d->rank] + lo;
  a.n_vec = S / zsm::kVec;
  a.sc = scalars_of(d->hp, p1, p2);
  if (a.n_vec > 0) {
    const int64_t want = (a.n_vec + zsm::kThreads - 1) / zsm::kThreads;
    cudaError_t e = zsm::launch_adam(a, (int)std::max<int64_t>(1, std::min<int64_t>(want, d->grid_simple)),
                                     static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return dcuda(d, e, "adam kernel launch");
  }
  d->t += 1;
  d->p1 = p1;
  d->p2 = p2;
  return ZERO_OK;
}

zero_status zero_dist_read_partial(zero_dist* d, void* stream, double* sumsq, int64_t* nonfinite, int64_t* step) {
  if (!d || !sumsq || !nonfinite) return ZERO_EINVAL;
  if (!d->bound) return dfail(d, ZERO_ESTATE, "arenas are not bound (zero_dist_bind)");
  const zsm::NormScratch ns = scratch_of(d);
  double sq = 0.0;
  unsigned long long nf = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(&sq, ns.step_sq, sizeof sq, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(&nf, ns.step_nf, sizeof nf, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return dcuda(d, e, "reading the step's partial statistics");
  *sumsq = sq;
  *nonfinite = (int64_t)nf;
  if (step) *step = d->t;
  return ZERO_OK;
}

zero_status zero_dist_view(const zero_dist* dc, int32_t what, void** ptr, int64_t* n_elems) {
  zero_dist* d = const_cast<zero_dist*>(dc);
  if (!d || !ptr || !n_elems) return ZERO_EINVAL;
  if (!d->bound) return dfail(d, ZERO_ESTATE, "arenas are not bound (zero_dist_bind)");
  switch (what) {
    case ZERO_VIEW_MASTER: *ptr = master_of(d); *n_elems = d->plan.shard; return ZERO_OK;
    case ZERO_VIEW_EXP_AVG: *ptr = m_of(d); *n_elems = d->plan.shard; return ZERO_OK;
    case ZERO_VIEW_EXP_AVG_SQ: *ptr = v_of(d); *n_elems = d->plan.shard; return ZERO_OK;
    case ZERO_VIEW_PARAM:
      *ptr = d->arena[ZERO_DIST_ARENA_PARAM];
      *n_elems = d->stage == ZERO_STAGE_3 ? d->plan.shard : d->plan.psi_pad;
      return ZERO_OK;
    case ZERO_VIEW_GRAD_BUF:
      *ptr = d->arena[ZERO_DIST_ARENA_GRAD];
      *n_elems = d->stage == ZERO_STAGE_3 ? d->plan.max_layer : d->plan.psi_pad;
      return ZERO_OK;
    case ZERO_VIEW_GATHER:
      if (d->stage != ZERO_STAGE_3) return dfail(d, ZERO_EINVAL, "the gathered-layer buffer is stage 3's");
      *ptr = d->arena[ZERO_DIST_ARENA_GATHER];
      *n_elems = d->plan.max_layer;
      return ZERO_OK;
    default: return dfail(d, ZERO_EINVAL, "view %d does not exist for one rank per GPU", what);
  }
}

zero_status zero_dist_combine_partials(int32_t world, const double* sumsq, const int64_t* nonfinite, double* norm,
                                       int64_t* nonfinite_total) {
  if (world < 1 || !sumsq || !nonfinite || !norm || !nonfinite_total) return ZERO_EINVAL;
  double total = 0.0;
  int64_t nf = 0;
  for (int32_t q = 0; q < world; ++q) {  // rank order, binary64
    total += sumsq[q];
    nf += nonfinite[q];
  }
  *norm = std::sqrt(total);
  *nonfinite_total = nf;
  return ZERO_OK;
}

const char* zero_dist_last_error(const zero_dist* d) { return d ? d->err.c_str() : g_dist_init_error.c_str(); }

void zero_dist_destroy(zero_dist* d) { delete d; }

}  // extern "C"
