// C ABI of the ZeRO optimizer-step library: validation, arena layout and the
// executor that sequences the kernels of each stage.  Declarations and the
// contract of every entry point are in include/zero_sm.h.
//
// The stage flows follow "ZERO训练技术" sections "ZeRO-1" (all-reduce, update
// of the owned shard, all-gather), "ZeRO-2" (bucketed reduce-scatter as the
// backward produces gradients, update, all-gather) and "ZeRO-3" (per-layer
// gather into a temporary full-layer buffer that the next layer reuses); the
// fixed-size gradient buffer and the one caller-owned pool are sections 3.3
// "CB" and 3.4 "MD" of "ZeRO：从优化器状态到残差状态的显存优化".
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "zero_sm.h"
#include "guards.cuh"
#include "kernels.cuh"
#include "two_pass_bulk.cuh"
#include "plan.hpp"

static_assert(ZERO_MAX_RANKS == zsm::kMaxRanks, "rank limit mismatch");

namespace {

thread_local std::string g_init_error;

constexpr int64_t kArenaAlign = 256;
constexpr int64_t kScratchBytes = 80 * 1024;
static_assert(16 * zsm::kMaxGrid + 128 + sizeof(zsm::StepState) <= kScratchBytes,
              "the scratch arena holds the norm partials, the step sums, the clip decision and the step state");
// Guard bytes (ZERO_OPT_GUARD): the tail after each arena; the guard check's
// two result words sit in the scratch arena past the step state.
constexpr int64_t kGuardBytes = 256;
constexpr int64_t kGuardResultOffset = 72 * 1024;
static_assert(16 * zsm::kMaxGrid + 128 + sizeof(zsm::StepState) <= kGuardResultOffset &&
                  kGuardResultOffset + 16 <= kScratchBytes,
              "the guard check's result words follow the step state in the scratch arena");
// The layered stage-3 launch's arrival counter, past the guard result.
constexpr int64_t kSegCounterOffset = kGuardResultOffset + 64;
static_assert(kSegCounterOffset + 4 <= kScratchBytes, "the layered launch's counter fits the scratch arena");

int64_t align_up(int64_t x, int64_t m) { return ((x + m - 1) / m) * m; }

// NVTX ranges on the library's own domain "zero_sm" (ZERO_OPT_NVTX): host
// ranges around the enqueueing of a step and of each of its launches, which
// a profiler projects onto the kernels they enqueue.  Without a tool
// attached each call returns at once.
nvtxDomainHandle_t nvtx_domain() {
  static const nvtxDomainHandle_t d = nvtxDomainCreateA("zero_sm");
  return d;
}

class NvtxRange {
 public:
  NvtxRange(bool on, const char* fmt, ...) : on_(on) {
    if (!on_) return;
    char msg[128];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(msg, sizeof msg, fmt, ap);
    va_end(ap);
    nvtxEventAttributes_t a;
    std::memset(&a, 0, sizeof a);
    a.version = NVTX_VERSION;
    a.size = NVTX_EVENT_ATTRIB_STRUCT_SIZE;
    a.messageType = NVTX_MESSAGE_TYPE_ASCII;
    a.message.ascii = msg;
    nvtxDomainRangePushEx(nvtx_domain(), &a);
  }
  ~NvtxRange() {
    if (on_) nvtxDomainRangePop(nvtx_domain());
  }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;

 private:
  bool on_;
};

}  // namespace

struct zero_ctx {
  zsm::Plan plan;
  int32_t stage = 0;
  // options
  bool keep_grad_shards = true;
  bool grad_buffers = true;
  int64_t replica_pad = 0;
  int blocks_per_sm_opt = 0;
  int kernel_opt = ZERO_KERNEL_AUTO;
  int tma_groups_opt = 0;  // 0 = the library's choice
  int tma_stages_opt = 0;  // 0 = the library's choice
  int tma_ctas_opt = 0;    // CTAs per SM of the staged kernel, 0 = the library's choice
  int tma_tile_opt = 0;    // bulk-store kernel: elements per tile, 0 = the library's choice
  int tma_warps_opt = 0;   // bulk-store kernel: consumer warps, 0 = the library's choice
  unsigned long long wait_ns = 2000000000ull;  // limit of the staged kernels' ring waits (ZERO_OPT_WAIT_LIMIT_NS)
  int store_hint = -1;     // bulk-store kernel: L2 evict-first hint on its stores (ZERO_OPT_STORE_HINT, -1 = policy)
  int tma_grid_key = -1;   // configuration the cached grid cap belongs to
  int tma_grid_cap = 0;
  // arena layout (bytes)
  int64_t arena_bytes[ZERO_NUM_ARENAS] = {};
  int64_t state_pitch = 0;   // bytes between master, m and v
  int64_t param_pitch = 0;   // bytes between parameter replicas (stage 1, 2)
  int64_t grad_pitch = 0;    // bytes between gradient buffers
  int64_t gather_pitch = 0;  // bytes between temporary layer buffers (stage 3)
  // binding
  bool bound = false;
  char* arena[ZERO_NUM_ARENAS] = {};
  int sm_count = 0;
  int grid_fused = 0;
  int grid_simple = 0;
  // run state
  bool have_hp = false;
  zero_adam_hparams hp{};
  bool loaded = false;
  int64_t t = 0;      // the step counter as the host last learnt it (the device holds it)
  int64_t calls = 0;  // step calls since the counter was last set: the callbacks' step number
  int fmt = zsm::kFmtBf16;     // storage format of gradients and parameters
  double loss_scale = 1.0;     // the gradients the ranks hold are loss_scale x the true ones
  double clip_norm = 0.0;      // > 0: global-norm clipping
  bool skip_nonfinite = false;
  bool norm_fresh = true;  // next norm-producing launch starts a new step's sum
  // callback pipeline (ZERO_OPT_PIPELINE): side stream and ordering events
  int pipeline = 0;  // ZERO_OPT_PIPELINE: 0, 1 or 2
  // Programmatic dependent launch between the step's fused launches (the
  // staged launches then reserve enough shared memory that a grid never puts
  // two CTAs on one SM); measured 0.5-2 % faster per step on B200.
  bool pdl = true;
  bool nvtx = false;  // ZERO_OPT_NVTX: ranges per step and per launch
  bool layered = true;  // ZERO_OPT_LAYERED: a callback-free stage-3 step as one launch
  int guard = 0;  // ZERO_OPT_GUARD: 0, 1 (laid out, armed at load, checked on request) or 2 (checked after each step)
  int slots = 1;  // gradient / gather slot sets: 2 with the pipeline at stage 2/3
  cudaStream_t side = nullptr;   // the callbacks' stream
  cudaStream_t kside = nullptr;  // the kernels' stream at the greatest priority (ZERO_OPT_PIPELINE = 2)
  bool own_side = false, own_kside = false;  // created here (destroyed with the context)
  bool pipeline_used = false;

  cudaEvent_t ev_start = nullptr, ev_join = nullptr, ev_kjoin = nullptr;
  cudaEvent_t ev_grads[2] = {}, ev_kernel[2] = {}, ev_consumed[2] = {};
  // fused-kernel timing
  bool timing = false;
  std::vector<cudaEvent_t> events;  // pairs (start, end), reused
  size_t timed = 0;                 // pairs recorded since the last read
  double timed_bytes = 0.0;
  int64_t launched = 0;             // kernels this context has enqueued (zero_launch_count)
  std::string err;
  ~zero_ctx() {
    for (cudaEvent_t e : events) cudaEventDestroy(e);
    for (cudaEvent_t e : {ev_start, ev_join, ev_kjoin, ev_grads[0], ev_grads[1], ev_kernel[0], ev_kernel[1],
                          ev_consumed[0], ev_consumed[1]})
      if (e) cudaEventDestroy(e);
    if (side && own_side) cudaStreamDestroy(side);
    if (kside && own_kside) cudaStreamDestroy(kside);
  }
};

namespace {

zero_status fail(zero_ctx* c, zero_status s, const char* fmt, ...) {
  if (c) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    c->err = buf;
  }
  return s;
}

zero_status cuda_fail(zero_ctx* c, cudaError_t e, const char* what) {
  return fail(c, ZERO_ECUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

void compute_layout(zero_ctx* c) {
  const zsm::Plan& p = c->plan;
  const int64_t N = p.n_ranks;
  const int64_t row2 = align_up(p.psi_pad * 2, kArenaAlign);
  c->state_pitch = align_up(p.psi_pad * 4, kArenaAlign) + c->replica_pad;
  c->param_pitch = row2 + c->replica_pad;
  std::fill(c->arena_bytes, c->arena_bytes + ZERO_NUM_ARENAS, 0);
  c->arena_bytes[ZERO_ARENA_STATES] = 3 * c->state_pitch;
  c->arena_bytes[ZERO_ARENA_SCRATCH] = kScratchBytes;
  // Stage 1's intervals are disjoint ranges of the full replicas, so the
  // pipeline needs a second slot set only for the stage 2 bucket and the
  // stage 3 layer buffers.
  c->slots = (c->pipeline && c->stage != ZERO_STAGE_1) ? 2 : 1;
  switch (c->stage) {
    case ZERO_STAGE_1:
      c->grad_pitch = c->param_pitch;
      c->arena_bytes[ZERO_ARENA_PARAMS] = N * c->param_pitch;
      c->arena_bytes[ZERO_ARENA_GRADS] = N * c->grad_pitch;
      break;
    case ZERO_STAGE_2:
      c->grad_pitch = align_up(p.max_bucket * 2, kArenaAlign) + c->replica_pad;
      c->arena_bytes[ZERO_ARENA_PARAMS] = N * c->param_pitch;
      c->arena_bytes[ZERO_ARENA_GRADS] = c->slots * N * c->grad_pitch;
      c->arena_bytes[ZERO_ARENA_GRAD_SHARDS] = c->keep_grad_shards ? row2 : 0;
      break;
    case ZERO_STAGE_3:
      c->param_pitch = row2;
      c->grad_pitch = align_up(p.max_layer * 2, kArenaAlign) + c->replica_pad;
      c->gather_pitch = c->grad_pitch;
      c->arena_bytes[ZERO_ARENA_PARAMS] = row2;
      c->arena_bytes[ZERO_ARENA_GRADS] = c->slots * N * c->grad_pitch;
      c->arena_bytes[ZERO_ARENA_GRAD_SHARDS] = c->keep_grad_shards ? row2 : 0;
      c->arena_bytes[ZERO_ARENA_GATHER] = c->slots * N * c->gather_pitch;
      break;
  }
  if (!c->grad_buffers) c->arena_bytes[ZERO_ARENA_GRADS] = 0;
  if (c->guard)
    for (int k = 0; k < ZERO_NUM_ARENAS; ++k)
      if (c->arena_bytes[k]) c->arena_bytes[k] += kGuardBytes;
}

float* master_ptr(zero_ctx* c) { return reinterpret_cast<float*>(c->arena[ZERO_ARENA_STATES]); }
float* m_ptr(zero_ctx* c) { return reinterpret_cast<float*>(c->arena[ZERO_ARENA_STATES] + c->state_pitch); }
float* v_ptr(zero_ctx* c) { return reinterpret_cast<float*>(c->arena[ZERO_ARENA_STATES] + 2 * c->state_pitch); }
uint16_t* param_ptr(zero_ctx* c, int r) {  // replica r (stage 1, 2) or the shards (stage 3)
  return reinterpret_cast<uint16_t*>(c->arena[ZERO_ARENA_PARAMS] + (c->stage == ZERO_STAGE_3 ? 0 : r * c->param_pitch));
}
// Rank r's gradient buffer in slot set `slot` (0, or 1 with the pipeline).
uint16_t* grad_buf_ptr(zero_ctx* c, int r, int slot = 0) {
  return reinterpret_cast<uint16_t*>(c->arena[ZERO_ARENA_GRADS] +
                                     ((int64_t)slot * c->plan.n_ranks + r) * c->grad_pitch);
}
uint16_t* grad_shard_ptr(zero_ctx* c) { return reinterpret_cast<uint16_t*>(c->arena[ZERO_ARENA_GRAD_SHARDS]); }
uint16_t* gather_ptr(zero_ctx* c, int r, int slot = 0) {
  return reinterpret_cast<uint16_t*>(c->arena[ZERO_ARENA_GATHER] +
                                     ((int64_t)slot * c->plan.n_ranks + r) * c->gather_pitch);
}

zsm::NormScratch norm_scratch(zero_ctx* c) {
  char* s = c->arena[ZERO_ARENA_SCRATCH];
  zsm::NormScratch ns;
  ns.partial_sq = reinterpret_cast<double*>(s);
  ns.partial_nf = reinterpret_cast<unsigned long long*>(s + 8 * zsm::kMaxGrid);
  ns.step_sq = reinterpret_cast<double*>(s + 16 * zsm::kMaxGrid);
  ns.step_nf = reinterpret_cast<unsigned long long*>(s + 16 * zsm::kMaxGrid + 8);
  ns.done = reinterpret_cast<unsigned int*>(s + 16 * zsm::kMaxGrid + 16);
  ns.error = reinterpret_cast<unsigned int*>(s + 16 * zsm::kMaxGrid + 20);
  ns.wait_ns = c->wait_ns;
  return ns;
}

// The scratch arena past the norm partials: the step's sums, then (at +64)
// the clipped step's decision and (at +128) the device step state; one copy
// of this block gives the host every statistic of the last step.
constexpr int64_t kDecisionOffset = 64, kStateOffset = 128;
struct StatsBlock {
  double sq;
  unsigned long long nf;
  unsigned int done;
  unsigned int error;
  char pad0[kDecisionOffset - 24];
  zsm::ClipDecision dec;
  char pad1[kStateOffset - kDecisionOffset - sizeof(zsm::ClipDecision)];
  zsm::StepState state;
};
static_assert(offsetof(StatsBlock, dec) == kDecisionOffset && offsetof(StatsBlock, state) == kStateOffset,
              "stats block layout");

char* stats_block(zero_ctx* c) { return c->arena[ZERO_ARENA_SCRATCH] + 16 * zsm::kMaxGrid; }
zsm::ClipDecision* decision_ptr(zero_ctx* c) {
  return reinterpret_cast<zsm::ClipDecision*>(stats_block(c) + kDecisionOffset);
}
zsm::StepState* state_ptr(zero_ctx* c) { return reinterpret_cast<zsm::StepState*>(stats_block(c) + kStateOffset); }

// The guard bytes of each bound arena: the end of every row past the bytes
// the library's buffers use, and the tail.  Returns false when the rows and
// the tail do not add up to the arena's size (a layout this code does not
// describe).
bool guard_args(zero_ctx* c, zsm::GuardArgs* g) {
  std::memset(g, 0, sizeof *g);
  const zsm::Plan& p = c->plan;
  const int64_t N = p.n_ranks;
  const int64_t row2 = align_up(p.psi_pad * 2, kArenaAlign);
  const int64_t grad_used = c->stage == ZERO_STAGE_1   ? p.psi_pad * 2
                            : c->stage == ZERO_STAGE_2 ? p.max_bucket * 2
                                                       : p.max_layer * 2;
  const int64_t grad_rows = c->stage == ZERO_STAGE_1 ? N : c->slots * N;
  const int64_t rows[ZERO_NUM_ARENAS] = {3, c->stage == ZERO_STAGE_3 ? 1 : N, grad_rows, 1, c->slots * N, 1};
  const int64_t pitch[ZERO_NUM_ARENAS] = {c->state_pitch, c->param_pitch, c->grad_pitch, row2, c->gather_pitch,
                                          kScratchBytes};
  const int64_t used[ZERO_NUM_ARENAS] = {p.psi_pad * 4, p.psi_pad * 2, grad_used, p.psi_pad * 2, p.max_layer * 2,
                                         kScratchBytes};
  static_assert(ZERO_NUM_ARENAS == zsm::kGuardSets, "one guard set per arena");
  for (int k = 0; k < ZERO_NUM_ARENAS; ++k) {
    if (!c->arena[k]) continue;
    if (rows[k] * pitch[k] + kGuardBytes != c->arena_bytes[k] || used[k] > pitch[k]) return false;
    g->set[k] = zsm::GuardSet{reinterpret_cast<unsigned char*>(c->arena[k]), pitch[k], used[k], rows[k], kGuardBytes};
  }
  g->result = reinterpret_cast<unsigned long long*>(c->arena[ZERO_ARENA_SCRATCH] + kGuardResultOffset);
  return true;
}

zsm::StepHparams step_hparams(const zero_ctx* c) {
  zsm::StepHparams h;
  h.lr = c->hp.lr;
  h.beta1 = c->hp.beta1;
  h.beta2 = c->hp.beta2;
  h.eps = c->hp.eps;
  h.weight_decay = c->hp.weight_decay;
  h.loss_scale = c->loss_scale;
  return h;
}

// The device step state for t completed steps: beta^t by t successive
// binary64 products, as the step kernels continue them.
zsm::StepState host_state(const zero_adam_hparams& hp, int64_t t) {
  zsm::StepState st;
  std::memset(&st, 0, sizeof st);
  double p1 = 1.0, p2 = 1.0;
  for (int64_t k = 0; k < t; ++k) {
    p1 *= hp.beta1;
    p2 *= hp.beta2;
  }
  st.t = t;
  st.p1 = p1;
  st.p2 = p2;
  st.t_next = t;
  st.p1_next = p1;
  st.p2_next = p2;
  return st;
}

// Reads the device step counter (waits for the device).
zero_status read_device_t(zero_ctx* c, int64_t* t) {
  long long v = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(&v, &state_ptr(c)->t, sizeof v, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(c, e, "reading the step counter");
  *t = (int64_t)v;
  c->t = *t;
  return ZERO_OK;
}

// Writes the device step state for t completed steps (waits for the device).
zero_status write_device_t(zero_ctx* c, int64_t t) {
  const zsm::StepState st = host_state(c->hp, t);
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(state_ptr(c), &st, sizeof st, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(c, e, "writing the step counter");
  c->t = t;
  c->calls = t;
  return ZERO_OK;
}

zsm::AdamScalars adam_scalars(const zero_adam_hparams& hp, int64_t t);

// The step's scalars plus the gradient factors: fp32(1/loss_scale) when that
// is not 1, and a clipping coefficient when below 1.
zsm::AdamScalars step_scalars(const zero_ctx* c, int64_t t, float coef) {
  zsm::AdamScalars s = adam_scalars(c->hp, t);
  s.inv_scale = (float)(1.0 / c->loss_scale);
  if (s.inv_scale != 1.0f) s.flags |= zsm::kUnscale;
  s.coef = coef;
  if (coef < 1.0f) s.flags |= zsm::kClip;
  return s;
}

zsm::AdamScalars adam_scalars(const zero_adam_hparams& hp, int64_t t) {
  double p1 = 1.0, p2 = 1.0;
  for (int64_t k = 0; k < t; ++k) {
    p1 *= hp.beta1;
    p2 *= hp.beta2;
  }
  zsm::AdamScalars s;
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

constexpr size_t kMaxTimed = 4096;
constexpr int64_t kTmaTile = 2048;  // elements per shared-memory tile of the staged kernel

// Staged-kernel configuration chosen for N and the stage (consumer groups,
// ring depth), measured on B200 with flat 256M-element buffers and the
// 1.2B-parameter transformer list.  Stage 2: few bytes per element (N <= 4)
// leave the consumers compute-bound, so two groups win; at N = 5..8 one group
// of eight warps with a two-deep ring keeps the fewest copies in flight and
// moves the most bytes; at N = 9..16 (only two stages fit) one group of
// sixteen warps wins.  Stage 1 stores 2N more bytes per element (the
// all-reduce write-back), and there the sixteen-warp group wins from N = 5
// (by 3.5 % at N = 8); stages 1 and 3 take two groups with a two-deep ring at
// N = 2.  Above N = 16 the rank-chunked staged kernel wins over the register
// kernel.
struct TmaChoice {
  int groups, stages;
};

TmaChoice tma_policy(int n_ranks, int stage) {
  if (stage == ZERO_STAGE_1) {
    if (n_ranks <= 1) return {2, 4};
    if (n_ranks <= 4) return {2, 2};
    return {zsm::kWideGroup, 2};
  }
  if (n_ranks <= 1) return {2, 4};
  if (n_ranks <= 2) return stage == ZERO_STAGE_3 ? TmaChoice{2, 2} : TmaChoice{2, 4};
  if (n_ranks <= 4) return {2, 2};
  if (n_ranks <= 8) return {1, 2};
  return {zsm::kWideGroup, 2};
}

// Consumer groups of the staged kernel for this context.
int tma_groups(const zero_ctx* c) {
  if (c->tma_groups_opt) return c->tma_groups_opt;
  return tma_policy(c->plan.n_ranks, c->stage).groups;
}

int tma_stages(const zero_ctx* c) {
  if (c->tma_stages_opt) return c->tma_stages_opt;
  return tma_policy(c->plan.n_ranks, c->stage).stages;
}

// CTAs of a staged-kernel launch: SMs x the CTAs per SM asked for (1 by
// default), capped by what fits; cached per configuration.
int tma_grid_cap(zero_ctx* c) {
  const int want = c->tma_ctas_opt > 0 ? c->tma_ctas_opt : 1;
  const int key = (tma_groups(c) * 16 + tma_stages(c)) * 64 + want;
  if (key != c->tma_grid_key) {
    const int fit = zsm::tma_ctas_per_sm(c->plan.n_ranks, tma_groups(c), tma_stages(c));
    c->tma_grid_cap = c->sm_count * std::max(1, std::min(want, fit));
    c->tma_grid_key = key;
  }
  return c->tma_grid_cap;
}

// Whether the fused step runs a shared-memory staged kernel: the all-ranks
// stage kernel for N <= 16, the rank-chunked one above.
bool use_bulk(const zero_ctx* c);

bool use_chunked(const zero_ctx* c) {
  if (c->plan.n_ranks <= zsm::kTmaMaxRanks || use_bulk(c)) return false;
  return c->kernel_opt != ZERO_KERNEL_REGISTER;  // AUTO and TMA
}

bool use_tma(const zero_ctx* c) {
  if (use_chunked(c)) return true;
  if (use_bulk(c)) return false;
  if (zsm::tma_stages_for(c->plan.n_ranks, tma_groups(c), tma_stages(c)) == 0) return false;
  if (c->kernel_opt == ZERO_KERNEL_TMA) return true;
  if (c->kernel_opt == ZERO_KERNEL_REGISTER) return false;
  return true;  // AUTO: the staged kernel wherever it applies (N <= 16)
}

int chunked_stages(const zero_ctx* c) { return c->tma_stages_opt ? c->tma_stages_opt : 3; }  // measured best at N = 32, 64

// The bulk-store staged kernel's configuration (tile, consumer warps, ring
// depth -- above 16 ranks the chunk ring's) chosen for N and the stage,
// measured on B200: flat 256M-element buffers at N = 1, 2, 4, 8, 16, flat
// 64M at N = 17, 32, 64, and the 1.2B-parameter transformer list at N = 8,
// every stage, two or three interleaved repetitions per cell, with the L2
// evict-first hint on the stores.  Few ranks leave each tile short and the
// arithmetic dominant: 2048-element tiles with sixteen warps.  From N = 5 the
// copies dominate: eight warps, 1024-element tiles, with the ring as deep as
// measured best (three stages at ZeRO-1, which also stages the averaged
// gradient, four otherwise; at N = 9..16, where a stage is twice as large,
// three).  Above 16 ranks the rank-chunked form; at N = 17..31 (a chunk ring
// of three 2048-element stages) the last chunk is short.  tile = 0: the TMA
// kernel measured faster there (N = 2 at ZeRO-3, by 4 %).  The stores' L2
// evict-first hint gained up to 4 % at stages 2 and 3 everywhere and is on
// there; at stage 1 it lost about 1 % at N = 5..8 and from N = 32 on (where
// it is off) and gained about as much at N = 3..4 and 9..31.
struct BulkChoice {
  int tile, warps, stages, hint;
};

BulkChoice bulk_policy(int n_ranks, int stage) {
  const bool z1 = stage == ZERO_STAGE_1;
  if (n_ranks <= 1) return {2048, 16, 3, 1};
  if (n_ranks == 2) return stage == ZERO_STAGE_3 ? BulkChoice{0, 0, 0, 1} : BulkChoice{2048, 16, 3, 1};
  if (n_ranks <= 4) return z1 ? BulkChoice{2048, 16, 2, 1} : BulkChoice{2048, 16, 3, 1};
  if (n_ranks <= 8) return z1 ? BulkChoice{1024, 8, 3, 0} : BulkChoice{1024, 8, 4, 1};
  if (n_ranks <= 16) return z1 ? BulkChoice{2048, 8, 2, 1} : BulkChoice{1024, 8, 3, 1};
  if (n_ranks < 32) return z1 ? BulkChoice{1024, 8, 3, 1} : BulkChoice{2048, 8, 3, 1};
  return z1 ? BulkChoice{1024, 8, 3, 0} : BulkChoice{1024, 8, 4, 1};
}

// The bulk-store staged kernel (fused_bulk.cu): its tile, consumer warps and
// ring depth for this context (the options where set, else the policy).
int bulk_tile(const zero_ctx* c) {
  if (c->tma_tile_opt) return c->tma_tile_opt;
  const int t = bulk_policy(c->plan.n_ranks, c->stage).tile;
  return t ? t : 2048;  // BULK asked for where the policy prefers TMA
}
int bulk_warps(const zero_ctx* c) {
  if (c->tma_warps_opt) return c->tma_warps_opt;
  const int w = bulk_policy(c->plan.n_ranks, c->stage).warps;
  return w ? w : 16;
}
bool bulk_need_g(const zero_ctx* c) {
  return c->stage == ZERO_STAGE_1 || c->arena[ZERO_ARENA_GRAD_SHARDS] != nullptr;
}
int bulk_ring(const zero_ctx* c) {
  if (c->tma_stages_opt) return c->tma_stages_opt;
  const int st = bulk_policy(c->plan.n_ranks, c->stage).stages;
  return st ? st : 3;
}
int bulk_stages(const zero_ctx* c) {
  return zsm::bulk_stages_for(c->plan.n_ranks, bulk_tile(c), bulk_need_g(c), bulk_ring(c));
}
bool bulk_fits(const zero_ctx* c) {
  return zsm::bulk_config_valid(c->plan.n_ranks, bulk_tile(c), bulk_warps(c)) && bulk_stages(c) > 0;
}
// Asked for, or AUTO where the policy picks it (any N; the rank-chunked form
// above 16); a (tile, warps) pair that is not built fails at launch.
bool use_bulk(const zero_ctx* c) {
  if (c->kernel_opt == ZERO_KERNEL_BULK) return true;
  return c->kernel_opt == ZERO_KERNEL_AUTO && bulk_policy(c->plan.n_ranks, c->stage).tile != 0;
}

// Bytes one element moves through HBM in the fused step (the byte model).
int64_t fused_bytes_per_elem(const zero_ctx* c) {
  const int64_t N = c->plan.n_ranks;
  const int64_t keep = c->arena[ZERO_ARENA_GRAD_SHARDS] ? 2 : 0;
  if (c->stage == ZERO_STAGE_1) return 6 * N + 24;
  if (c->stage == ZERO_STAGE_2) return 4 * N + 24 + keep;
  return 4 * N + 26 + keep;
}

// Counts a kernel the context enqueued (zero_launch_count) and passes the
// launch status through.
cudaError_t counted(zero_ctx* c, cudaError_t e) {
  if (e == cudaSuccess) ++c->launched;
  return e;
}

// Event pair for the next timed launch, or nullptr when the record is full.
cudaEvent_t* timing_pair(zero_ctx* c) {
  if (c->timed >= kMaxTimed) return nullptr;
  while (c->events.size() < 2 * (c->timed + 1)) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    c->events.push_back(e);
  }
  return &c->events[2 * c->timed];
}

int grid_for(int64_t n_vec, int cap) {
  const int64_t want = (n_vec + zsm::kThreads - 1) / zsm::kThreads;
  return (int)std::max<int64_t>(1, std::min<int64_t>(want, cap));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

zero_status check_interval(zero_ctx* c, int64_t lo, int64_t hi) {
  if (lo < 0 || hi < lo || hi > c->plan.psi_pad || lo % zsm::kGranule || hi % zsm::kGranule)
    return fail(c, ZERO_EINVAL, "interval [%lld, %lld) must satisfy 0 <= lo <= hi <= psi_pad=%lld, both multiples of 8",
                (long long)lo, (long long)hi, (long long)c->plan.psi_pad);
  return ZERO_OK;
}

zero_status check_ready(zero_ctx* c, bool need_hp) {
  if (!c) return ZERO_EINVAL;
  if (!c->bound) return fail(c, ZERO_ESTATE, "arenas are not bound (zero_bind)");
  if (!c->loaded) return fail(c, ZERO_ESTATE, "state is not initialised (zero_load_master)");
  if (need_hp && !c->have_hp) return fail(c, ZERO_ESTATE, "hyper-parameters are not set (zero_set_hparams)");
  return ZERO_OK;
}

// Which flat ranges a stage's step walks: the bucket schedule (stage 1, 2) or
// the layers from last to first (stage 3).
std::vector<zsm::Span> step_intervals(const zero_ctx* c) {
  std::vector<zsm::Span> out;
  if (c->stage == ZERO_STAGE_3) {
    for (auto it = c->plan.layers.rbegin(); it != c->plan.layers.rend(); ++it) out.push_back({it->lo, it->hi});
  } else {
    out = c->plan.buckets;
  }
  return out;
}

// A launch range against the planner's buffers: inside the flat space, on
// the 8-element granule, and no longer than the buffer it passes through
// (the stage-3 layer buffers; the stage-2 gradient bucket when the
// gradients come through it).  A failure is a planner error, reported
// before anything is launched.
zero_status check_launch_range(zero_ctx* c, int64_t lo, int64_t hi, bool through_bucket) {
  const zsm::Plan& p = c->plan;
  const bool ok = 0 <= lo && lo <= hi && hi <= p.psi_pad && lo % zsm::kVec == 0 && hi % zsm::kVec == 0 &&
                  (c->stage != ZERO_STAGE_3 || hi - lo <= p.max_layer) &&
                  (!through_bucket || c->stage != ZERO_STAGE_2 || hi - lo <= p.max_bucket);
  if (ok) return ZERO_OK;
  return fail(c, ZERO_EINVAL, "launch range [%lld, %lld) does not fit the plan (psi_pad %lld, largest layer %lld, "
              "bucket %lld)", (long long)lo, (long long)hi, (long long)p.psi_pad, (long long)p.max_layer,
              (long long)p.max_bucket);
}

// One fused launch over [lo, hi).  grad[r] are at flat element lo.
zero_status fused_interval(zero_ctx* c, int64_t lo, int64_t hi, uint16_t* const* grad, int layer_idx,
                           bool accumulate, const zsm::AdamScalars& sc, cudaStream_t s, int slot = 0,
                           int pdl = zsm::kPdlNone, const zsm::AdamScalars* sc_dev = nullptr, bool twin = false,
                           bool through_bucket = false) {
  if (hi == lo) return ZERO_OK;
  {
    const zero_status st = check_launch_range(c, lo, hi, through_bucket);
    if (st != ZERO_OK) return st;
  }
  const int N = c->plan.n_ranks;
  zsm::FusedArgs a;
  std::memset(&a, 0, sizeof a);
  a.fmt = c->fmt;
  for (int r = 0; r < N; ++r) {
    a.grad[r] = grad[r];
    if (c->stage == ZERO_STAGE_3) {
      const int64_t off = lo - c->plan.layers[layer_idx].lo;
      a.out[r] = gather_ptr(c, r, slot) + off;
    } else {
      a.out[r] = param_ptr(c, r) + lo;
    }
  }
  a.master = master_ptr(c) + lo;
  a.m = m_ptr(c) + lo;
  a.v = v_ptr(c) + lo;
  a.grad_shard = c->arena[ZERO_ARENA_GRAD_SHARDS] ? grad_shard_ptr(c) + lo : nullptr;
  a.param_shard = c->stage == ZERO_STAGE_3 ? param_ptr(c, 0) + lo : nullptr;
  a.n_vec = (hi - lo) / zsm::kVec;
  a.n_ranks = N;
  a.accumulate = accumulate ? 1 : 0;
  a.inv_n = (float)(1.0 / (double)N);
  a.sc = sc;
  a.sc_dev = sc_dev;
  a.ns = norm_scratch(c);
  a.pdl = c->timing ? zsm::kPdlNone : pdl;  // an event record between launches ends the overlap
  a.store_hint = c->store_hint >= 0 ? c->store_hint : bulk_policy(c->plan.n_ranks, c->stage).hint;
  const int mode = c->stage == ZERO_STAGE_1 ? zsm::kFusedZ1 : c->stage == ZERO_STAGE_2 ? zsm::kFusedZ2 : zsm::kFusedZ3;
  cudaEvent_t* ev = c->timing ? timing_pair(c) : nullptr;
  if (ev) cudaEventRecord(ev[0], s);
  cudaError_t e;
  if (twin || use_bulk(c)) {
    const int64_t tiles = (hi - lo + bulk_tile(c) - 1) / bulk_tile(c);
    e = counted(c, zsm::launch_fused_bulk(mode, a, (int)std::max<int64_t>(1, std::min<int64_t>(tiles, c->sm_count)),
                                          bulk_tile(c), bulk_warps(c), bulk_ring(c), twin, 0u, s));
  } else if (use_chunked(c)) {
    const int64_t tiles = (hi - lo + kTmaTile - 1) / kTmaTile;
    e = counted(c, zsm::launch_fused_chunked(mode, a, (int)std::max<int64_t>(1, std::min<int64_t>(tiles, c->sm_count)),
                                  chunked_stages(c), s));
  } else if (use_tma(c)) {
    const int64_t tiles = (hi - lo + kTmaTile - 1) / kTmaTile;
    e = counted(c, zsm::launch_fused_tma(mode, a, (int)std::max<int64_t>(1, std::min<int64_t>(tiles, tma_grid_cap(c))),
                              tma_groups(c), tma_stages(c), s));
  } else {
    e = counted(c, zsm::launch_fused(mode, a, grid_for(a.n_vec, c->grid_fused), s));
  }
  if (e != cudaSuccess) return cuda_fail(c, e, "fused step kernel launch");
  if (ev) {
    cudaEventRecord(ev[1], s);
    c->timed += 1;
    c->timed_bytes += (double)fused_bytes_per_elem(c) * (double)(hi - lo);
  }
  return ZERO_OK;
}

// A callback-free stage-3 step as one launch (ZERO_OPT_LAYERED): the
// bulk-store kernel at N <= 16, at least two non-empty layers, at most
// kMaxSegments, and one CTA per SM.
bool layered_ok(const zero_ctx* c, bool callbacks, const std::vector<zsm::Span>& iv) {
  if (!c->layered || callbacks || c->stage != ZERO_STAGE_3 || !use_bulk(c) || !bulk_fits(c) ||
      c->plan.n_ranks > zsm::kTmaMaxRanks || c->tma_ctas_opt > 1)
    return false;
  int n = 0;
  for (const zsm::Span& sp : iv) n += sp.hi > sp.lo ? 1 : 0;
  return n >= 2 && n <= zsm::kMaxSegments;
}

// Every layer of the schedule in one cooperative launch of the bulk-store
// kernel: the layers in schedule order (last to first), each CTA's ring
// running on across layer boundaries, and each layer's stores into the
// temporary layer buffers issued only after every CTA has finished storing
// the layers before it -- the order of the per-layer launches, without a
// launch boundary at each layer.  grad0[r] are the ranks' full replicas.
// *refused: the device could not hold every CTA at once (a cooperative launch
// refused, e.g. with fewer SMs available to this process); nothing was
// launched, and the caller runs one launch per layer instead.
zero_status fused_layered(zero_ctx* c, const std::vector<zsm::Span>& iv, uint16_t* const* grad0, cudaStream_t s,
                          const zsm::AdamScalars* sc_dev, bool twin, bool* refused) {
  *refused = false;
  const int N = c->plan.n_ranks;
  zsm::FusedArgs a;
  std::memset(&a, 0, sizeof a);
  a.fmt = c->fmt;
  for (int r = 0; r < N; ++r) {
    a.grad[r] = grad0[r];
    a.out[r] = gather_ptr(c, r, 0);
  }
  a.master = master_ptr(c);
  a.m = m_ptr(c);
  a.v = v_ptr(c);
  a.grad_shard = c->arena[ZERO_ARENA_GRAD_SHARDS] ? grad_shard_ptr(c) : nullptr;
  a.param_shard = param_ptr(c, 0);
  a.n_vec = c->plan.psi_pad / zsm::kVec;
  a.n_ranks = N;
  a.accumulate = 0;
  a.inv_n = (float)(1.0 / (double)N);
  a.sc_dev = sc_dev;
  a.ns = norm_scratch(c);
  a.pdl = zsm::kPdlNone;
  a.store_hint = c->store_hint >= 0 ? c->store_hint : bulk_policy(c->plan.n_ranks, c->stage).hint;
  zsm::SegTable g;
  std::memset(&g, 0, sizeof g);
  g.counter = reinterpret_cast<unsigned*>(c->arena[ZERO_ARENA_SCRATCH] + kSegCounterOffset);
  int64_t elems = 0, max_tiles = 1;
  const int64_t tile = bulk_tile(c);
  for (const zsm::Span& sp : iv) {
    if (sp.hi == sp.lo) continue;
    const zero_status st = check_launch_range(c, sp.lo, sp.hi, false);
    if (st != ZERO_OK) return st;
    g.lo[g.n] = sp.lo;
    g.len[g.n] = sp.hi - sp.lo;
    ++g.n;
    elems += sp.hi - sp.lo;
    max_tiles = std::max(max_tiles, (sp.hi - sp.lo + tile - 1) / tile);
  }
  const NvtxRange range(c->nvtx, "layers x %d [%lld, %lld) in one launch", g.n, (long long)g.lo[g.n - 1],
                        (long long)(g.lo[0] + g.len[0]));
  cudaError_t e = cudaMemsetAsync(g.counter, 0, sizeof(unsigned), s);
  if (e != cudaSuccess) return cuda_fail(c, e, "clearing the layered launch's counter");
  cudaEvent_t* ev = c->timing ? timing_pair(c) : nullptr;
  if (ev) cudaEventRecord(ev[0], s);
  e = zsm::launch_fused_bulk_layered(a, g, (int)std::min<int64_t>(max_tiles, c->sm_count), (int)tile,
                                     bulk_warps(c), bulk_ring(c), twin, s);
  if (e == cudaErrorCooperativeLaunchTooLarge) {
    (void)cudaGetLastError();  // a launch-configuration error: the context stays usable
    *refused = true;            // (an event pair recorded above is re-recorded by the next timed launch)
    return ZERO_OK;
  }
  e = counted(c, e);
  if (e != cudaSuccess) return cuda_fail(c, e, "layered fused step kernel launch");
  if (ev) {
    cudaEventRecord(ev[1], s);
    c->timed += 1;
    c->timed_bytes += (double)fused_bytes_per_elem(c) * (double)elems;
  }
  return ZERO_OK;
}

// Reads and clears the device error word (a bounded wait that ran out).
zero_status check_device_error(zero_ctx* c, unsigned int err, cudaStream_t s) {
  if (err == 0) return ZERO_OK;
  cudaMemsetAsync(norm_scratch(c).error, 0, sizeof(unsigned int), s);
  return fail(c, ZERO_ECUDA, "a bounded wait in the staged fused kernel ran out (code %u): results of the step are invalid", err);
}

// Synchronises `s` and reads the last step's statistics, its decision and
// the step counter from the device in one copy.
zero_status finish_stats(zero_ctx* c, cudaStream_t s, zero_step_stats* out) {
  StatsBlock host;
  cudaError_t e = cudaMemcpyAsync(&host, stats_block(c), sizeof host, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(c, e, "reading step statistics");
  zero_status st = check_device_error(c, host.error, s);
  if (st != ZERO_OK) return st;
  c->t = (int64_t)host.state.t;
  std::memset(out, 0, sizeof *out);
  out->grad_norm = std::sqrt(host.sq) / c->loss_scale;
  out->nonfinite = (int64_t)host.nf;
  out->step = c->t;
  zero_comm_elems(c, out->comm_elems);
  out->clip_coef = host.dec.coef < 1.0f ? (double)host.dec.coef : 1.0;
  out->skipped = host.dec.skip ? 1 : 0;
  return ZERO_OK;
}

// Orders one step's work across the caller's stream `s`, the stream the
// callbacks get (`q`) and the stream of the step's kernels (`ks`).  Without
// ZERO_OPT_PIPELINE all three are `s` and everything runs in program order
// with one slot set.  With it, the callbacks run on the context's side stream
// one interval ahead -- grad_fn(k+1) and gather_fn(k) overlap the kernel of
// interval k+1 or k -- and the kernels on `s` (option value 1) or on a
// stream of the context's own at the device's greatest priority (value 2,
// so that their CTAs take the SMs the callbacks' work frees first).  Events
// keep each slot set from being refilled before its reader is done:
//   grad_fn(k)   (q)    after the kernel of k-2 read slot k%2 (stage 2/3)
//   kernel(k)    (ks)   after grad_fn(k), and (stage 3) after gather_fn(k-2)
//                       finished reading gather slot k%2
//   gather_fn(k) (q)    after kernel(k)
// and `s` waits for all of q's and ks's work before the step returns.
struct StepOrder {
  zero_ctx* c;
  cudaStream_t s;
  cudaStream_t q;
  cudaStream_t ks;
  bool on;
  bool joined = false;
  cudaError_t err = cudaSuccess;

  // `callbacks`: the step calls grad_fn or gather_fn (without any there is
  // nothing to run ahead, and the step stays on `s` alone)
  StepOrder(zero_ctx* ctx, cudaStream_t stream, bool callbacks)
      : c(ctx), s(stream), q(stream), ks(stream), on(ctx->pipeline != 0 && callbacks) {
    if (on) q = c->side;
    if (on && c->pipeline == 2) ks = c->kside;
  }
  void record(cudaEvent_t e, cudaStream_t st) {
    if (err == cudaSuccess) err = cudaEventRecord(e, st);
  }
  void wait(cudaStream_t st, cudaEvent_t e) {
    if (err == cudaSuccess) err = cudaStreamWaitEvent(st, e, 0);
  }
  int slot(size_t k) const { return (on && c->slots == 2) ? (int)(k & 1) : 0; }
  size_t ahead() const { return on ? 1 : 0; }
  void begin() {
    if (!on) return;
    record(c->ev_start, s);
    wait(q, c->ev_start);
    if (ks != s) wait(ks, c->ev_start);
  }
  void before_grads(size_t k) {
    if (on && c->slots == 2 && k >= 2) wait(q, c->ev_kernel[k & 1]);
  }
  void after_grads(size_t k) {
    if (on) record(c->ev_grads[k & 1], q);
  }
  void before_kernel(size_t k, bool grads, size_t gather_k) {
    if (!on) return;
    if (grads) wait(ks, c->ev_grads[k & 1]);
    if (gather_k != (size_t)-1 && gather_k >= 2) wait(ks, c->ev_consumed[gather_k & 1]);
  }
  void after_kernel(size_t k) {
    if (on) record(c->ev_kernel[k & 1], ks);
  }
  void before_gather(size_t k) {
    if (on) wait(q, c->ev_kernel[k & 1]);
  }
  void after_gather(size_t k) {
    if (on) record(c->ev_consumed[k & 1], q);
  }
  // Joins the callbacks' and the kernels' streams into `s`; returns the
  // first CUDA error seen.
  cudaError_t end() {
    if (on && !joined) {
      joined = true;
      // the join is attempted even after an error, so that `s` never runs ahead
      // of work already enqueued on the other streams
      cudaError_t e1 = cudaEventRecord(c->ev_join, q);
      cudaError_t e2 = e1 == cudaSuccess ? cudaStreamWaitEvent(s, c->ev_join, 0) : e1;
      if (ks != s) {
        cudaError_t e3 = cudaEventRecord(c->ev_kjoin, ks);
        cudaError_t e4 = e3 == cudaSuccess ? cudaStreamWaitEvent(s, c->ev_kjoin, 0) : e3;
        if (e2 == cudaSuccess) e2 = e4;
      }
      if (err == cudaSuccess) err = e2;
    }
    return err;
  }
};

// Creates the side stream and events of ZERO_OPT_PIPELINE on first use.
// Creates what ZERO_OPT_PIPELINE needs and the caller did not give
// (zero_set_pipeline_streams) on first use: the streams and the events.
zero_status ensure_pipeline(zero_ctx* c) {
  if (!c->pipeline) return ZERO_OK;
  c->pipeline_used = true;
  cudaError_t e = cudaSuccess;
  if (!c->side) {
    e = cudaStreamCreateWithFlags(&c->side, cudaStreamNonBlocking);
    c->own_side = e == cudaSuccess;
  }
  if (e == cudaSuccess && c->pipeline == 2 && !c->kside) {
    int least = 0, greatest = 0;
    e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
    if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&c->kside, cudaStreamNonBlocking, greatest);
    c->own_kside = e == cudaSuccess;
  }
  for (cudaEvent_t* ev : {&c->ev_start, &c->ev_join, &c->ev_kjoin, &c->ev_grads[0], &c->ev_grads[1],
                          &c->ev_kernel[0], &c->ev_kernel[1], &c->ev_consumed[0], &c->ev_consumed[1]})
    if (e == cudaSuccess && !*ev) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
  if (e != cudaSuccess) return cuda_fail(c, e, "creating the pipeline streams and events");
  return ZERO_OK;
}

// The N gradient pointers of interval k (at flat element lo): the caller's
// resident replicas, the full replicas at stage 1, or slot k's buffers.
void interval_grads(zero_ctx* c, const void* const* resident, int64_t lo, int slot, uint16_t** out) {
  const int N = c->plan.n_ranks;
  for (int r = 0; r < N; ++r) {
    if (resident)
      out[r] = const_cast<uint16_t*>(static_cast<const uint16_t*>(resident[r])) + lo;
    else
      out[r] = c->stage == ZERO_STAGE_1 ? grad_buf_ptr(c, r) + lo : grad_buf_ptr(c, r, slot);
  }
}

// Calls grad_fn for interval k of `iv` (no-op with resident gradients).
zero_status issue_grads(zero_ctx* c, StepOrder& o, zero_grad_fn fn, void* user, const void* const* resident,
                        const std::vector<zsm::Span>& iv, size_t k, int64_t t) {
  if (resident || !fn) return ZERO_OK;
  const int N = c->plan.n_ranks;
  std::vector<uint16_t*> bufs(N);
  interval_grads(c, nullptr, iv[k].lo, o.slot(k), bufs.data());
  o.before_grads(k);
  const int rc = fn(user, t, iv[k].lo, iv[k].hi, reinterpret_cast<void* const*>(bufs.data()), o.q);
  if (rc != 0)
    return fail(c, ZERO_EINVAL, "grad_fn returned %d for [%lld, %lld)", rc, (long long)iv[k].lo, (long long)iv[k].hi);
  o.after_grads(k);
  return ZERO_OK;
}

// Calls gather_fn for stage-3 layer `layer_idx`, whose gathered copy is in
// gather slot `slot`.
zero_status issue_gather(zero_ctx* c, StepOrder& o, zero_gather_fn gfn, void* guser, int layer_idx, size_t k) {
  const int N = c->plan.n_ranks;
  std::vector<uint16_t*> bufs(N);
  for (int r = 0; r < N; ++r) bufs[r] = gather_ptr(c, r, o.slot(k));
  const zsm::LayerSpan& L = c->plan.layers[layer_idx];
  o.before_gather(k);
  const int rc = gfn(guser, L.id, L.lo, L.hi, reinterpret_cast<void* const*>(bufs.data()), o.q);
  if (rc != 0) return fail(c, ZERO_EINVAL, "gather_fn returned %d for layer %d", rc, L.id);
  o.after_gather(k);
  return ZERO_OK;
}

// The two-pass step's kernels (and the unfused reduce calls): staged through
// shared memory unless the register path is asked for; timed
// (ZERO_OPT_TIMING) like the fused launches, with their own byte models.
bool use_two_pass_tma(const zero_ctx* c) { return c->kernel_opt != ZERO_KERNEL_REGISTER; }

int two_pass_grid(const zero_ctx* c, int64_t elems) {
  const int64_t tiles = (elems + zsm::two_pass_tile() - 1) / zsm::two_pass_tile();
  return (int)std::max<int64_t>(1, std::min<int64_t>(tiles, c->sm_count));
}

cudaError_t launch_pass1(zero_ctx* c, const zsm::ReduceArgs& a, cudaStream_t s) {
  const int64_t elems = a.n_vec * zsm::kVec;
  cudaEvent_t* ev = c->timing ? timing_pair(c) : nullptr;
  if (ev) cudaEventRecord(ev[0], s);
  cudaError_t e;
  if (use_bulk(c) && a.write_back && a.n_ranks <= zsm::kTmaMaxRanks) {
    // the all-reduce's N write-backs through bulk stores: 1024-element tiles,
    // as deep a ring as fits (8 stages, 128 KB at N = 8) unless it is set; the
    // reduce-scatter's single shard store stays with the staged reduce, whose
    // 2048-element ring keeps more loads in flight (measured 12 % faster there)
    const int64_t tiles = (elems + 1023) / 1024;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(tiles, c->sm_count));
    e = counted(c, zsm::launch_reduce_bulk(a, grid, c->tma_stages_opt ? c->tma_stages_opt : 8,
                                           c->store_hint >= 0 ? c->store_hint : 1, s));
  } else {
    e = counted(c, use_two_pass_tma(c) ? zsm::launch_reduce_tma(a, two_pass_grid(c, elems), s)
                                       : zsm::launch_reduce(a, grid_for(a.n_vec, c->grid_simple), s));
  }
  if (e == cudaSuccess && ev) {
    cudaEventRecord(ev[1], s);
    c->timed += 1;
    c->timed_bytes += (double)(a.write_back ? 4 * a.n_ranks : 2 * a.n_ranks + 2) * (double)elems;
  }
  return e;
}

cudaError_t launch_pass2(zero_ctx* c, const zsm::AdamBcastArgs& b, bool uniform, cudaStream_t s) {
  const int64_t elems = b.n_vec * zsm::kVec;
  cudaEvent_t* ev = c->timing ? timing_pair(c) : nullptr;
  if (ev) cudaEventRecord(ev[0], s);
  cudaError_t e;
  if (use_bulk(c)) {
    // the bulk-store pass 2: four 1024-element stages unless the ring depth is set
    const int64_t tiles = (elems + zsm::bulk_bcast_tile() - 1) / zsm::bulk_bcast_tile();
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(tiles, c->sm_count));
    e = counted(c, zsm::launch_adam_bcast_bulk(b, grid, uniform, c->tma_stages_opt ? c->tma_stages_opt : 4,
                                               c->store_hint >= 0 ? c->store_hint : 1, s));
  } else {
    e = counted(c, use_two_pass_tma(c) ? zsm::launch_adam_bcast_tma(b, two_pass_grid(c, elems), uniform, s)
                                       : zsm::launch_adam_bcast(b, grid_for(b.n_vec, c->grid_simple), s));
  }
  if (e == cudaSuccess && ev) {
    cudaEventRecord(ev[1], s);
    c->timed += 1;
    c->timed_bytes += (double)(2 + 24 + 2 * b.n_out + (b.param_shard ? 2 : 0)) * (double)elems;
  }
  return e;
}

// Clipped / overflow-checked step: reduce everything, read the norm, then
// Adam + broadcast.
// Pass 2 of a clipped stage-3 step without a gather callback as one
// cooperative launch over its layers (ZERO_OPT_LAYERED, the bulk-store pass
// 2): each layer's stores into the temporary layer buffers follow every
// CTA's stores of the layers before it.  *refused: the device could not hold
// every CTA at once; nothing was launched.
zero_status pass2_layered(zero_ctx* c, const std::vector<zsm::Span>& iv, zsm::ClipDecision* dec, cudaStream_t s,
                          bool* refused) {
  *refused = false;
  const int N = c->plan.n_ranks;
  zsm::AdamBcastArgs b;
  std::memset(&b, 0, sizeof b);
  b.fmt = c->fmt;
  for (int r = 0; r < N; ++r) {
    b.gsrc[r] = grad_shard_ptr(c);
    b.out[r] = gather_ptr(c, r, 0);
  }
  b.n_out = N;
  b.master = master_ptr(c);
  b.m = m_ptr(c);
  b.v = v_ptr(c);
  b.param_shard = param_ptr(c, 0);
  b.lo = 0;
  b.shard = c->plan.shard;
  b.n_vec = c->plan.psi_pad / zsm::kVec;
  b.sc_dev = &state_ptr(c)->sc;
  b.dec = dec;
  b.error = norm_scratch(c).error;
  b.wait_ns = c->wait_ns;
  zsm::SegTable g;
  std::memset(&g, 0, sizeof g);
  g.counter = reinterpret_cast<unsigned*>(c->arena[ZERO_ARENA_SCRATCH] + kSegCounterOffset);
  int64_t elems = 0, max_tiles = 1;
  const int64_t tile = zsm::bulk_bcast_tile();
  for (const zsm::Span& sp : iv) {
    if (sp.hi == sp.lo) continue;
    const zero_status st = check_launch_range(c, sp.lo, sp.hi, false);
    if (st != ZERO_OK) return st;
    g.lo[g.n] = sp.lo;
    g.len[g.n] = sp.hi - sp.lo;
    ++g.n;
    elems += sp.hi - sp.lo;
    max_tiles = std::max(max_tiles, (sp.hi - sp.lo + tile - 1) / tile);
  }
  const NvtxRange range(c->nvtx, "update layers x %d [%lld, %lld) in one launch", g.n, (long long)g.lo[g.n - 1],
                        (long long)(g.lo[0] + g.len[0]));
  cudaError_t e = cudaMemsetAsync(g.counter, 0, sizeof(unsigned), s);
  if (e != cudaSuccess) return cuda_fail(c, e, "clearing the layered launch's counter");
  cudaEvent_t* ev = c->timing ? timing_pair(c) : nullptr;
  if (ev) cudaEventRecord(ev[0], s);
  e = zsm::launch_adam_bcast_bulk_layered(b, g, (int)std::min<int64_t>(max_tiles, c->sm_count), true,
                                          c->tma_stages_opt ? c->tma_stages_opt : 4,
                                          c->store_hint >= 0 ? c->store_hint : 1, s);
  if (e == cudaErrorCooperativeLaunchTooLarge) {
    (void)cudaGetLastError();  // a launch-configuration error: the context stays usable
    *refused = true;
    return ZERO_OK;
  }
  e = counted(c, e);
  if (e != cudaSuccess) return cuda_fail(c, e, "layered adam-broadcast kernel launch");
  if (ev) {
    cudaEventRecord(ev[1], s);
    c->timed += 1;
    c->timed_bytes += (double)(2 + 24 + 2 * N + 2) * (double)elems;
  }
  return ZERO_OK;
}

zero_status run_two_pass(zero_ctx* c, zero_grad_fn fn, void* user, const void* const* resident,
                         zero_gather_fn gfn, void* guser, StepOrder& o, zero_step_stats* stats) {
  const int N = c->plan.n_ranks;
  if (c->stage != ZERO_STAGE_1 && !c->arena[ZERO_ARENA_GRAD_SHARDS])
    return fail(c, ZERO_ESTATE, "clipping / skipping needs the reduced-gradient shards (ZERO_OPT_KEEP_GRAD_SHARDS = 1)");
  cudaStream_t s = o.ks;  // the step's kernels; statistics are read on o.s after the join
  const int64_t t = c->calls + 1;  // the callbacks' step number (the kernels use the device's count)
  const std::vector<zsm::Span> iv = step_intervals(c);
  const int n_layers = (int)c->plan.layers.size();
  std::vector<uint16_t*> grad(N);
  // the scalars of step t + 1 from the device step state, committed by the decision
  {
    const cudaError_t e = counted(c, zsm::launch_step_begin(state_ptr(c), step_hparams(c), nullptr, s));
    if (e != cudaSuccess) return cuda_fail(c, e, "step-begin kernel launch");
  }
  // pass 1: reduce every interval.  Resident gradients are all there at
  // once and pass 1 writes only the flat shard (or, at stage 1, each
  // replica in place), so the whole flat space is reduced in one launch; the
  // intervals are for gradients that arrive interval by interval.
  const std::vector<zsm::Span> p1 = resident ? std::vector<zsm::Span>{zsm::Span{0, c->plan.psi_pad}} : iv;
  bool launched = false;  // the first launch of the step starts the norm sum
  size_t issued = 0;
  for (size_t k = 0; k < p1.size(); ++k) {
    for (; !resident && issued < iv.size() && issued <= k + o.ahead(); ++issued) {
      zero_status st = issue_grads(c, o, fn, user, resident, iv, issued, t);
      if (st != ZERO_OK) return st;
    }
    const int64_t lo = p1[k].lo, hi = p1[k].hi;
    zsm::ReduceArgs a;
    std::memset(&a, 0, sizeof a);
    a.fmt = c->fmt;
    interval_grads(c, resident, lo, o.slot(k), grad.data());
    for (int r = 0; r < N; ++r) a.grad[r] = grad[r];
    a.shard_out = c->stage == ZERO_STAGE_1 ? nullptr : grad_shard_ptr(c) + lo;
    a.write_back = c->stage == ZERO_STAGE_1 ? 1 : 0;
    a.n_vec = (hi - lo) / zsm::kVec;
    a.n_ranks = N;
    a.accumulate = launched ? 1 : 0;
    a.inv_n = (float)(1.0 / (double)N);
    a.ns = norm_scratch(c);
    o.before_kernel(k, !resident && fn, (size_t)-1);
    if (a.n_vec > 0) {
      const NvtxRange range(c->nvtx, "reduce %s %d [%lld, %lld)",
                            resident ? "all" : c->stage == ZERO_STAGE_3 ? "layer" : "bucket",
                            resident ? 0 : c->stage == ZERO_STAGE_3 ? c->plan.layers[n_layers - 1 - (int)k].id : (int)k,
                            (long long)lo, (long long)hi);
      cudaError_t e = launch_pass1(c, a, s);
      if (e != cudaSuccess) return cuda_fail(c, e, "reduce kernel launch");
      launched = true;
    }
    o.after_kernel(k);
  }
  if (o.err != cudaSuccess) return cuda_fail(c, o.err, "ordering the pipeline streams");
  // The decision -- norm, skip, clipping coefficient -- is taken on the device
  // from the sums pass 1 left and read there by pass 2, so nothing waits
  // between the passes; it also commits the step counter unless the step is
  // skipped.
  zero_status st = ZERO_OK;
  zsm::ClipParams cp;
  cp.max_norm = c->clip_norm;
  cp.loss_scale = c->loss_scale;
  cp.skip_nonfinite = c->skip_nonfinite ? 1 : 0;
  zsm::ClipDecision* dec = decision_ptr(c);
  cudaError_t e;
  {
    const NvtxRange range(c->nvtx, "clip decision");
    e = counted(c, zsm::launch_clip_decide(norm_scratch(c), cp, dec, state_ptr(c), s));
  }
  if (e != cudaSuccess) return cuda_fail(c, e, "the clipped step's decision");
  const zsm::AdamScalars sc{};  // the kernels read the step's scalars from the device step state
  // pass 2: Adam + broadcast, over everything (stage 1/2) or per layer (stage 3);
  // a skipped step writes the unchanged parameters only
  std::vector<zsm::Span> p2;
  if (c->stage == ZERO_STAGE_3) p2 = iv;
  else p2.push_back({0, c->plan.psi_pad});
  if (c->stage == ZERO_STAGE_3 && !gfn && c->layered && use_bulk(c)) {
    int n = 0;
    for (const zsm::Span& sp : iv) n += sp.hi > sp.lo ? 1 : 0;
    if (n >= 2 && n <= zsm::kMaxSegments) {
      bool refused = false;
      st = pass2_layered(c, iv, dec, s, &refused);
      if (st != ZERO_OK) return st;
      if (!refused) p2.clear();  // every layer done in the one launch
    }
  }
  for (size_t k = 0; k < p2.size(); ++k) {
    const int64_t lo = p2[k].lo, hi = p2[k].hi;
    const int layer_idx = c->stage == ZERO_STAGE_3 ? n_layers - 1 - (int)k : 0;
    zsm::AdamBcastArgs b;
    std::memset(&b, 0, sizeof b);
    b.fmt = c->fmt;
    for (int r = 0; r < N; ++r) {
      if (c->stage == ZERO_STAGE_1)
        b.gsrc[r] = resident ? static_cast<const uint16_t*>(resident[r]) : grad_buf_ptr(c, r);
      else
        b.gsrc[r] = grad_shard_ptr(c);
      b.out[r] = c->stage == ZERO_STAGE_3 ? gather_ptr(c, r, o.slot(k)) : param_ptr(c, r) + lo;
    }
    b.n_out = N;
    b.master = master_ptr(c) + lo;
    b.m = m_ptr(c) + lo;
    b.v = v_ptr(c) + lo;
    b.param_shard = c->stage == ZERO_STAGE_3 ? param_ptr(c, 0) + lo : nullptr;
    b.lo = lo;
    b.shard = c->plan.shard;
    b.n_vec = (hi - lo) / zsm::kVec;
    b.sc = sc;
    b.sc_dev = &state_ptr(c)->sc;
    b.dec = dec;
    b.error = norm_scratch(c).error;
    b.wait_ns = c->wait_ns;
    o.before_kernel(k, false, c->stage == ZERO_STAGE_3 && gfn ? k : (size_t)-1);
    if (b.n_vec > 0) {
      const NvtxRange range(c->nvtx, "update %s %d [%lld, %lld)", c->stage == ZERO_STAGE_3 ? "layer" : "all",
                            c->stage == ZERO_STAGE_3 ? c->plan.layers[layer_idx].id : 0, (long long)lo,
                            (long long)hi);
      // stages 2 and 3 read every owner's reduced gradient from the one shard array
      e = launch_pass2(c, b, c->stage != ZERO_STAGE_1, s);
      if (e != cudaSuccess) return cuda_fail(c, e, "adam-broadcast kernel launch");
    }
    o.after_kernel(k);
    if (c->stage == ZERO_STAGE_3 && gfn) {
      st = issue_gather(c, o, gfn, guser, layer_idx, k);
      if (st != ZERO_OK) return st;
    }
  }
  if (o.end() != cudaSuccess) return cuda_fail(c, o.err, "ordering the pipeline streams");
  c->calls = t;
  c->norm_fresh = true;
  if (stats) return finish_stats(c, o.s, stats);
  return ZERO_OK;
}

// Checks the guard bytes on `s` and waits for the result; out = {changed
// bytes, arena of the first, its byte offset in the arena} (-1, -1 when none).
zero_status check_guards(zero_ctx* c, cudaStream_t s, int64_t out[3]) {
  out[0] = 0;
  out[1] = out[2] = -1;
  zsm::GuardArgs g;
  if (!guard_args(c, &g)) return fail(c, ZERO_EINVAL, "guard layout does not match the arenas");
  unsigned long long h[2] = {0ull, ~0ull};
  cudaError_t e = cudaMemcpyAsync(g.result, h, sizeof h, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = counted(c, zsm::launch_guards(g, true, s));
  if (e == cudaSuccess) e = cudaMemcpyAsync(h, g.result, sizeof h, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(c, e, "guard check");
  if (h[0] == 0) return ZERO_OK;
  const int arena = (int)(h[1] >> 56);
  const int64_t off = (int64_t)(h[1] & ((1ull << 56) - 1));
  out[0] = (int64_t)h[0];
  out[1] = arena;
  out[2] = off;
  const zsm::GuardSet& gs = g.set[arena];
  if (off >= gs.rows * gs.pitch)
    return fail(c, ZERO_EGUARD, "%lld guard bytes changed; the first: arena %d, byte %lld of its %lld-byte tail",
                (long long)h[0], arena, (long long)(off - gs.rows * gs.pitch), (long long)gs.tail);
  return fail(c, ZERO_EGUARD, "%lld guard bytes changed; the first: arena %d, row %lld, byte %lld past its %lld used bytes",
              (long long)h[0], arena, (long long)(off / gs.pitch), (long long)(off % gs.pitch - gs.used),
              (long long)gs.used);
}

zero_status run_step(zero_ctx* c, zero_grad_fn fn, void* user, const void* const* resident,
                     zero_gather_fn gfn, void* guser, void* stream, zero_step_stats* stats) {
  zero_status st = check_ready(c, true);
  if (st != ZERO_OK) return st;
  const int N = c->plan.n_ranks;
  if (resident) {
    for (int r = 0; r < N; ++r)
      if (!resident[r] || !aligned16(resident[r]))
        return fail(c, ZERO_EINVAL, "rank_grads[%d] is null or not 16-byte aligned", r);
  } else if (!fn && c->stage != ZERO_STAGE_1) {
    return fail(c, ZERO_EINVAL, "grad_fn may be NULL only for stage 1");
  } else if (!c->arena[ZERO_ARENA_GRADS]) {
    return fail(c, ZERO_ESTATE, "no gradient buffers (ZERO_OPT_GRAD_BUFFERS = 0): use zero_step_resident");
  }
  st = ensure_pipeline(c);
  if (st != ZERO_OK) return st;
  const bool callbacks = (!resident && fn) || (c->stage == ZERO_STAGE_3 && gfn);
  StepOrder o(c, static_cast<cudaStream_t>(stream), callbacks);
  const NvtxRange step_range(c->nvtx, "step %lld (stage %d, N = %d)", (long long)(c->calls + 1), c->stage, N);
  o.begin();
  if (c->clip_norm > 0.0 || c->skip_nonfinite) {
    st = run_two_pass(c, fn, user, resident, gfn, guser, o, stats);
    o.end();  // joins the side stream also on the error paths
    return st;
  }
  cudaStream_t s = o.ks;  // the step's kernels
  const int64_t t = c->calls + 1;  // the callbacks' step number (the kernels use the device's count)
  // the kernels read the step's scalars from the device step state (no host
  // copy: forming beta^t on the host would cost t multiplications a step)
  const zsm::AdamScalars sc{};
  {
    const cudaError_t e = counted(c, zsm::launch_step_begin(state_ptr(c), step_hparams(c), decision_ptr(c), s));
    if (e != cudaSuccess) return cuda_fail(c, e, "step-begin kernel launch");
  }
  const std::vector<zsm::Span> iv = step_intervals(c);
  std::vector<uint16_t*> grad(N);
  const int n_layers = (int)c->plan.layers.size();
  const bool gathers = c->stage == ZERO_STAGE_3 && gfn;
  bool launched = false;  // the first non-empty launch of the step starts the norm sum
  size_t issued = 0;
  // Programmatic dependent launch only between this step's own back-to-back
  // launches: with callbacks other work sits between them.  The first launch
  // follows unknown work and waits for it before touching memory; the later
  // ones at stage 1/2 touch disjoint intervals and share only the norm
  // scratch, so they stream at once; stage 3's launches all write the one
  // temporary gather buffer, so they load and compute at once but store only
  // after the launch before has finished.
  // (and not with two staged CTAs per SM asked for: a programmatic launch
  // keeps one per SM)
  const bool pdl_ok = c->pdl && !callbacks && c->tma_ctas_opt <= 1;
  bool one_launch = layered_ok(c, callbacks, iv);  // every layer in one launch
  if (one_launch) {
    interval_grads(c, resident, 0, 0, grad.data());
    bool refused = false;
    st = fused_layered(c, iv, grad.data(), s, &state_ptr(c)->sc, false, &refused);
    one_launch = !refused;
  }
  for (size_t k = 0; k < iv.size() && st == ZERO_OK && !one_launch; ++k) {
    for (; issued < iv.size() && issued <= k + o.ahead() && st == ZERO_OK; ++issued)
      st = issue_grads(c, o, fn, user, resident, iv, issued, t);
    if (st != ZERO_OK) break;
    const int64_t lo = iv[k].lo, hi = iv[k].hi;
    const int layer_idx = c->stage == ZERO_STAGE_3 ? n_layers - 1 - (int)k : 0;
    interval_grads(c, resident, lo, o.slot(k), grad.data());
    o.before_kernel(k, !resident && fn, gathers ? k : (size_t)-1);
    const int pdl = !pdl_ok ? zsm::kPdlNone
                    : !launched ? zsm::kPdlWaitFirst
                    : c->stage != ZERO_STAGE_3 ? zsm::kPdlEarly
                                               : zsm::kPdlEarlyLoads;
    const NvtxRange range(c->nvtx, "%s %d [%lld, %lld)", c->stage == ZERO_STAGE_3 ? "layer" : "bucket",
                          c->stage == ZERO_STAGE_3 ? c->plan.layers[layer_idx].id : (int)k, (long long)lo,
                          (long long)hi);
    st = fused_interval(c, lo, hi, grad.data(), layer_idx, launched, sc, s, o.slot(k), pdl, &state_ptr(c)->sc,
                        false, !resident);
    if (st != ZERO_OK) break;
    launched = launched || hi > lo;
    o.after_kernel(k);
    if (gathers) st = issue_gather(c, o, gfn, guser, layer_idx, k);
  }
  if (st == ZERO_OK) {
    const cudaError_t e = counted(c, zsm::launch_step_commit(state_ptr(c), s));
    if (e != cudaSuccess) st = cuda_fail(c, e, "step-commit kernel launch");
  }
  if (o.end() != cudaSuccess && st == ZERO_OK) st = cuda_fail(c, o.err, "ordering the pipeline streams");
  if (st != ZERO_OK) return st;
  c->calls = t;
  c->t = t;
  c->norm_fresh = true;
  if (stats) return finish_stats(c, o.s, stats);
  return ZERO_OK;
}

}  // namespace

extern "C" {

int32_t zero_version(void) { return ZERO_SM_VERSION; }

zero_status zero_init(const zero_layout* layout, int32_t n_ranks, int32_t stage, int64_t bucket_elems,
                      zero_ctx** out) {
  g_init_error.clear();
  if (!out) return g_init_error = "out is NULL", ZERO_EINVAL;
  *out = nullptr;
  if (!layout) return g_init_error = "layout is NULL", ZERO_EINVAL;
  if (n_ranks < 1 || n_ranks > ZERO_MAX_RANKS)
    return g_init_error = "n_ranks must be 1.." + std::to_string(ZERO_MAX_RANKS), ZERO_EINVAL;
  if (stage == ZERO_STAGE_DP) return g_init_error = "stage 0 (plain DP) is not provided on the device", ZERO_ENOTIMPL;
  if (stage < ZERO_STAGE_1 || stage > ZERO_STAGE_3) return g_init_error = "stage must be 1, 2 or 3", ZERO_EINVAL;
  zero_ctx* c = new (std::nothrow) zero_ctx();
  if (!c) return g_init_error = "out of host memory", ZERO_ENOMEM;
  std::string err;
  if (!zsm::make_plan(layout->n_tensors, layout->numel, layout->layer_id, n_ranks, bucket_elems, &c->plan, &err)) {
    delete c;
    g_init_error = err;
    return ZERO_EINVAL;
  }
  c->stage = stage;
  compute_layout(c);
  *out = c;
  return ZERO_OK;
}

zero_status zero_set_option(zero_ctx* c, int32_t key, int64_t value) {
  if (!c) return ZERO_EINVAL;
  if (key == ZERO_OPT_TIMING) {
    c->timing = value != 0;
    return ZERO_OK;
  }
  if (key == ZERO_OPT_KERNEL) {
    if (value < ZERO_KERNEL_AUTO || value > ZERO_KERNEL_BULK) return fail(c, ZERO_EINVAL, "unknown kernel %lld", (long long)value);
    c->kernel_opt = (int)value;
    return ZERO_OK;
  }
  if (key == ZERO_OPT_PDL) {
    c->pdl = value != 0;
    return ZERO_OK;
  }
  if (key == ZERO_OPT_TMA_CTAS_PER_SM) {
    if (value < 0 || value > 4) return fail(c, ZERO_EINVAL, "CTAs per SM must be 0..4");
    c->tma_ctas_opt = (int)value;
    return ZERO_OK;
  }
  if (key == ZERO_OPT_TMA_STAGES) {
    if (value < 0 || value > zsm::kTmaMaxStages) return fail(c, ZERO_EINVAL, "stages must be 0..%d", zsm::kTmaMaxStages);
    c->tma_stages_opt = (int)value;
    return ZERO_OK;
  }
  if (key == ZERO_OPT_STORE_HINT) {
    if (value < -1 || value > 1) return fail(c, ZERO_EINVAL, "store hint must be -1 (the library's choice), 0 or 1");
    c->store_hint = (int)value;
    return ZERO_OK;
  }
  if (key == ZERO_OPT_WAIT_LIMIT_NS) {
    if (value < 0 || value > 60000000000ll) return fail(c, ZERO_EINVAL, "wait limit must be 0..60e9 ns");
    c->wait_ns = (unsigned long long)value;
    return ZERO_OK;
  }
  if (key == ZERO_OPT_TMA_TILE) {
    if (value != 0 && value != 1024 && value != 2048) return fail(c, ZERO_EINVAL, "tile must be 0 (auto), 1024 or 2048");
    c->tma_tile_opt = (int)value;
    return ZERO_OK;
  }
  if (key == ZERO_OPT_TMA_WARPS) {
    if (value != 0 && value != 4 && value != 8 && value != 16)
      return fail(c, ZERO_EINVAL, "consumer warps must be 0 (auto), 4, 8 or 16");
    c->tma_warps_opt = (int)value;
    return ZERO_OK;
  }
  if (key == ZERO_OPT_TMA_GROUPS) {
    if (value < 0 || value > 3) return fail(c, ZERO_EINVAL, "consumer groups must be 0 (auto), 1, 2 or 3 (one wide group)");
    if (value > 0 && zsm::tma_stages_for(c->plan.n_ranks, (int)value) == 0)
      return fail(c, ZERO_EINVAL, "%lld consumer groups do not fit at N = %d", (long long)value, c->plan.n_ranks);
    c->tma_groups_opt = (int)value;
    return ZERO_OK;
  }
  if (key == ZERO_OPT_LAYERED) {
    c->layered = value != 0;
    return ZERO_OK;
  }
  if (key == ZERO_OPT_NVTX) {
    c->nvtx = value != 0;
    return ZERO_OK;
  }
  if (key == ZERO_OPT_GUARD) {
    if (value < 0 || value > 2) return fail(c, ZERO_EINVAL, "guard must be 0, 1 or 2");
    if (c->bound && (value != 0) != (c->guard != 0))
      return fail(c, ZERO_ESTATE, "guard bytes are laid out before zero_bind (after it only 1 <-> 2)");
    c->guard = (int)value;
    if (!c->bound) compute_layout(c);
    return ZERO_OK;
  }
  if (c->bound) return fail(c, ZERO_ESTATE, "options must be set before zero_bind");
  switch (key) {
    case ZERO_OPT_KEEP_GRAD_SHARDS:
      c->keep_grad_shards = value != 0;
      break;
    case ZERO_OPT_REPLICA_PAD:
      if (value < 0 || value % kArenaAlign || value >= (1 << 20))
        return fail(c, ZERO_EINVAL, "replica pad must be a multiple of 256 below 1 MiB");
      c->replica_pad = value;
      break;
    case ZERO_OPT_GRAD_BUFFERS:
      c->grad_buffers = value != 0;
      break;
    case ZERO_OPT_DTYPE:
      if (value != ZERO_DTYPE_BF16 && value != ZERO_DTYPE_F16) return fail(c, ZERO_EINVAL, "unknown dtype %lld", (long long)value);
      c->fmt = value == ZERO_DTYPE_F16 ? zsm::kFmtF16 : zsm::kFmtBf16;
      break;
    case ZERO_OPT_BLOCKS_PER_SM:
      if (value < 0 || value > 32) return fail(c, ZERO_EINVAL, "blocks per SM must be 0..32");
      c->blocks_per_sm_opt = (int)value;
      break;
    case ZERO_OPT_PIPELINE:
      if (value < 0 || value > 2) return fail(c, ZERO_EINVAL, "pipeline must be 0, 1 or 2");
      c->pipeline = (int)value;
      break;
    default:
      return fail(c, ZERO_EINVAL, "unknown option %d", key);
  }
  compute_layout(c);
  return ZERO_OK;
}

zero_status zero_set_pipeline_streams(zero_ctx* c, void* callback_stream, void* kernel_stream) {
  if (!c) return ZERO_EINVAL;
  if (c->pipeline_used) return fail(c, ZERO_ESTATE, "the pipeline streams are set before the first pipelined step");
  if (!callback_stream && !kernel_stream) return ZERO_OK;
  c->side = static_cast<cudaStream_t>(callback_stream);
  c->kside = static_cast<cudaStream_t>(kernel_stream);
  c->own_side = c->own_kside = false;
  return ZERO_OK;
}

zero_status zero_buffer_sizes(const zero_ctx* c, zero_sizes* out) {
  if (!c || !out) return ZERO_EINVAL;
  std::memset(out, 0, sizeof *out);
  out->psi = c->plan.psi;
  out->psi_pad = c->plan.psi_pad;
  out->shard = c->plan.shard;
  out->max_layer = c->plan.max_layer;
  out->replica_pitch = c->stage == ZERO_STAGE_3 ? c->gather_pitch : c->param_pitch;
  out->n_buckets = (int32_t)c->plan.buckets.size();
  out->n_layers = (int32_t)c->plan.layers.size();
  for (int k = 0; k < ZERO_NUM_ARENAS; ++k) out->arena_bytes[k] = c->arena_bytes[k];
  return ZERO_OK;
}

zero_status zero_tensor_offsets(const zero_ctx* c, int64_t* out, int32_t cap) {
  if (!c || (!out && cap > 0)) return ZERO_EINVAL;
  const int32_t n = (int32_t)c->plan.start.size();
  for (int32_t k = 0; k < std::min(n, cap); ++k) out[k] = c->plan.start[k];
  return cap < n ? ZERO_EINVAL : ZERO_OK;
}

zero_status zero_buckets(const zero_ctx* c, int64_t* lo_hi, int32_t cap, int32_t* n_out) {
  if (!c || !n_out || (!lo_hi && cap > 0)) return ZERO_EINVAL;
  const int32_t n = (int32_t)c->plan.buckets.size();
  for (int32_t k = 0; k < std::min(n, cap); ++k) {
    lo_hi[2 * k] = c->plan.buckets[k].lo;
    lo_hi[2 * k + 1] = c->plan.buckets[k].hi;
  }
  *n_out = n;
  return ZERO_OK;
}

zero_status zero_layers(const zero_ctx* c, int64_t* id_lo_hi, int32_t cap, int32_t* n_out) {
  if (!c || !n_out || (!id_lo_hi && cap > 0)) return ZERO_EINVAL;
  const int32_t n = (int32_t)c->plan.layers.size();
  for (int32_t k = 0; k < std::min(n, cap); ++k) {
    id_lo_hi[3 * k] = c->plan.layers[k].id;
    id_lo_hi[3 * k + 1] = c->plan.layers[k].lo;
    id_lo_hi[3 * k + 2] = c->plan.layers[k].hi;
  }
  *n_out = n;
  return ZERO_OK;
}

zero_status zero_bind(zero_ctx* c, void* const* arenas) {
  if (!c) return ZERO_EINVAL;
  if (c->bound) return fail(c, ZERO_ESTATE, "arenas are already bound");
  if (!arenas) return fail(c, ZERO_EINVAL, "arenas is NULL");
  for (int k = 0; k < ZERO_NUM_ARENAS; ++k) {
    if (c->arena_bytes[k] == 0) continue;
    if (!arenas[k]) return fail(c, ZERO_EINVAL, "arena %d (%lld bytes) is NULL", k, (long long)c->arena_bytes[k]);
    if (reinterpret_cast<uintptr_t>(arenas[k]) % kArenaAlign)
      return fail(c, ZERO_EINVAL, "arena %d is not 256-byte aligned", k);
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&c->sm_count, cudaDevAttrMultiProcessorCount, dev);
  int fused_blocks = 0, simple_blocks = 0;
  const int mode = c->stage == ZERO_STAGE_1 ? zsm::kFusedZ1 : c->stage == ZERO_STAGE_2 ? zsm::kFusedZ2 : zsm::kFusedZ3;
  if (e == cudaSuccess) e = zsm::occupancy(mode, c->plan.n_ranks, &fused_blocks, &simple_blocks);
  if (e == cudaSuccess) e = zsm::tma_configure();
  if (e == cudaSuccess) e = zsm::bulk_configure();
  if (e == cudaSuccess) e = zsm::two_pass_configure();
  if (e != cudaSuccess) return cuda_fail(c, e, "device query");
  if (c->blocks_per_sm_opt > 0) fused_blocks = std::min(fused_blocks, c->blocks_per_sm_opt);
  c->grid_fused = std::max(1, std::min(zsm::kMaxGrid, c->sm_count * std::max(1, fused_blocks)));
  c->grid_simple = std::max(1, std::min(zsm::kMaxGrid, c->sm_count * std::max(1, simple_blocks)));
  for (int k = 0; k < ZERO_NUM_ARENAS; ++k) c->arena[k] = c->arena_bytes[k] ? static_cast<char*>(arenas[k]) : nullptr;
  c->bound = true;
  return ZERO_OK;
}

zero_status zero_set_hparams(zero_ctx* c, const zero_adam_hparams* hp) {
  if (!c || !hp) return ZERO_EINVAL;
  if (!(hp->lr >= 0.0) || !(hp->beta1 >= 0.0 && hp->beta1 < 1.0) || !(hp->beta2 >= 0.0 && hp->beta2 < 1.0) ||
      !(hp->eps >= 0.0) || !(hp->weight_decay >= 0.0))
    return fail(c, ZERO_EINVAL, "hyper-parameters out of range (lr, eps, wd >= 0; 0 <= beta < 1)");
  const bool new_betas = c->have_hp && (hp->beta1 != c->hp.beta1 || hp->beta2 != c->hp.beta2);
  c->hp = *hp;
  c->have_hp = true;
  if (new_betas && c->bound && c->loaded) {
    // the bias corrections are the new betas to the power t: rebuild the
    // device powers for the current t (waits for the device)
    int64_t t = 0;
    const zero_status st = read_device_t(c, &t);
    return st != ZERO_OK ? st : write_device_t(c, t);
  }
  return ZERO_OK;
}

namespace {

// Fills the state from sources (see InitArgs) and resets the run state.
zero_status load_state(zero_ctx* c, const float* master, const float* m, const float* v, int64_t n,
                       int64_t t, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(c->arena[ZERO_ARENA_SCRATCH], 0, kScratchBytes, s);
  if (e == cudaSuccess) {
    // the step state for t completed steps and a decision of "no clipping, not
    // skipped" (pageable sources: copied before the calls return)
    const zsm::StepState st = host_state(c->hp, t);
    e = cudaMemcpyAsync(state_ptr(c), &st, sizeof st, cudaMemcpyHostToDevice, s);
    zsm::ClipDecision d;
    std::memset(&d, 0, sizeof d);
    d.coef = 1.0f;
    if (e == cudaSuccess) e = cudaMemcpyAsync(decision_ptr(c), &d, sizeof d, cudaMemcpyHostToDevice, s);
  }
  if (e != cudaSuccess) return cuda_fail(c, e, "clearing scratch");
  zsm::InitArgs a;
  std::memset(&a, 0, sizeof a);
  a.fmt = c->fmt;
  a.master_src = master;
  a.m_src = m;
  a.v_src = v;
  a.n_src_vec = n / zsm::kVec;
  a.master = master_ptr(c);
  a.m = m_ptr(c);
  a.v = v_ptr(c);
  a.n_out = c->stage == ZERO_STAGE_3 ? 1 : c->plan.n_ranks;
  for (int r = 0; r < a.n_out; ++r) a.out[r] = param_ptr(c, r);
  a.grad_shard = c->arena[ZERO_ARENA_GRAD_SHARDS] ? grad_shard_ptr(c) : nullptr;
  a.n_vec = c->plan.psi_pad / zsm::kVec;
  e = counted(c, zsm::launch_init(a, grid_for(a.n_vec, c->grid_simple), s));
  if (e != cudaSuccess) return cuda_fail(c, e, "init kernel launch");
  if (c->guard) {  // arm the guard bytes
    zsm::GuardArgs g;
    if (!guard_args(c, &g)) return fail(c, ZERO_EINVAL, "guard layout does not match the arenas");
    e = counted(c, zsm::launch_guards(g, false, s));
    if (e != cudaSuccess) return cuda_fail(c, e, "guard fill launch");
  }
  c->t = t;
  c->calls = t;
  c->loaded = true;
  c->norm_fresh = true;
  return ZERO_OK;
}

}  // namespace

zero_status zero_load_master(zero_ctx* c, const float* master_dev, void* stream) {
  if (!c) return ZERO_EINVAL;
  if (!c->bound) return fail(c, ZERO_ESTATE, "arenas are not bound (zero_bind)");
  if (master_dev && !aligned16(master_dev)) return fail(c, ZERO_EINVAL, "master_dev is not 16-byte aligned");
  return load_state(c, master_dev ? master_dev : master_ptr(c), nullptr, nullptr, c->plan.psi_pad, 0,
                    static_cast<cudaStream_t>(stream));
}

zero_status zero_import_state(zero_ctx* c, const float* master, const float* exp_avg, const float* exp_avg_sq,
                              int64_t n, int64_t t, void* stream) {
  if (!c) return ZERO_EINVAL;
  if (!c->bound) return fail(c, ZERO_ESTATE, "arenas are not bound (zero_bind)");
  if (!aligned16(master) || !aligned16(exp_avg) || !aligned16(exp_avg_sq))
    return fail(c, ZERO_EINVAL, "master, exp_avg and exp_avg_sq must be 16-byte aligned device pointers");
  const int64_t flat = c->plan.start.back() + ((c->plan.numel.back() + zsm::kGranule - 1) / zsm::kGranule) * zsm::kGranule;
  if (n % zsm::kGranule || n < flat || n > c->plan.psi_pad)
    return fail(c, ZERO_EINVAL, "n = %lld must be a multiple of 8 in [%lld, %lld] (every real element, at most psi_pad)",
                (long long)n, (long long)flat, (long long)c->plan.psi_pad);
  if (t < 0) return fail(c, ZERO_EINVAL, "t must be >= 0");
  return load_state(c, master, exp_avg, exp_avg_sq, n, t, static_cast<cudaStream_t>(stream));
}

zero_status zero_get_step(const zero_ctx* cc, int64_t* t) {
  zero_ctx* c = const_cast<zero_ctx*>(cc);
  if (!c || !t) return ZERO_EINVAL;
  if (!c->bound || !c->loaded) {
    *t = c->t;
    return ZERO_OK;
  }
  return read_device_t(c, t);
}

zero_status zero_set_step(zero_ctx* c, int64_t t) {
  if (!c || t < 0) return ZERO_EINVAL;
  if (!c->bound || !c->loaded) {
    c->t = t;
    c->calls = t;
    return ZERO_OK;
  }
  return write_device_t(c, t);
}

zero_status zero_view(const zero_ctx* cc, int32_t what, int32_t rank, void** ptr, int64_t* n_elems) {
  zero_ctx* c = const_cast<zero_ctx*>(cc);
  if (!c || !ptr || !n_elems) return ZERO_EINVAL;
  if (!c->bound) return fail(c, ZERO_ESTATE, "arenas are not bound (zero_bind)");
  const int N = c->plan.n_ranks;
  const bool slotted = what == ZERO_VIEW_GRAD_BUF || what == ZERO_VIEW_GATHER;
  const bool per_rank = slotted || (what == ZERO_VIEW_PARAM && c->stage != ZERO_STAGE_3);
  const int n_views = slotted ? N * c->slots : N;  // rank + N selects the second slot set
  if (per_rank && (rank < 0 || rank >= n_views)) return fail(c, ZERO_EINVAL, "rank %d out of range", rank);
  const int64_t P = c->plan.psi_pad;
  switch (what) {
    case ZERO_VIEW_MASTER: *ptr = master_ptr(c); *n_elems = P; break;
    case ZERO_VIEW_EXP_AVG: *ptr = m_ptr(c); *n_elems = P; break;
    case ZERO_VIEW_EXP_AVG_SQ: *ptr = v_ptr(c); *n_elems = P; break;
    case ZERO_VIEW_PARAM: *ptr = param_ptr(c, rank); *n_elems = P; break;
    case ZERO_VIEW_GRAD_SHARD:
      if (!c->arena[ZERO_ARENA_GRAD_SHARDS]) return fail(c, ZERO_EINVAL, "stage %d has no gradient shards", c->stage);
      *ptr = grad_shard_ptr(c);
      *n_elems = P;
      break;
    case ZERO_VIEW_GRAD_BUF:
      if (!c->arena[ZERO_ARENA_GRADS]) return fail(c, ZERO_EINVAL, "no gradient buffers (ZERO_OPT_GRAD_BUFFERS = 0)");
      *ptr = grad_buf_ptr(c, rank % N, rank / N);
      *n_elems = c->stage == ZERO_STAGE_1 ? P : c->stage == ZERO_STAGE_2 ? c->plan.max_bucket : c->plan.max_layer;
      break;
    case ZERO_VIEW_GATHER:
      if (c->stage != ZERO_STAGE_3) return fail(c, ZERO_EINVAL, "only stage 3 has gather buffers");
      *ptr = gather_ptr(c, rank % N, rank / N);
      *n_elems = c->plan.max_layer;
      break;
    default:
      return fail(c, ZERO_EINVAL, "unknown view %d", what);
  }
  return ZERO_OK;
}

zero_status zero_state_bytes(const zero_ctx* c, int32_t rank, int64_t out[3]) {
  if (!c || !out || rank < 0 || rank >= c->plan.n_ranks) return ZERO_EINVAL;
  const int64_t P = c->plan.psi_pad, S = c->plan.shard;
  out[0] = 2 * (c->stage == ZERO_STAGE_3 ? S : P);
  out[1] = 2 * (c->stage == ZERO_STAGE_1 ? P : S);
  out[2] = 12 * S;
  return ZERO_OK;
}

zero_status zero_comm_elems(const zero_ctx* c, int64_t out[3]) {
  if (!c || !out) return ZERO_EINVAL;
  const int64_t N = c->plan.n_ranks;
  const int64_t one = c->plan.psi_pad * (N - 1) / N;
  out[0] = c->stage == ZERO_STAGE_1 ? 2 * one : 0;
  out[1] = c->stage == ZERO_STAGE_1 ? 0 : one;
  out[2] = c->stage == ZERO_STAGE_3 ? 2 * one : one;
  return ZERO_OK;
}

zero_status zero_reduce_scatter(zero_ctx* c, int64_t lo, int64_t hi, const void* const* rank_grads, void* stream) {
  zero_status st = check_ready(c, false);
  if (st != ZERO_OK) return st;
  const NvtxRange range(c->nvtx, "reduce-scatter [%lld, %lld)", (long long)lo, (long long)hi);
  if (c->stage == ZERO_STAGE_1) return fail(c, ZERO_EINVAL, "stage 1 keeps full gradients: use zero_all_reduce");
  if (!c->arena[ZERO_ARENA_GRAD_SHARDS])
    return fail(c, ZERO_ESTATE, "gradient shards were dropped (ZERO_OPT_KEEP_GRAD_SHARDS = 0)");
  if ((st = check_interval(c, lo, hi)) != ZERO_OK) return st;
  const int N = c->plan.n_ranks;
  zsm::ReduceArgs a;
  std::memset(&a, 0, sizeof a);
  a.fmt = c->fmt;
  if (rank_grads) {
    for (int r = 0; r < N; ++r) {
      if (!rank_grads[r] || !aligned16(rank_grads[r]))
        return fail(c, ZERO_EINVAL, "rank_grads[%d] is null or not 16-byte aligned", r);
      a.grad[r] = static_cast<const uint16_t*>(rank_grads[r]);
    }
  } else if (!c->arena[ZERO_ARENA_GRADS]) {
    return fail(c, ZERO_EINVAL, "rank_grads is NULL but there are no gradient buffers");
  } else if (c->stage == ZERO_STAGE_2) {
    if (hi - lo > c->plan.max_bucket)
      return fail(c, ZERO_EINVAL, "[%lld, %lld) is larger than the bucket buffer", (long long)lo, (long long)hi);
    for (int r = 0; r < N; ++r) a.grad[r] = grad_buf_ptr(c, r);
  } else {
    const int li = c->plan.layer_of(lo);
    if (hi > c->plan.layers[li].hi) return fail(c, ZERO_EINVAL, "[%lld, %lld) crosses a layer boundary", (long long)lo, (long long)hi);
    for (int r = 0; r < N; ++r) a.grad[r] = grad_buf_ptr(c, r) + (lo - c->plan.layers[li].lo);
  }
  if (hi == lo) return ZERO_OK;
  a.shard_out = grad_shard_ptr(c) + lo;
  a.n_vec = (hi - lo) / zsm::kVec;
  a.n_ranks = N;
  a.accumulate = c->norm_fresh ? 0 : 1;
  a.write_back = 0;
  a.inv_n = (float)(1.0 / (double)N);
  a.ns = norm_scratch(c);
  cudaError_t e = launch_pass1(c, a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(c, e, "reduce-scatter kernel launch");
  c->norm_fresh = false;
  return ZERO_OK;
}

zero_status zero_all_reduce(zero_ctx* c, int64_t lo, int64_t hi, void* const* rank_grads, void* stream) {
  zero_status st = check_ready(c, false);
  if (st != ZERO_OK) return st;
  const NvtxRange range(c->nvtx, "all-reduce [%lld, %lld)", (long long)lo, (long long)hi);
  if (c->stage != ZERO_STAGE_1) return fail(c, ZERO_EINVAL, "all-reduce keeps full gradients: stage 1 only");
  if ((st = check_interval(c, lo, hi)) != ZERO_OK) return st;
  const int N = c->plan.n_ranks;
  zsm::ReduceArgs a;
  std::memset(&a, 0, sizeof a);
  a.fmt = c->fmt;
  if (!rank_grads && !c->arena[ZERO_ARENA_GRADS])
    return fail(c, ZERO_EINVAL, "rank_grads is NULL but there are no gradient buffers");
  for (int r = 0; r < N; ++r) {
    const void* p = rank_grads ? rank_grads[r] : static_cast<const void*>(grad_buf_ptr(c, r) + lo);
    if (!p || !aligned16(p)) return fail(c, ZERO_EINVAL, "rank_grads[%d] is null or not 16-byte aligned", r);
    a.grad[r] = static_cast<const uint16_t*>(p);
  }
  if (hi == lo) return ZERO_OK;
  a.shard_out = nullptr;
  a.n_vec = (hi - lo) / zsm::kVec;
  a.n_ranks = N;
  a.accumulate = c->norm_fresh ? 0 : 1;
  a.write_back = 1;
  a.inv_n = (float)(1.0 / (double)N);
  a.ns = norm_scratch(c);
  cudaError_t e = launch_pass1(c, a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(c, e, "all-reduce kernel launch");
  c->norm_fresh = false;
  return ZERO_OK;
}

}  // extern "C"

namespace {
zero_status adam_shard_launch(zero_ctx* c, int32_t rank, int64_t t, cudaStream_t s);
}  // namespace

extern "C" {

zero_status zero_adam_shard(zero_ctx* c, int32_t rank, int64_t t, void* stream) {
  zero_status st = check_ready(c, true);
  if (st != ZERO_OK) return st;
  const NvtxRange range(c->nvtx, "adam shard %d", rank);
  const int N = c->plan.n_ranks;
  if (rank < -1 || rank >= N) return fail(c, ZERO_EINVAL, "rank %d out of range", rank);
  if (t < 0) return fail(c, ZERO_EINVAL, "step t must be >= 1, or 0 for the context's counter + 1");
  if (c->stage != ZERO_STAGE_1 && !c->arena[ZERO_ARENA_GRAD_SHARDS])
    return fail(c, ZERO_ESTATE, "gradient shards were dropped (ZERO_OPT_KEEP_GRAD_SHARDS = 0)");
  if (c->stage == ZERO_STAGE_1 && !c->arena[ZERO_ARENA_GRADS])
    return fail(c, ZERO_ESTATE, "stage 1 Adam reads the gradient buffers, which were dropped");
  // t = 0: the step after the context's counter; a call for every shard
  // (rank = -1) then completes that step and advances the counter
  const bool from_counter = t == 0;
  if (from_counter) {
    int64_t done = 0;
    st = read_device_t(c, &done);
    if (st != ZERO_OK) return st;
    t = done + 1;
  }
  st = adam_shard_launch(c, rank, t, static_cast<cudaStream_t>(stream));
  if (st == ZERO_OK && from_counter && rank < 0) st = write_device_t(c, t);
  return st;
}

}  // extern "C"

namespace {

zero_status adam_shard_launch(zero_ctx* c, int32_t rank, int64_t t, cudaStream_t s) {
  const int N = c->plan.n_ranks;
  const zsm::AdamScalars sc = step_scalars(c, t, 1.0f);
  const int64_t S = c->plan.shard;
  const int r0 = rank < 0 ? 0 : rank, r1 = rank < 0 ? N : rank + 1;
  // Stage 2/3 (and stage 1 with one launch for all ranks, since every replica
  // holds the same reduced gradient): the shards are contiguous, so ranks
  // r0..r1-1 form one launch over [r0*S, r1*S).  Stage 1 per rank reads the
  // owner's own replica.
  const int64_t lo = r0 * S, hi = r1 * S;
  zsm::AdamArgs a;
  std::memset(&a, 0, sizeof a);
  a.fmt = c->fmt;
  a.sc = sc;
  a.master = master_ptr(c) + lo;
  a.m = m_ptr(c) + lo;
  a.v = v_ptr(c) + lo;
  a.n_vec = (hi - lo) / zsm::kVec;
  if (c->stage == ZERO_STAGE_3) {
    a.grad = grad_shard_ptr(c) + lo;
    a.out = param_ptr(c, 0) + lo;
  } else if (c->stage == ZERO_STAGE_2) {
    a.grad = grad_shard_ptr(c) + lo;
    if (rank >= 0) {
      a.out = param_ptr(c, rank) + lo;
    } else {
      // every rank writes its own replica's owned segment: one launch per rank
      for (int r = 0; r < N; ++r) {
        zsm::AdamArgs b = a;
        b.master = master_ptr(c) + r * S;
        b.m = m_ptr(c) + r * S;
        b.v = v_ptr(c) + r * S;
        b.grad = grad_shard_ptr(c) + r * S;
        b.out = param_ptr(c, r) + r * S;
        b.n_vec = S / zsm::kVec;
        cudaError_t e = counted(c, zsm::launch_adam(b, grid_for(b.n_vec, c->grid_simple), s));
        if (e != cudaSuccess) return cuda_fail(c, e, "adam kernel launch");
      }
      c->norm_fresh = true;
      return ZERO_OK;
    }
  } else {
    if (rank >= 0) {
      a.grad = grad_buf_ptr(c, rank) + lo;
      a.out = param_ptr(c, rank) + lo;
    } else {
      for (int r = 0; r < N; ++r) {
        zsm::AdamArgs b = a;
        b.master = master_ptr(c) + r * S;
        b.m = m_ptr(c) + r * S;
        b.v = v_ptr(c) + r * S;
        b.grad = grad_buf_ptr(c, r) + r * S;
        b.out = param_ptr(c, r) + r * S;
        b.n_vec = S / zsm::kVec;
        cudaError_t e = counted(c, zsm::launch_adam(b, grid_for(b.n_vec, c->grid_simple), s));
        if (e != cudaSuccess) return cuda_fail(c, e, "adam kernel launch");
      }
      c->norm_fresh = true;
      return ZERO_OK;
    }
  }
  if (a.n_vec > 0) {
    cudaError_t e = counted(c, zsm::launch_adam(a, grid_for(a.n_vec, c->grid_simple), s));
    if (e != cudaSuccess) return cuda_fail(c, e, "adam kernel launch");
  }
  c->norm_fresh = true;
  return ZERO_OK;
}

}  // namespace

extern "C" {

zero_status zero_all_gather(zero_ctx* c, int64_t lo, int64_t hi, void* const* rank_out, void* stream) {
  zero_status st = check_ready(c, false);
  if (st != ZERO_OK) return st;
  const NvtxRange range(c->nvtx, "all-gather [%lld, %lld)", (long long)lo, (long long)hi);
  if ((st = check_interval(c, lo, hi)) != ZERO_OK) return st;
  if (hi == lo) return ZERO_OK;
  const int N = c->plan.n_ranks;
  const int64_t S = c->plan.shard;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::vector<uint16_t*> dst(N);
  int layer_idx = 0;
  if (!rank_out && c->stage == ZERO_STAGE_3) {
    layer_idx = c->plan.layer_of(lo);
    if (hi > c->plan.layers[layer_idx].hi)
      return fail(c, ZERO_EINVAL, "[%lld, %lld) crosses a layer boundary", (long long)lo, (long long)hi);
  }
  for (int r = 0; r < N; ++r) {
    if (rank_out) {
      if (!rank_out[r] || !aligned16(rank_out[r])) return fail(c, ZERO_EINVAL, "rank_out[%d] is null or not 16-byte aligned", r);
      dst[r] = static_cast<uint16_t*>(rank_out[r]);
    } else if (c->stage == ZERO_STAGE_3) {
      dst[r] = gather_ptr(c, r) + (lo - c->plan.layers[layer_idx].lo);
    } else {
      dst[r] = param_ptr(c, r) + lo;
    }
  }
  // Each owner's piece of [lo, hi) goes out from the owner's copy.
  for (int owner = (int)(lo / S); owner < N && owner * S < hi; ++owner) {
    const int64_t a_lo = std::max(lo, owner * S), a_hi = std::min(hi, (owner + 1) * S);
    if (a_hi <= a_lo) continue;
    zsm::GatherArgs g;
    std::memset(&g, 0, sizeof g);
    g.src = (c->stage == ZERO_STAGE_3 ? param_ptr(c, 0) : param_ptr(c, owner)) + a_lo;
    g.n_out = 0;
    for (int r = 0; r < N; ++r) {
      // the owner's own replica already holds the source (stage 1, 2)
      if (!rank_out && c->stage != ZERO_STAGE_3 && r == owner) continue;
      g.out[g.n_out++] = dst[r] + (a_lo - lo);
    }
    g.n_vec = (a_hi - a_lo) / zsm::kVec;
    if (g.n_out == 0) continue;
    cudaError_t e = counted(c, zsm::launch_gather(g, grid_for(g.n_vec, c->grid_simple), s));
    if (e != cudaSuccess) return cuda_fail(c, e, "all-gather kernel launch");
  }
  return ZERO_OK;
}

zero_status zero_step(zero_ctx* c, zero_grad_fn grad_fn, void* grad_user, zero_gather_fn gather_fn,
                      void* gather_user, void* stream, zero_step_stats* stats) {
  if (!c) return ZERO_EINVAL;
  const zero_status st = run_step(c, grad_fn, grad_user, nullptr, gather_fn, gather_user, stream, stats);
  int64_t g[3];
  return st == ZERO_OK && c->guard == 2 ? check_guards(c, static_cast<cudaStream_t>(stream), g) : st;
}

zero_status zero_step_resident(zero_ctx* c, const void* const* rank_grads, zero_gather_fn gather_fn,
                               void* gather_user, void* stream, zero_step_stats* stats) {
  if (!c) return ZERO_EINVAL;
  if (!rank_grads) return fail(c, ZERO_EINVAL, "rank_grads is NULL");
  const zero_status st = run_step(c, nullptr, nullptr, rank_grads, gather_fn, gather_user, stream, stats);
  int64_t g[3];
  return st == ZERO_OK && c->guard == 2 ? check_guards(c, static_cast<cudaStream_t>(stream), g) : st;
}

zero_status zero_check_guards(zero_ctx* c, void* stream, int64_t out[3]) {
  if (!c) return ZERO_EINVAL;
  int64_t local[3];
  if (!out) out = local;
  out[0] = 0;
  out[1] = out[2] = -1;
  if (!c->guard) return fail(c, ZERO_ESTATE, "the arenas have no guard bytes (ZERO_OPT_GUARD before zero_bind)");
  if (!c->bound || !c->loaded)
    return fail(c, ZERO_ESTATE, "the guard bytes are armed by zero_load_master / zero_import_state");
  return check_guards(c, static_cast<cudaStream_t>(stream), out);
}

zero_status zero_kernel_timing(zero_ctx* c, double* ms, int64_t* launches, double* model_bytes) {
  if (!c || !ms || !launches || !model_bytes) return ZERO_EINVAL;
  double total = 0.0;
  if (c->timed > 0) {
    cudaError_t e = cudaEventSynchronize(c->events[2 * c->timed - 1]);
    if (e != cudaSuccess) return cuda_fail(c, e, "waiting for timed launches");
    for (size_t k = 0; k < c->timed; ++k) {
      float one = 0.f;
      e = cudaEventElapsedTime(&one, c->events[2 * k], c->events[2 * k + 1]);
      if (e != cudaSuccess) return cuda_fail(c, e, "reading launch time");
      total += one;
    }
  }
  *ms = total;
  *launches = (int64_t)c->timed;
  *model_bytes = c->timed_bytes;
  c->timed = 0;
  c->timed_bytes = 0.0;
  if (c->bound) {
    unsigned int err = 0;
    cudaError_t e = cudaMemcpy(&err, norm_scratch(c).error, sizeof err, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(c, e, "reading the device error word");
    return check_device_error(c, err, nullptr);
  }
  return ZERO_OK;
}

zero_status zero_set_loss_scale(zero_ctx* c, double scale) {
  if (!c) return ZERO_EINVAL;
  if (!(scale > 0.0) || std::isinf(scale)) return fail(c, ZERO_EINVAL, "the loss scale must be finite and > 0");
  c->loss_scale = scale;
  return ZERO_OK;
}

zero_status zero_set_clip(zero_ctx* c, double max_norm, int32_t skip_nonfinite) {
  if (!c) return ZERO_EINVAL;
  if (!(max_norm >= 0.0) || std::isinf(max_norm)) return fail(c, ZERO_EINVAL, "max_norm must be finite and >= 0");
  c->clip_norm = max_norm;
  c->skip_nonfinite = skip_nonfinite != 0;
  return ZERO_OK;
}

zero_status zero_fused_config(const zero_ctx* c, int32_t* kernel, int32_t* groups, int32_t* stages) {
  if (!c || !kernel || !groups || !stages) return ZERO_EINVAL;
  if (use_bulk(c)) {
    *kernel = ZERO_KERNEL_BULK;
    *groups = bulk_warps(c);
    *stages = bulk_stages(c);
  } else if (use_chunked(c)) {
    *kernel = ZERO_KERNEL_TMA;
    *groups = 1;
    *stages = chunked_stages(c);
  } else if (use_tma(c)) {
    *kernel = ZERO_KERNEL_TMA;
    *groups = tma_groups(c);
    *stages = zsm::tma_stages_for(c->plan.n_ranks, *groups, tma_stages(c));
  } else {
    *kernel = ZERO_KERNEL_REGISTER;
    *groups = 0;
    *stages = 0;
  }
  return ZERO_OK;
}

zero_status zero_fused_tile(const zero_ctx* c, int32_t* tile) {
  if (!c || !tile) return ZERO_EINVAL;
  *tile = use_bulk(c) ? bulk_tile(c) : use_tma(c) ? (int32_t)kTmaTile : 0;
  return ZERO_OK;
}

zero_status zero_probe_pattern(zero_ctx* c, const void* const* rank_grads, void* stream) {
  zero_status st = check_ready(c, false);
  if (st != ZERO_OK) return st;
  if (!rank_grads) return fail(c, ZERO_EINVAL, "rank_grads is NULL");
  const int N = c->plan.n_ranks;
  for (int r = 0; r < N; ++r)
    if (!rank_grads[r] || !aligned16(rank_grads[r]))
      return fail(c, ZERO_EINVAL, "rank_grads[%d] is null or not 16-byte aligned", r);
  if (!bulk_fits(c))
    return fail(c, ZERO_ENOTIMPL, "the movement-only pass exists for the bulk-store kernel's built configurations");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const std::vector<zsm::Span> iv = step_intervals(c);
  std::vector<uint16_t*> grad(N);
  const int n_layers = (int)c->plan.layers.size();
  const bool pdl_ok = c->pdl && c->tma_ctas_opt <= 1;
  if (layered_ok(c, false, iv)) {  // the step's own form: every layer in one launch
    interval_grads(c, rank_grads, 0, 0, grad.data());
    bool refused = false;
    st = fused_layered(c, iv, grad.data(), s, nullptr, true, &refused);
    if (st != ZERO_OK) return st;
    if (!refused) {
      c->norm_fresh = true;
      return ZERO_OK;
    }
  }
  bool launched = false;
  for (size_t k = 0; k < iv.size(); ++k) {
    const int64_t lo = iv[k].lo, hi = iv[k].hi;
    const int layer_idx = c->stage == ZERO_STAGE_3 ? n_layers - 1 - (int)k : 0;
    interval_grads(c, rank_grads, lo, 0, grad.data());
    const int pdl = !pdl_ok ? zsm::kPdlNone
                    : !launched ? zsm::kPdlWaitFirst
                    : c->stage != ZERO_STAGE_3 ? zsm::kPdlEarly
                                               : zsm::kPdlEarlyLoads;
    st = fused_interval(c, lo, hi, grad.data(), layer_idx, launched, zsm::AdamScalars{}, s, 0, pdl, nullptr, true);
    if (st != ZERO_OK) return st;
    launched = launched || hi > lo;
  }
  c->norm_fresh = true;
  return ZERO_OK;
}

zero_status zero_launch_count(const zero_ctx* c, int64_t* n) {
  if (!c || !n) return ZERO_EINVAL;
  *n = c->launched;
  return ZERO_OK;
}

zero_status zero_read_stats(zero_ctx* c, void* stream, zero_step_stats* out) {
  if (!c || !out) return ZERO_EINVAL;
  if (!c->bound || !c->loaded) return fail(c, ZERO_ESTATE, "nothing to read: not bound or not initialised");
  return finish_stats(c, static_cast<cudaStream_t>(stream), out);
}

const char* zero_last_error(const zero_ctx* c) { return c ? c->err.c_str() : g_init_error.c_str(); }

void zero_destroy(zero_ctx* c) { delete c; }

}  // extern "C"
