// Device kernels of the ZeRO optimizer step and their launch arguments.
//
// All kernels are memory-bound streams over 16-byte vectors of 8 bf16 (or two
// float4 of fp32) elements: one lane owns 8 consecutive flat elements per
// iteration of a grid-stride loop sized to the SM count.  Nothing here is a
// contraction, so no tensor core is involved.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace zsm {

constexpr int kMaxRanks = 128;   // mirrors ZERO_MAX_RANKS
constexpr int kVec = 8;          // bf16 elements per 16-byte vector
constexpr int kThreads = 256;    // threads per CTA for every kernel
constexpr int kMaxGrid = 4096;   // upper bound on CTAs of a norm-reducing launch
constexpr int kTmaMaxRanks = 16; // the shared-memory staged kernel handles N <= 16
constexpr int kTmaMaxSmem = 227 * 1024 - 1024;  // dynamic smem cap (1 KB left for static)
constexpr int kTmaMaxStages = 8;                // ring depth limit of the staged kernel
constexpr int kTmaDefaultStages = 4;            // ring depth when the caller does not choose
constexpr int kWideGroup = 3;  // "groups" value that selects one group of 16 consumer warps

// Binary32 scalars of one Adam step, each rounded once from binary64 on the host,
// and the gradient factors applied before the update (flags say which).
enum AdamFlags { kUnscale = 1, kClip = 2 };
struct AdamScalars {
  float b1, b2, omb1, omb2, bc1, bc2, decay, lr, eps;
  float inv_scale;  // fp32(1 / loss scale), applied when flags & kUnscale
  float coef;       // clipping coefficient, applied when flags & kClip
  int flags;
};

enum StorageFormat { kFmtBf16 = 0, kFmtF16 = 1 };

// Programmatic dependent launch of a fused-step kernel.  With kPdlWaitFirst
// or kPdlEarly the launch carries the programmatic-serialization attribute,
// so it may start while the grid before it in the stream is still running;
// each CTA of a fused kernel releases its dependents (griddepcontrol
// .launch_dependents) once it has no more input loads to issue.
//   kPdlWaitFirst  the kernel waits for the grid before it (griddepcontrol
//                  .wait) before touching global memory: safe after anything;
//   kPdlEarly      the kernel streams its interval at once and waits only
//                  before the norm epilogue.  Only for a launch whose
//                  predecessor is a fused kernel of the same step on a
//                  disjoint interval with disjoint destinations, so that the
//                  two share nothing but the norm scratch.
//   kPdlEarlyLoads the kernel loads and computes at once but each thread
//                  waits before its first store (and before the epilogue):
//                  for a predecessor on a disjoint interval that writes the
//                  same destination buffer (stage 3's temporary layer buffer).
enum PdlMode { kPdlNone = 0, kPdlWaitFirst = 1, kPdlEarly = 2, kPdlEarlyLoads = 3 };

// cudaLaunchKernelEx with the programmatic-serialization attribute when `pdl`.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), int grid, int block, size_t smem, cudaStream_t s, bool pdl,
                          Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// Gradient-norm / non-finite accumulation in the scratch arena.
struct NormScratch {
  double* partial_sq;              // [kMaxGrid] per-CTA partial sums of g^2
  unsigned long long* partial_nf;  // [kMaxGrid] per-CTA non-finite counts
  unsigned int* done;              // CTAs of the current launch that finished
  double* step_sq;                 // sum over the launches of the current step
  unsigned long long* step_nf;
  unsigned int* error;             // non-zero after a bounded device wait ran out
  unsigned long long wait_ns;      // limit of a staged kernel's ring waits (0: one non-blocking test)
};

// Fused reduce + Adam + broadcast over one interval [lo, hi) of the flat space.
// Every pointer is already offset to flat element lo of its buffer.
struct FusedArgs {
  int fmt;                          // StorageFormat of every 16-bit buffer
  const uint16_t* grad[kMaxRanks];  // rank r's bf16 gradient (stage 1: written back)
  uint16_t* out[kMaxRanks];         // rank r's bf16 parameter destination
  float* master;
  float* m;
  float* v;
  uint16_t* grad_shard;             // reduced bf16 gradient, or nullptr
  uint16_t* param_shard;            // stage 3 bf16 parameter shard, or nullptr
  int64_t n_vec;                    // (hi - lo) / 8
  int n_ranks;
  int accumulate;                   // 0: first launch of the step (norm overwrites)
  float inv_n;                      // binary32 1/N
  int pdl;                          // PdlMode of this launch
  int store_hint;                   // bulk-store kernel: 1 = its stores carry an L2 evict-first hint
  AdamScalars sc;
  const AdamScalars* sc_dev;        // when set, the scalars are read here instead (StepState::sc)
  NormScratch ns;
};

// Reduce only (reduce-scatter to a shard, or all-reduce written back).
struct ReduceArgs {
  int fmt;                          // StorageFormat of every 16-bit buffer
  const uint16_t* grad[kMaxRanks];
  uint16_t* shard_out;              // reduce-scatter destination, or nullptr
  int64_t n_vec;
  int n_ranks;
  int accumulate;
  int write_back;                   // all-reduce: write the mean to every grad[r]
  float inv_n;
  NormScratch ns;
};

struct AdamArgs {
  int fmt;                          // StorageFormat of every 16-bit buffer
  const uint16_t* grad;
  float* master;
  float* m;
  float* v;
  uint16_t* out;
  int64_t n_vec;
  AdamScalars sc;
};

// Adam + broadcast from an already reduced gradient (second pass of a clipped
// or overflow-checked step).  The gradient of flat element i comes from
// gsrc[i / shard] + i (the owner's copy); every pointer but gsrc is at flat
// element `lo`.
// The clipped step's decision, taken on the device between the two passes
// from the step's gradient sums: norm = sqrt(sum of squares) / loss scale,
// skip when the overflow skip is on and a value is not finite, and the
// clipping coefficient fp32(max_norm / (norm + 1e-6)) (binary64 quotient),
// applied when below 1 -- the host's formula, the same binary64 operations.
struct ClipDecision {
  double norm;
  unsigned long long nonfinite;
  float coef;    // 1 when no clipping applies
  int skip;
};

struct ClipParams {
  double max_norm;     // 0: no clipping
  double loss_scale;
  int skip_nonfinite;
};

// The optimizer's step state on the device: t and beta1^t, beta2^t as t
// successive binary64 products (the host's definition of the bias-correction
// powers, so the same bits), and the binary32 scalars of the step being run.
// A step's first kernel forms the scalars for t + 1; the update kernels read
// them here, so a step enqueues nothing but kernels and can be captured in a
// CUDA graph and replayed.
struct StepState {
  long long t;        // completed steps
  double p1, p2;      // beta1^t, beta2^t
  long long t_next;   // the step being run (committed when it completes unskipped)
  double p1_next, p2_next;
  AdamScalars sc;     // its scalars
};

// Hyper-parameters as the user gave them (binary64) and the loss scale.
struct StepHparams {
  double lr, beta1, beta2, eps, weight_decay, loss_scale;
};

struct AdamBcastArgs {
  int fmt;                          // StorageFormat of every 16-bit buffer
  const uint16_t* gsrc[kMaxRanks];
  uint16_t* out[kMaxRanks];
  float* master;
  float* m;
  float* v;
  uint16_t* param_shard;            // stage 3 bf16 parameter shard, or nullptr
  int64_t lo;
  int64_t shard;
  int64_t n_vec;
  int n_out;
  AdamScalars sc;                   // including the unscale factor
  const AdamScalars* sc_dev;        // when set, the scalars are read here instead (StepState::sc)
  const ClipDecision* dec;          // the step's decision (clip coefficient, skip), or nullptr
  unsigned int* error;              // staged kernel: set when a bounded wait runs out
  unsigned long long wait_ns;       // staged kernel: limit of its ring waits (0: one non-blocking test)
};

struct GatherArgs {
  const uint16_t* src;
  uint16_t* out[kMaxRanks];
  int64_t n_vec;
  int n_out;
};

struct InitArgs {
  int fmt;                          // StorageFormat of every 16-bit buffer
  const float* master_src;          // elements [0, n_src_vec*8) come from these sources,
  const float* m_src;               // m and v are 0 where their source is nullptr,
  const float* v_src;               // everything beyond the sources is 0
  int64_t n_src_vec;
  float* master;
  float* m;
  float* v;
  uint16_t* out[kMaxRanks];         // bf16(master) destinations, each at element 0
  int n_out;
  uint16_t* grad_shard;             // zeroed when not null
  int64_t n_vec;
};

enum FusedMode { kFusedZ1 = 1, kFusedZ2 = 2, kFusedZ3 = 3 };
enum FusedKernel { kKernelAuto = 0, kKernelRegister = 1, kKernelTma = 2, kKernelBulk = 3 };

// Launchers (return the launch's cudaError_t).
cudaError_t launch_fused(int mode, const FusedArgs& a, int grid, cudaStream_t s);
cudaError_t launch_reduce(const ReduceArgs& a, int grid, cudaStream_t s);
cudaError_t launch_adam(const AdamArgs& a, int grid, cudaStream_t s);
cudaError_t launch_gather(const GatherArgs& a, int grid, cudaStream_t s);
cudaError_t launch_adam_bcast(const AdamBcastArgs& a, int grid, cudaStream_t s);
// The clipped step's decision; commits the step state's t_next when the step
// is not skipped.
cudaError_t launch_clip_decide(const NormScratch& ns, const ClipParams& p, ClipDecision* out, StepState* state,
                               cudaStream_t s);
// A step's first kernel: the scalars of step t + 1 into state->sc (t and the
// powers advance when the step completes: step_commit, or the clipped step's
// decision); `dec`, when given, is reset to "no clipping, not skipped".
cudaError_t launch_step_begin(StepState* state, const StepHparams& hp, ClipDecision* dec, cudaStream_t s);
cudaError_t launch_step_commit(StepState* state, cudaStream_t s);
cudaError_t launch_init(const InitArgs& a, int grid, cudaStream_t s);

// Shared-memory staged fused kernel (fused_tma.cu): one CTA per SM with
// `groups` (1 or 2) producer/consumer groups.
cudaError_t launch_fused_tma(int mode, const FusedArgs& a, int grid, int groups, int max_stages,
                             cudaStream_t s);
// Ring depth for N and `groups` (max_stages 0 = the default depth), 0 when out of range.
int tma_stages_for(int n_ranks, int groups, int max_stages = 0);
// Rank-chunked staged kernel (fused_tma.cu) for any N, meant for N > 16: the
// replicas stream in chunks of 8 ranks through a `cstages`-deep ring.
cudaError_t launch_fused_chunked(int mode, const FusedArgs& a, int grid, int cstages, cudaStream_t s);

// A stage-3 step's layers as one launch of the bulk-store kernel
// (launch_fused_bulk_layered): segment k is one layer's flat range
// [lo[k], lo[k] + len[k]), in the schedule's order, whose parameters go to
// the temporary layer buffers from their start.  `counter` (zero before the
// launch) counts the storers' arrivals: one per CTA for each segment whose
// stores it has finished.
constexpr int kMaxSegments = 64;
struct SegTable {
  int n;
  unsigned* counter;
  long long lo[kMaxSegments];
  long long len[kMaxSegments];
};

// Staged kernel with bulk stores (fused_bulk.cu): tiles of `tile` elements,
// `warps` consumer warps, a ring of at most `max_stages` stages (0 = the
// default depth); above N = 16 the rank-chunked form (max_stages bounds its
// chunk ring).  One CTA per SM.  `move` launches the movement-only twin (same
// copies, no arithmetic; `opaque` must be 0), which measures the pattern's
// ceiling and is never part of a step.
cudaError_t launch_fused_bulk(int mode, const FusedArgs& a, int grid, int tile, int warps, int max_stages, bool move,
                              uint32_t opaque, cudaStream_t s);
// Stage 3, N <= 16: every segment of `g` in one cooperative launch of that
// kernel (`a`'s pointers at flat element 0, its layer-buffer pointers at the
// buffers' start, no programmatic launch).  Each CTA walks its tiles layer
// after layer with its ring running on across the boundaries; its storer
// issues a layer's stores only after every CTA has finished storing the
// layers before (g.counter).
cudaError_t launch_fused_bulk_layered(const FusedArgs& a, const SegTable& g, int grid, int tile, int warps,
                                      int max_stages, bool move, cudaStream_t s);
// Ring depth of that kernel for N, the tile and whether the averaged gradient
// is stored (the chunk ring above N = 16; 0 when nothing fits); whether
// (tile, warps) is a built configuration at that N.
int bulk_stages_for(int n_ranks, int tile, bool need_g, int max_stages);
bool bulk_config_valid(int n_ranks, int tile, int warps);
cudaError_t bulk_configure();  // opt in to the large dynamic smem (current device)

// Resident CTAs per SM of the staged kernel in that configuration (0 on error).
int tma_ctas_per_sm(int n_ranks, int groups, int max_stages);
cudaError_t tma_configure();       // opt in to the large dynamic smem (current device)

// Resident CTAs per SM of the fused kernel for `mode` and of the simple kernels.
cudaError_t occupancy(int mode, int n_ranks, int* fused_blocks, int* simple_blocks);

// The two passes of the clipped / overflow-checked step, staged through
// shared memory (two_pass_tma.cu; the reduce streams the ranks in chunks of 8
// above 16 ranks).  `uniform`: every gsrc[r] is the same array (the
// reduced-gradient shards), so one copy per tile suffices.
cudaError_t two_pass_configure();
cudaError_t launch_reduce_tma(const ReduceArgs& a, int grid, cudaStream_t s);
cudaError_t launch_adam_bcast_tma(const AdamBcastArgs& a, int grid, bool uniform, cudaStream_t s);
int64_t two_pass_tile();

}  // namespace zsm
