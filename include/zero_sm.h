/*
 * zero_sm.h -- C ABI of the B200 (sm_100a) ZeRO optimizer-step library.
 *
 * The library runs the data-parallel optimizer step of ZeRO (Zero Redundancy
 * Optimizer) over N logical data-parallel ranks whose buffers all live in one
 * GPU's HBM: it reduces the N ranks' bf16 gradient replicas (fp32 sum in rank
 * order 0..N-1, then the 1/N mean), runs mixed-precision Adam on each rank's
 * owned shard (fp32 master weight, m and v, bias-corrected, decoupled weight
 * decay) and all-gathers the updated bf16 parameters back to the ranks.
 *
 * Sources (three web pages on ZeRO; cited by title and section):
 *   [T] "ZERO训练技术" (wqh011128.github.io)
 *   [M] "ZeRO：从优化器状态到残差状态的显存优化" (xuesongtap.github.io)
 *   [Q] mstx.cn post 475, a ZeRO interview write-up
 *
 * Conventions for every entry point
 *   - Returns a zero_status; ZERO_OK (0) on success.  No exception, signal,
 *     device trap or assert crosses this boundary.  On failure the context
 *     (when there is one) keeps a message readable through zero_last_error().
 *   - The library never allocates device memory.  The caller sizes the arenas
 *     with zero_buffer_sizes(), allocates them (any allocator; 256-byte
 *     aligned) and lends them with zero_bind() until zero_destroy().  This is
 *     the pre-allocated contiguous pool of [M] section 3.4 ("MD"): buffer
 *     lifetimes are managed inside caller-owned memory, never by the system
 *     allocator during a step.
 *   - "stream" is a cudaStream_t passed as void*; NULL is the legacy default
 *     stream.  All device work of a call is enqueued on it, asynchronously.
 *     Launch errors are reported as ZERO_ECUDA by the call that launched;
 *     asynchronous device faults surface as ZERO_ECUDA from the next call that
 *     synchronises (zero_read_stats, or zero_step with a stats pointer).
 *   - Element indices refer to the padded flat parameter space [0, psi_pad):
 *     tensors laid end to end in list order, each starting on a multiple of
 *     8 elements, the total padded to a multiple of 8*N.  Rank r owns the
 *     contiguous shard [r*S, (r+1)*S), S = psi_pad / N ([T] section "ZeRO-1",
 *     part on how optimizer states are split).  Interval bounds lo, hi passed
 *     to the library must be multiples of 8 with 0 <= lo <= hi <= psi_pad.
 *   - bf16 data travels as raw 16-bit patterns (uint16_t); pad elements of
 *     every gradient input must be 0.
 *   - The calls that take a context are not thread-safe on the same context.
 */
#ifndef ZERO_SM_H
#define ZERO_SM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ZERO_SM_VERSION 3
#define ZERO_MAX_RANKS 128

typedef enum zero_status {
  ZERO_OK = 0,
  ZERO_EINVAL = 1,   /* a bad argument: null, misaligned, out of range, wrong stage */
  ZERO_ENOMEM = 2,   /* an arena the caller sized is too small for this context */
  ZERO_ECUDA = 3,    /* a CUDA runtime error (launch or asynchronous fault) */
  ZERO_ESTATE = 4,   /* call out of order: arenas not bound, hyper-parameters unset */
  ZERO_ENOTIMPL = 5, /* a combination the library does not provide */
  ZERO_EGUARD = 6    /* a guard byte of an arena changed (ZERO_OPT_GUARD, zero_check_guards) */
} zero_status;

/* ZeRO stages ([T] section "一张总对比表"; [Q] section 一). */
enum {
  ZERO_STAGE_DP = 0, /* plain data parallel: every rank holds everything */
  ZERO_STAGE_1 = 1,  /* optimizer states sharded */
  ZERO_STAGE_2 = 2,  /* + gradients sharded (bucketed reduce-scatter) */
  ZERO_STAGE_3 = 3   /* + parameters sharded (per-layer gather into a temporary) */
};

/* The parameter list: n_tensors sizes in flat order, each tagged with a layer
 * id; layer ids must be non-decreasing (a layer is a contiguous run). */
typedef struct zero_layout {
  int32_t n_tensors;
  const int64_t* numel;     /* host array, n_tensors entries, each >= 0 */
  const int32_t* layer_id;  /* host array, n_tensors entries, non-decreasing */
} zero_layout;

/* Adam hyper-parameters as the user writes them (binary64).  Each scalar the
 * device uses (beta1, beta2, 1-beta1, 1-beta2, 1-beta^t, 1-lr*wd, lr, eps) is
 * derived in binary64 and rounded once to binary32. */
typedef struct zero_adam_hparams {
  double lr, beta1, beta2, eps, weight_decay;
} zero_adam_hparams;

/* Arenas the caller allocates and lends (zero_bind).  Unused arenas have
 * size 0 and may be NULL. */
enum {
  ZERO_ARENA_STATES = 0,      /* fp32 master, m, v: 3 x psi_pad x 4 B */
  ZERO_ARENA_PARAMS = 1,      /* bf16 params: N replicas of psi_pad (stage 1, 2) or the
                                 psi_pad owned shards, rank order (stage 3) */
  ZERO_ARENA_GRADS = 2,       /* bf16 gradient inputs: N full replicas (stage 1), N buckets
                                 of bucket_elems (stage 2, the fixed buffer "CB" of [M]
                                 section 3.3), N slots of the largest layer (stage 3) */
  ZERO_ARENA_GRAD_SHARDS = 3, /* bf16 reduced gradient shards, psi_pad (stage 2, 3, unless
                                 ZERO_OPT_KEEP_GRAD_SHARDS is 0) */
  ZERO_ARENA_GATHER = 4,      /* stage 3: N temporary full-layer buffers (largest layer) */
  ZERO_ARENA_SCRATCH = 5,     /* norm partials, counters and stats (small) */
  ZERO_NUM_ARENAS = 6
};

typedef struct zero_sizes {
  int64_t psi;            /* real parameter count */
  int64_t psi_pad;        /* padded flat length */
  int64_t shard;          /* S = psi_pad / N */
  int64_t max_layer;      /* largest layer span (elements, padded) */
  int64_t replica_pitch;  /* bytes between consecutive rank buffers in PARAMS/GRADS/GATHER */
  int32_t n_buckets;      /* intervals of the bucket schedule */
  int32_t n_layers;
  int64_t arena_bytes[ZERO_NUM_ARENAS];
} zero_sizes;

typedef struct zero_step_stats {
  double grad_norm;        /* sqrt(sum of squares of the averaged bf16 gradient), fp64 */
  int64_t nonfinite;       /* averaged gradient elements that are Inf or NaN */
  int64_t step;            /* the step counter after the step (unchanged by a skipped step) */
  int64_t comm_elems[3];   /* logical elements each rank sends per step: all-reduce,
                              reduce-scatter, all-gather (ring convention) */
  double clip_coef;        /* gradient scale the update used (1 = none; zero_set_clip) */
  int64_t skipped;         /* 1 when the step was skipped for non-finite gradients */
} zero_step_stats;

/* Options (zero_set_option): before zero_bind unless an entry says otherwise. */
enum {
  ZERO_OPT_KEEP_GRAD_SHARDS = 1, /* stage 2/3: 1 (default) keeps the reduced bf16 gradient
                                    shards (GRAD_SHARDS arena; the fused step stores them and
                                    the unfused reduce-scatter/Adam calls use them); 0 drops
                                    that arena: the fused step keeps the reduced gradient in
                                    registers only and zero_reduce_scatter/zero_adam_shard
                                    return ZERO_ESTATE */
  ZERO_OPT_REPLICA_PAD = 2,      /* extra bytes (multiple of 256, < 1 MiB) between consecutive
                                    buffers of an arena (rank replicas, master/m/v), to keep
                                    streams that are read together off the same DRAM banks when
                                    the buffers' lengths are large powers of two; default 0 */
  ZERO_OPT_BLOCKS_PER_SM = 3,    /* fused-kernel CTAs per SM (0 = occupancy maximum) */
  ZERO_OPT_TIMING = 4,           /* 1: record a CUDA event pair on the launching stream around
                                    every launch of the step's kernels -- the fused kernel, or
                                    the two passes of a clipped step -- (read with
                                    zero_kernel_timing); may be set at any time; default 0 */
  ZERO_OPT_KERNEL = 5,           /* fused-step kernel: ZERO_KERNEL_AUTO (default),
                                    ZERO_KERNEL_REGISTER, ZERO_KERNEL_TMA or ZERO_KERNEL_BULK;
                                    may be set at any time */
  ZERO_OPT_GRAD_BUFFERS = 6,     /* 1 (default) sizes the GRADS arena; 0 drops it for callers
                                    that only use zero_step_resident and the calls given explicit
                                    pointers (zero_step then returns ZERO_ESTATE) */
  ZERO_OPT_TMA_GROUPS = 7,       /* staged kernel: producer/consumer groups per CTA, 1 or 2,
                                    or 3 = one group of 16 consumer warps of 4 elements each
                                    (0 = the library's choice); may be set at any time */
  ZERO_OPT_TMA_STAGES = 8,       /* staged kernel: shared-memory ring depth, at most 8 and at
                                    most what fits in 227 KB (0 = the library's choice); may be
                                    set at any time */
  ZERO_OPT_TMA_CTAS_PER_SM = 9,  /* staged kernel: CTAs per SM, 1..4, capped by what fits in
                                    shared memory (0 = the library's choice); any time */
  ZERO_OPT_DTYPE = 10,           /* storage format of every 16-bit buffer (gradients,
                                    parameters, reduced shards): ZERO_DTYPE_BF16 (default) or
                                    ZERO_DTYPE_F16 (IEEE binary16); before zero_bind */
  ZERO_OPT_PIPELINE = 11,        /* 1: zero_step / zero_step_resident run grad_fn and
                                    gather_fn on a stream of the context's own, one interval
                                    ahead of the kernels on the caller's stream, so that the
                                    caller's backward of the next interval and its use of the
                                    last gathered layer overlap the step's kernel -- the
                                    overlap and prefetch that ZeRO-3's layer-by-layer gathers
                                    and reduce-scatters depend on ([T] section "ZeRO-3", part
                                    on its communication volume; [Q] section 五).  Stages 2 and
                                    3 then hold two gradient slot sets (GRADS doubles) and
                                    stage 3 two gather slot sets (GATHER doubles), used
                                    alternately; stage 1 needs none.  2: as 1, and the step's
                                    kernels run on a stream of the context's own at the
                                    device's greatest priority (joined into the caller's stream
                                    at the end), so that their CTAs take the SMs that the
                                    callbacks' work frees first.  Values are unchanged.
                                    Default 0; before zero_bind */
  ZERO_OPT_TMA_TILE = 13,        /* bulk-store kernel: elements per tile, 1024 or 2048 (0 = the
                                    library's choice); may be set at any time */
  ZERO_OPT_TMA_WARPS = 14,       /* bulk-store kernel: consumer warps, 4, 8 or 16 (8, 4 or 2
                                    elements per lane; 0 = the library's choice); the built
                                    (tile, warps) pairs are 2048 x 8, 2048 x 16, 1024 x 4,
                                    1024 x 8 and 1024 x 16 for N <= 16, 2048 x 8 and 1024 x 8
                                    above; another pair makes the next fused launch fail with
                                    ZERO_ECUDA; may be set at any time */
  ZERO_OPT_STORE_HINT = 16,      /* bulk-store kernel: 1 marks its bulk stores L2 evict-first
                                    (written lines leave L2 first), 0 plain, -1 (default) the
                                    library's measured choice for N and the stage (on at stages
                                    2 and 3, where it gained up to 4 % on B200); values are
                                    unchanged either way; may be set at any time */
  ZERO_OPT_WAIT_LIMIT_NS = 15,   /* limit, in ns of wall time, of each wait of the staged
                                    kernels on their shared-memory ring (default 2e9, at most
                                    60e9).  0 makes every ring wait one non-blocking test: a
                                    wait whose copies have not already landed runs out at once,
                                    so the kernel takes its failure path (error word, drain of
                                    the copies in flight -- those waits keep 2 s -- and a
                                    ZERO_ECUDA from the next synchronising call) without
                                    anything stalling; it exists to test that path.  The
                                    parameters and states of a step that ran out are partly
                                    updated: restore them (zero_import_state) before going on.
                                    May be set at any time */
  ZERO_OPT_LAYERED = 19,         /* 1 (default): a stage-3 step without callbacks
                                    (zero_step_resident with no gather_fn) on the bulk-store
                                    kernel at N <= 16, with 2..64 non-empty layers, runs as
                                    one cooperative launch.  Its CTAs take the layers in the
                                    schedule's order (last to first), their shared-memory
                                    rings running on across the layer boundaries.  A layer's
                                    stores into the temporary layer buffers go out only after
                                    every CTA has finished storing the layers before it -- the
                                    order of one launch per layer, without a launch boundary at
                                    each layer.  The gradient norm is summed over the whole
                                    step at once (the same value up to rounding order, the same
                                    bits run to run).  The same holds for the update pass of a
                                    clipped stage-3 step without gather_fn (zero_set_clip),
                                    on the bulk-store kernel at any N.  Where the device cannot
                                    hold every CTA at once (a cooperative launch refused), the
                                    step runs one launch per layer instead.  0: one launch per
                                    layer.  The movement-
                                    only pass (zero_probe_pattern) follows the same choice.
                                    May be set at any time */
  ZERO_OPT_NVTX = 18,            /* 1: NVTX ranges on the domain "zero_sm" around the host side
                                    of each step ("step t (stage s, N = n)"), of each of its
                                    launches ("bucket k [lo, hi)", "layer id [lo, hi)"; a
                                    clipped step: "reduce ...", "clip decision", "update
                                    ..."), and of each unfused call, so that a profiler
                                    attributes the kernels to buckets and layers; without a
                                    tool attached a range costs a function call.  Default 0;
                                    may be set at any time */
  ZERO_OPT_GUARD = 17,           /* guard bytes around the library's buffers, a stand-in for a
                                    bounds-checking sanitizer: 1 adds 256 bytes after each
                                    arena (arena_bytes grows by 256 for every arena in use) and
                                    makes the unused end of every row of an arena -- each rank
                                    replica, master / m / v, gradient or layer buffer: the
                                    pitch's 256-byte alignment slack and ZERO_OPT_REPLICA_PAD --
                                    a guard too.  zero_load_master and zero_import_state fill
                                    them with the byte 0xA5; zero_check_guards finds bytes
                                    that changed.  2: as 1, and zero_step / zero_step_resident
                                    check them after every step (waiting for the step) and
                                    return ZERO_EGUARD when one changed.  Values are
                                    unchanged.  Default 0; 0 <-> 1 or 2 before zero_bind, 1 <->
                                    2 at any time */
  ZERO_OPT_PDL = 12              /* 1 (default): a step without callbacks (zero_step_resident
                                    with no gather_fn) launches its fused kernels with
                                    programmatic dependent launch, so that each launch's CTAs
                                    start on the SMs the previous launch leaves and, at stage
                                    1/2, stream their own interval while it finishes; at stage 3
                                    a launch loads and computes at once and stores after the
                                    launch before has completed (a staged launch then reserves
                                    at least 116 KB of shared memory, so that an SM never holds
                                    two CTAs of one grid).  A stage-3 step that runs as one
                                    layered launch (ZERO_OPT_LAYERED) has no launch to chain.
                                    0: plain launches.  Values are unchanged either way.  Off while
                                    ZERO_OPT_TIMING is on, and with ZERO_OPT_TMA_CTAS_PER_SM
                                    above 1.  May be set at any time */
};

/* 16-bit storage formats (ZERO_OPT_DTYPE).  The pages account gradients and
 * parameters at 2 bytes and name fp16 as a communication type ([M] section 3.3
 * configuration); bf16 is the default. */
enum { ZERO_DTYPE_BF16 = 0, ZERO_DTYPE_F16 = 1 };

/* Fused-step kernels (ZERO_OPT_KERNEL).  Both compute the same bits, and the
 * choice also applies to the two passes of a clipped step (zero_set_clip),
 * which TMA stages the same way for N <= 16.
 *   REGISTER: each lane loads its 16-byte slices of the N replicas and of
 *             master/m/v straight into registers (any N).
 *   TMA:      one CTA per SM with one or two groups, each a producer thread
 *             that streams its 2048-element tiles of the N replicas and
 *             master/m/v into its own shared-memory stages with bulk copies
 *             (mbarrier-counted) and eight consumer warps that compute from
 *             shared memory (N <= 16); above N = 16, one group whose
 *             producer streams each tile's replicas in chunks of 8 ranks
 *             through a ring of 32 KB stages and its master/m/v through a
 *             second ring (ZERO_OPT_TMA_STAGES = chunk-ring depth).  Its waits are
 *             bounded; one that runs out is reported as ZERO_ECUDA by the next
 *             synchronising call (zero_read_stats, zero_step with stats,
 *             zero_kernel_timing).
 *   BULK:     the staged loads of TMA with bulk stores: one CTA per SM, a
 *             producer thread streaming tiles (ZERO_OPT_TMA_TILE) of the N
 *             replicas and master/m/v into a ring of shared-memory stages
 *             (above N = 16 the replicas in chunks of 8 ranks through a ring
 *             of their own), consumer warps (ZERO_OPT_TMA_WARPS) that
 *             compute and write every result back into shared memory, and a
 *             storer thread that copies the results to master/m/v and the N
 *             destinations with bulk copies (shared -> global), so that no
 *             consumer lane issues a global store.  Bounded waits as TMA.
 *   AUTO:     the bulk-store staged kernel (BULK) for every N, in the
 *             configuration measured fastest on B200 for that N and stage
 *             (zero_fused_config and zero_fused_tile report it). */
enum { ZERO_KERNEL_AUTO = 0, ZERO_KERNEL_REGISTER = 1, ZERO_KERNEL_TMA = 2, ZERO_KERNEL_BULK = 3 };

/* Views (zero_view). */
enum {
  ZERO_VIEW_MASTER = 0,      /* fp32 [psi_pad] */
  ZERO_VIEW_EXP_AVG = 1,     /* fp32 [psi_pad] (m) */
  ZERO_VIEW_EXP_AVG_SQ = 2,  /* fp32 [psi_pad] (v) */
  ZERO_VIEW_PARAM = 3,       /* bf16: rank r's replica [psi_pad] (stage 1, 2) or the
                                shards [psi_pad] (stage 3, rank ignored) */
  ZERO_VIEW_GRAD_SHARD = 4,  /* bf16 [psi_pad] (stage 2, 3) */
  ZERO_VIEW_GRAD_BUF = 5,    /* bf16: rank r's gradient input buffer; with ZERO_OPT_PIPELINE
                                at stage 2/3, rank r + N is rank r's buffer in the second
                                slot set */
  ZERO_VIEW_GATHER = 6       /* bf16: rank r's temporary full-layer buffer (stage 3); with
                                ZERO_OPT_PIPELINE, rank r + N is the second slot set's */
};

typedef struct zero_ctx zero_ctx;

/*
 * Gradient producer: the stand-in for the backward pass ([T] section
 * "ZeRO-2", part "2. 反向": a layer's gradients exist as soon as its backward
 * finishes).  Called once per interval of the schedule, in schedule order,
 * before that interval is reduced.  It must fill, for every rank r, the
 * hi - lo bf16 values of flat elements [lo, hi) at rank_bufs[r] (device
 * pointers into the GRADS arena) with work enqueued on `stream`.  `step` is
 * the number of this step call since the step counter was last set (loaded,
 * imported or zero_set_step): the counter + 1, unless an earlier clipped step
 * was skipped.  Returns 0 on success; any other value aborts the step with
 * ZERO_EINVAL (intervals already updated stay updated; the step counter does
 * not advance).  With ZERO_OPT_PIPELINE, `stream` is the context's own stream
 * (not the one given to zero_step), the call for interval k+1 comes before
 * the step's kernel of interval k has run, and consecutive intervals get
 * alternating buffers.
 */
typedef int (*zero_grad_fn)(void* user, int64_t step, int64_t lo, int64_t hi,
                            void* const* rank_bufs, void* stream);

/*
 * Consumer of a stage-3 temporary gathered layer ([T] section "ZeRO-3",
 * parts "1. 前向" and "2. 反向"): called after the layer [lo, hi) has been
 * gathered into every rank's temporary buffer rank_bufs[r] (hi - lo bf16
 * values) and before the buffer is reused for the next layer.  Work must be
 * enqueued on `stream`.  Returns 0 on success.  With ZERO_OPT_PIPELINE,
 * `stream` is the context's own stream, consecutive layers come in
 * alternating buffers, and the call for layer k follows the grad_fn call of
 * the next interval; the buffers stay valid until the work enqueued by the
 * call has run.
 */
typedef int (*zero_gather_fn)(void* user, int32_t layer, int64_t lo, int64_t hi,
                              void* const* rank_bufs, void* stream);

/* ------------------------------------------------------------------ setup -- */

/* Library ABI version (ZERO_SM_VERSION). */
int32_t zero_version(void);

/*
 * Plan a context for `layout` over n_ranks logical ranks (1..ZERO_MAX_RANKS)
 * at `stage` (ZERO_STAGE_1..3; ZERO_STAGE_DP returns ZERO_ENOTIMPL), with the
 * fixed communication buffer of bucket_elems elements per rank ([M] section
 * 3.3 "CB"; a positive multiple of 8, or 0 for one bucket spanning the whole
 * padded flat space).  Host only, no device work.  *out receives
 * a context owned by the caller (free with zero_destroy).
 * Errors: ZERO_EINVAL for null pointers, bad sizes or decreasing layer ids.
 */
zero_status zero_init(const zero_layout* layout, int32_t n_ranks, int32_t stage,
                      int64_t bucket_elems, zero_ctx** out);

/* Set an option (ZERO_OPT_*).  ZERO_OPT_TIMING, ZERO_OPT_KERNEL, ZERO_OPT_PDL
 * and the staged-kernel options (ZERO_OPT_TMA_GROUPS, ZERO_OPT_TMA_STAGES,
 * ZERO_OPT_TMA_CTAS_PER_SM) may be set at any time; the others size or shape
 * the arenas and are refused with ZERO_ESTATE once the context is bound (so
 * is an unknown key then).  ZERO_EINVAL for a value out of range, and before
 * binding for an unknown key.
 * Library plumbing: no passage of the pages defines it.
 */
zero_status zero_set_option(zero_ctx* ctx, int32_t key, int64_t value);

/*
 * Streams of ZERO_OPT_PIPELINE (host only; before the first pipelined step,
 * ZERO_ESTATE after it): callback_stream is the stream grad_fn and gather_fn
 * receive, kernel_stream the one the step's kernels run on at option value 2.
 * NULL leaves that stream to the context, which then creates it on the first
 * pipelined step (callbacks: a non-blocking stream; kernels: a non-blocking
 * stream at the device's greatest priority) and destroys it in zero_destroy
 * -- so work or bookkeeping of the caller's that still refers to it (for
 * instance a memory allocator that remembers the streams a block was used
 * on) must be finished by then.  Streams given here stay the caller's: the
 * context never destroys them, and they must outlive it.
 * The overlap it serves is [T] section "ZeRO-2"'s reduce-scatter of a bucket
 * while the backward of the next layers runs, and [T] section "ZeRO-3"'s
 * per-layer gathers; the streams themselves are library plumbing.
 */
zero_status zero_set_pipeline_streams(zero_ctx* ctx, void* callback_stream, void* kernel_stream);

/* Sizes of the plan and of each arena (bytes).  Host only.
 * The arenas are [M] section 3.4 "MD"'s one pre-allocated pool; the gradient
 * arena's size is [M] section 3.3 "CB"'s fixed buffer, the gather arena [T]
 * section "ZeRO-3"'s temporary full-layer buffer.
 */
zero_status zero_buffer_sizes(const zero_ctx* ctx, zero_sizes* out);

/* Flat start of every tensor (host array of n_tensors).
 * The flat layout behind [T] section "ZeRO-1"'s partition of the parameter
 * vector (part "optimizer state 怎么切分").
 */
zero_status zero_tensor_offsets(const zero_ctx* ctx, int64_t* out, int32_t cap);

/* The bucket schedule ([M] section 3.3; [T] section "ZeRO-2"): tensors
 * walked from the last to the first, packed into intervals of at most
 * bucket_elems; a larger tensor is cut into bucket-sized chunks from its end.
 * Writes min(cap, n) (lo, hi) pairs to lo_hi and returns n through *n_out. */
zero_status zero_buckets(const zero_ctx* ctx, int64_t* lo_hi, int32_t cap, int32_t* n_out);

/* Layer spans in layer order: (layer id, lo, hi) triples as int64.
 * The layers of [T] section "ZeRO-3" (one layer's parameters gathered at a
 * time).
 */
zero_status zero_layers(const zero_ctx* ctx, int64_t* id_lo_hi, int32_t cap, int32_t* n_out);

/*
 * Lend the arenas: arenas[k] is a device pointer to at least arena_bytes[k]
 * bytes (zero_buffer_sizes), 256-byte aligned, or NULL when that size is 0.
 * Reads the device's SM count and the kernels' occupancy once (the current
 * CUDA device must be the one the arenas live on).  The memory stays the
 * caller's; the library uses it until zero_destroy.
 * Errors: ZERO_EINVAL (null or misaligned), ZERO_ESTATE (already bound),
 * ZERO_ECUDA (device query failed).
 * [M] section 3.4 "MD": one caller-owned pool, lifetimes managed inside it.
 */
zero_status zero_bind(zero_ctx* ctx, void* const* arenas);

/* Adam hyper-parameters (required before any update).
 * The Adam every page names ([T] sections "ZeRO-1" to "ZeRO-3", part "3.
 * 更新").
 */
zero_status zero_set_hparams(zero_ctx* ctx, const zero_adam_hparams* hp);

/*
 * Initialise the optimizer state from fp32 master weights: master_dev is a
 * device array of psi_pad floats (pads 0, 16-byte aligned), or NULL when the
 * caller has already written the master weights into ZERO_VIEW_MASTER (which
 * saves a second psi_pad-sized buffer).  Copies them into the master shards,
 * zeroes m, v and the reduced-gradient shards, writes bf16(master) (round to
 * nearest even) to every rank's parameter replica (stage 1, 2) or to the
 * parameter shards (stage 3), and resets the step counter to 0.
 * Plain DP's identical starting replicas ([T] section "先立一个基线"), with the
 * fp32 master, m and v of [M] section 1's state set.
 */
zero_status zero_load_master(zero_ctx* ctx, const float* master_dev, void* stream);

/*
 * Resume from a checkpoint, possibly taken with a different N or stage (the
 * ownership map of [T] section "ZeRO-1" cuts the same flat vector into N
 * segments, so a re-shard is a reload of the flat state).  master, exp_avg,
 * exp_avg_sq: device arrays (16-byte aligned) holding the flat fp32 state of
 * elements [0, n) -- e.g. copies of another context's ZERO_VIEW_MASTER /
 * _EXP_AVG / _EXP_AVG_SQ; n must be a multiple of 8 that covers every real
 * element (from the end of the last tensor's 8-element slot, which does not
 * depend on N, up to psi_pad).  Elements [n, psi_pad) become 0.  Writes
 * bf16(master) to the parameter replicas (stage 1, 2) or shards (stage 3),
 * clears the reduced-gradient shards and sets the step counter to t, so the
 * next step is t + 1.  The sources are read on `stream`.
 */
zero_status zero_import_state(zero_ctx* ctx, const float* master, const float* exp_avg,
                              const float* exp_avg_sq, int64_t n, int64_t t, void* stream);

/*
 * Step counter: the t of the last update (0 after zero_load_master).  The
 * device holds it, with the bias-correction powers beta^t (t successive
 * binary64 products), and each step's first kernel forms that step's scalars
 * from it -- so a step enqueues nothing but kernels and a step captured in a
 * CUDA graph advances it on every replay.  Both calls wait for the device
 * once the state is loaded.  Changing the betas (zero_set_hparams) rebuilds
 * the powers for the current t.
 * The t of Adam's bias correction (the Adam of [T] sections "ZeRO-1" to
 * "ZeRO-3", part "3. 更新").
 */
zero_status zero_get_step(const zero_ctx* ctx, int64_t* t);
zero_status zero_set_step(zero_ctx* ctx, int64_t t);

/* Device pointer and element count of a view (ZERO_VIEW_*) for rank r.
 * Which rank holds which state follows [T] sections "ZeRO-1" to "ZeRO-3"
 * (owned shards of master, m, v; replicas or shards of the 16-bit
 * parameters).
 */
zero_status zero_view(const zero_ctx* ctx, int32_t what, int32_t rank, void** ptr,
                      int64_t* n_elems);

/* Per-rank long-lived model-state bytes {params, grads, optimizer states}
 * ([Q] sections 二, 三.2, 四.2, 五.2; [M] section 1): 2 B per 16-bit param or
 * grad, 12 B per fp32 master+m+v, each sharded 1/N where the stage shards it.
 * Temporary buffers (the bucket and the gather slots) are not included. */
zero_status zero_state_bytes(const zero_ctx* ctx, int32_t rank, int64_t out[3]);

/* Logical elements each rank sends per step {all-reduce, reduce-scatter,
 * all-gather}, ring convention: a reduce-scatter or an all-gather of P
 * elements sends P(N-1)/N, an all-reduce twice that.  Stage 1: all-reduce +
 * all-gather ([T] section "ZeRO-1"); stage 2: reduce-scatter + all-gather;
 * stage 3: reduce-scatter + two all-gathers, forward and backward ([Q]
 * section 五.4) -- 1.5 times the all-reduce volume ([M] section 2). */
zero_status zero_comm_elems(const zero_ctx* ctx, int64_t out[3]);

/* ------------------------------------------------ the step and its parts -- */
/*
 * Optional global-norm clipping and overflow skip.  Not on the pages (they
 * describe no clipping); the conventions of mixed-precision training:
 *   max_norm > 0     the update uses g * c with c = fp32(max_norm / (||g|| +
 *                    1e-6)) (the quotient in binary64) whenever c < 1, where
 *                    ||g|| is the fp64 norm of the whole averaged gradient;
 *   skip_nonfinite   a step whose averaged gradient holds an Inf or NaN
 *                    changes no state and does not advance the step counter.
 * With either enabled the step needs the norm before any update, so zero_step
 * and zero_step_resident run two passes: every interval is reduced first
 * (stage 2/3 into the reduced-gradient shards, which must be kept; stage 1
 * into the replicas, the all-reduce), a one-thread kernel takes the decision
 * (norm, skip, coefficient) on the device, and a second kernel runs Adam and
 * the broadcast (per layer at stage 3, with gather_fn as before) reading that
 * decision -- no host synchronisation between the passes.  A skipped step
 * writes no state and broadcasts the unchanged parameters.  The host learns
 * the decision when it next needs it (the statistics, zero_get_step, the next
 * step), which advances the step counter only for a step that was not
 * skipped.  Bytes per element at stage 2: (2N+2) + (2+24+2N) = 4N+28.
 * max_norm = 0 and skip_nonfinite = 0 (the default) restore the single fused
 * pass.
 */
zero_status zero_set_clip(zero_ctx* ctx, double max_norm, int32_t skip_nonfinite);

/*
 * Loss scale of mixed-precision training with 16-bit gradients (default 1):
 * the gradients the ranks hold are `scale` times the true ones (so that small
 * values survive binary16).  The averaged gradient is formed and stored in
 * the 16-bit format still scaled -- an overflow there shows as Inf, which
 * zero_set_clip's skip catches -- and the update multiplies it by
 * fp32(1/scale) in binary32 before any clipping.  The reported grad_norm and
 * the clip use the norm of the unscaled gradient.  Not on the pages beyond
 * their mention of fp16 communication; the usual convention.  scale > 0.
 */
zero_status zero_set_loss_scale(zero_ctx* ctx, double scale);



/*
 * Reduce-scatter of [lo, hi) ([T] section "ZeRO-2", part on reduce-scatter;
 * [Q] section 四.3): for every element i, g_i = bf16(fp32 sum over ranks
 * 0..N-1 of rank_grads[r][i - lo], times fp32(1/N)), written to the owner's
 * reduced-gradient shard (GRAD_SHARDS arena, flat index i).  rank_grads is a
 * host array of N device pointers, each at flat element lo of that rank's
 * gradient (16-byte aligned); NULL means the bound GRADS arena buffers
 * (bucket/slot start at lo).  Stage 2 and 3 only.  Also accumulates the
 * gradient norm and non-finite count of the current step.
 */
zero_status zero_reduce_scatter(zero_ctx* ctx, int64_t lo, int64_t hi,
                                const void* const* rank_grads, void* stream);

/*
 * All-reduce of [lo, hi) in place ([T] section "ZeRO-1", part "2. 反向"):
 * every rank's gradient buffer receives the same g_i as above.  rank_grads
 * as for zero_reduce_scatter (NULL = the bound full replicas).  Stage 1.
 */
zero_status zero_all_reduce(zero_ctx* ctx, int64_t lo, int64_t hi, void* const* rank_grads,
                            void* stream);

/*
 * Adam on rank `rank`'s owned shard (-1 = every rank's shard in one launch)
 * for step t >= 1 ([T] section "ZeRO-1", part "3. 更新"): per element, in
 * binary32 with each operation rounded to nearest even, in this order:
 *   p = p*(1-lr*wd);  m = b1*m + (1-b1)*g;  v = b2*v + (1-b2)*(g*g);
 *   p = p - lr*((m/(1-b1^t)) / (sqrt(v/(1-b2^t)) + eps));  out = bf16(p).
 * g is the reduced bf16 gradient (stage 2/3: GRAD_SHARDS; stage 1: the
 * owner's full replica in GRADS).  out goes to the owner's own parameter
 * replica (stage 1/2) or to the parameter shards (stage 3).
 * The step number and the context's step counter (the count of completed
 * steps that zero_step / zero_step_resident use and advance, kept on the
 * device):
 *   t >= 1  the caller's step number is used; the counter is neither read
 *           nor changed.  A caller that mixes explicit-t calls with fused
 *           steps sets the counter with zero_set_step(ctx, k) after its k-th
 *           unfused step, so that the next zero_step runs step k + 1.
 *   t = 0   the step after the counter's value is used (the device is
 *           synchronised to read it); with rank = -1 the call completes that
 *           step and advances the counter by one (again synchronising), with
 *           rank >= 0 the counter is left for the caller to advance
 *           (zero_set_step, or a final rank = -1 call of the same step is NOT
 *           the way: it would update every shard a second time).
 * Errors: ZERO_EINVAL (rank out of range, t < 0), ZERO_ESTATE (not bound,
 * not initialised, hyper-parameters not set, or the gradient buffers it reads
 * were dropped), ZERO_ECUDA (launch, or reading / writing the counter).
 */
zero_status zero_adam_shard(zero_ctx* ctx, int32_t rank, int64_t t, void* stream);

/*
 * All-gather of [lo, hi) ([T] section "ZeRO-1", part on all-gather): the
 * owners' updated bf16 parameters are copied to every rank's destination.
 * Source: stage 1/2 the owner's own replica, stage 3 the parameter shards.
 * rank_out: host array of N device pointers, each at flat element lo of the
 * destination; NULL = the bound destinations (stage 1/2: the N parameter
 * replicas; stage 3: the N temporary layer buffers, [lo, hi) inside one
 * layer, placed at offset lo - layer start).
 */
zero_status zero_all_gather(zero_ctx* ctx, int64_t lo, int64_t hi, void* const* rank_out,
                            void* stream);

/*
 * One full optimizer step t = (step counter) + 1, fused: per interval of the
 * stage's schedule -- stage 1 and 2 the bucket schedule, stage 3 the layers
 * from last to first -- grad_fn fills the ranks' gradient buffers, then one
 * kernel reads the N replicas of each owned element once, reduces them,
 * runs Adam in registers, writes master/m/v once and writes the bf16 result
 * to all N destinations ([T] sections "ZeRO-1", "ZeRO-2", "ZeRO-3").
 * Stage 1 also writes the averaged gradient back to the N replicas (the
 * all-reduce result); stage 3 also writes the parameter shard and then calls
 * gather_fn (may be NULL) with the layer's temporary buffers.
 * grad_fn may be NULL for stage 1 only (the replicas are already filled).
 * stats (may be NULL): when given, the call synchronises `stream` and fills
 * it; otherwise nothing synchronises (zero_read_stats reads it later).
 * The step's scalars come from the device step counter (zero_get_step), so
 * with stats = NULL and ZERO_OPT_TIMING off a step enqueues only kernels and
 * may be captured in a CUDA graph on `stream` and replayed (each replay is
 * one more step; the callbacks run at capture time only, so a captured step
 * replays the work they enqueued then).
 */
zero_status zero_step(zero_ctx* ctx, zero_grad_fn grad_fn, void* grad_user,
                      zero_gather_fn gather_fn, void* gather_user, void* stream,
                      zero_step_stats* stats);

/*
 * The same step reading the gradients from caller-held full replicas:
 * rank_grads is a host array of N device pointers to psi_pad bf16 values
 * each (16-byte aligned).  The schedule, kernels and results are those of
 * zero_step; the intervals index straight into the replicas instead of
 * passing through the fixed-size buffer.  Stage 1 writes the all-reduced
 * gradient back into these replicas.
 * The step of [T] sections "ZeRO-1" to "ZeRO-3", as zero_step.
 */
zero_status zero_step_resident(zero_ctx* ctx, const void* const* rank_grads,
                               zero_gather_fn gather_fn, void* gather_user, void* stream,
                               zero_step_stats* stats);

/*
 * Fused-kernel timing (ZERO_OPT_TIMING = 1): waits for the last recorded
 * launch, then returns the summed device time of the launches recorded since
 * the previous call (*ms), their number (*launches) and the bytes those
 * launches must move by the byte model of the fused step (*model_bytes):
 * per element, stage 1: 6N+24 (N gradient reads, N all-reduce write-backs,
 * 12 B of state read and written, N parameter writes), stage 2: 4N+24,
 * stage 3: 4N+26 (plus the parameter shard), each +2 when the reduced
 * gradient shard is kept.  A clipped step's passes count the reduce as 2N+2
 * (4N at stage 1, the all-reduce written back) and the Adam-broadcast as
 * 2+24+2N (+2 at stage 3).  Resets the record.  At most 4096 launches are
 * recorded between two calls; later ones are not timed.
 * Measurement plumbing: no passage of the pages defines it.
 */
zero_status zero_kernel_timing(zero_ctx* ctx, double* ms, int64_t* launches, double* model_bytes);

/*
 * zero_launch_count -- the number of kernels this context has enqueued since
 * zero_init: every fused, staged, two-pass, Adam, all-gather and
 * initialisation launch, and the one-thread kernels that form and commit the
 * step's device-held counter and scalars.  A zero_step / zero_step_resident
 * enqueues the launches zero_kernel_timing times (one fused launch per
 * non-empty interval; a clipped step its reduce launches and its
 * Adam-broadcast launches, one over the whole buffer at stage 1/2, one per
 * layer at stage 3) plus two of those one-thread kernels.  Host only: reads a
 * counter kept by the launching calls, no device work and no wait.
 * ZERO_EINVAL for a NULL argument.
 * Measurement plumbing: no passage of the pages defines it.
 */
zero_status zero_launch_count(const zero_ctx* ctx, int64_t* n);

/*
 * zero_fused_step_static -- one fused ZeRO-2 step over a single flat interval
 * that allocates nothing.  The pages have no counterpart to this entry point:
 * it exists for callers that cannot allocate device memory when they run the
 * step -- code whose device memory is already entirely owned by another
 * allocator (a framework's caching allocator that reserved the whole device,
 * where an extra cudaMalloc fails or fragments that pool), latency-critical
 * loops that cannot afford the device synchronisation cudaMalloc/cudaFree may
 * cause, and one-off callers that keep no context object to hold a scratch
 * arena.  Such a caller passes only the step's inputs and outputs:
 *   rank_grads   host array of n_ranks device pointers, each to n bf16
 *                gradient values of that rank (16-byte aligned)
 *   master, exp_avg, exp_avg_sq
 *                device fp32 arrays of n values, updated in place
 *   rank_params  host array of n_ranks device pointers, each receiving the n
 *                updated bf16 parameters (16-byte aligned)
 *   hp, t        Adam hyper-parameters and the step number (t >= 1)
 *   stats_out    NULL, or a device pointer to 16 bytes that receives the
 *                step's sum of squares of the averaged gradient (double) and
 *                its non-finite count (uint64)
 * n must be a multiple of 8 and 1 <= n_ranks <= ZERO_MAX_RANKS.  master, m,
 * v and the parameters are those of zero_step for a stage-2 context whose
 * single bucket is this interval, bit for bit; the sum of squares in
 * stats_out is the same sum added in another order (per CTA of this call's
 * own grid), so it may differ from the context step's in the last bits; the
 * non-finite count is exact.  beta^t is formed on the host by t binary64
 * products on every call (no state survives between calls), so a call at
 * step t costs O(t) host time until both powers reach 0.
 *
 * The kernel's scratch (per-CTA norm partials, an arrival counter and the
 * step's sums) is a 32 KiB + 64 B array in the library's device memory,
 * reserved on every GPU that loads the library until the process exits; it
 * holds partials for 2048 CTAs, and a launch takes at most that many CTAs
 * (the kernel loops over any n).  Every call on a device shares that array
 * and it keeps the previous call's contents (the call clears what must start
 * at zero), so two calls that may run at the same time on the GPU -- on
 * different streams with no ordering between them -- race: the statistics
 * are wrong, and stats_out may receive an earlier call's sums with nothing
 * to tell them apart (master, m, v and the parameters are unaffected); calls
 * ordered on one stream are safe.  The first call on each device looks up the
 * array's device address with that device current (a one-time set-up); make
 * that first call before any stream capture begins.
 * Errors: ZERO_EINVAL (bad size, pointer, alignment or hyper-parameter),
 * ZERO_ECUDA (set-up or launch failed).
 */
zero_status zero_fused_step_static(int32_t n_ranks, int64_t n, const void* const* rank_grads,
                                   float* master, float* exp_avg, float* exp_avg_sq,
                                   void* const* rank_params, const zero_adam_hparams* hp,
                                   int64_t t, void* stats_out, void* stream);

/* The fused-step kernel this context launches: *kernel = ZERO_KERNEL_REGISTER,
 * ZERO_KERNEL_TMA or ZERO_KERNEL_BULK; for a staged kernel also its consumer
 * groups (BULK: its consumer warps) and ring depth (0 otherwise).  Host only.
 * Library plumbing: no passage of the pages defines it.
 */
zero_status zero_fused_config(const zero_ctx* ctx, int32_t* kernel, int32_t* groups, int32_t* stages);

/* Elements per tile of the staged kernel this context launches (0 for the
 * register kernel).  Host only.  Library plumbing: no passage defines it. */
zero_status zero_fused_tile(const zero_ctx* ctx, int32_t* tile);

/*
 * zero_probe_pattern -- the ceiling of the step's own memory traffic on this
 * device.  Enqueues on `stream`, for every interval of the step in the step's
 * order and launch chaining, the movement-only twin of the bulk-store kernel
 * in this context's configuration: the same bulk loads of the N gradient
 * slices (rank_grads, as for zero_step_resident) and of master/m/v, the same
 * shared-memory reads and writes, the same bulk stores of master/m/v, of the
 * N parameter destinations, of the ZeRO-3 shard and of the ZeRO-1 write-back
 * or reduced shard -- with no reduction and no Adam: master/m/v are stored
 * back unchanged and the destinations receive the 16-bit rounding of the
 * unchanged master weights.  So a probe leaves the optimizer state and the
 * parameters as a step left them (the ZeRO-1 write-back and the reduced
 * shards receive an XOR of the gradient slices; the step statistics are
 * overwritten with zeros); the step counter does not move.  Timed against
 * the step's byte model it gives the fraction of the traffic pattern's own
 * ceiling that the step reaches.  Not part of the method: no passage of the
 * pages defines it; measurement plumbing.
 * Errors: ZERO_EINVAL (NULL or misaligned pointers), ZERO_ESTATE (not bound
 * or not initialised), ZERO_ENOTIMPL (the configuration of
 * ZERO_OPT_TMA_TILE / ZERO_OPT_TMA_WARPS is not built at this N), ZERO_ECUDA
 * (launch).
 */
zero_status zero_probe_pattern(zero_ctx* ctx, const void* const* rank_grads, void* stream);

/* Synchronise `stream` and read the last step's statistics.
 * The norm and overflow count are not on the pages (the usual mixed-
 * precision checks).
 */
zero_status zero_read_stats(zero_ctx* ctx, void* stream, zero_step_stats* out);

/* Check the guard bytes (ZERO_OPT_GUARD) on `stream` and wait for the
 * result.  Every guard byte that is not 0xA5 is counted and written back,
 * so a later check reports only later changes.  out (may be NULL) =
 * {changed bytes, arena of the first changed byte (ZERO_ARENA_*), its byte
 * offset in that arena}, or {0, -1, -1}.  Returns ZERO_OK when none changed,
 * ZERO_EGUARD when some did (the message names the arena and the row or the
 * tail), ZERO_ESTATE when the context has no guard bytes or its state is
 * not loaded.  A check made while a step is still running on another stream
 * may see that step's stores in progress, never outside its buffers. */
zero_status zero_check_guards(zero_ctx* ctx, void* stream, int64_t out[3]);

/* Message of the last failure on ctx (never NULL; "" when none).  With
 * ctx == NULL: the reason the calling thread's last zero_init failed.
 * Library plumbing: no passage of the pages defines it.
 */
const char* zero_last_error(const zero_ctx* ctx);

/* Release a context (the arenas stay the caller's). NULL is a no-op.  Does
 * not wait for the device: work already enqueued keeps using the arenas, so
 * the caller frees them only after the stream given to the last call has
 * reached that point (every call joins its side streams back into that
 * stream before it returns).  Streams and events the context created are
 * released once their work completes; streams given by
 * zero_set_pipeline_streams stay the caller's.
 * Library plumbing: no passage of the pages defines it.
 */
void zero_destroy(zero_ctx* ctx);

/* ------------------------------------------------ one logical rank per GPU -- */
/*
 * The same step with each data-parallel rank on its own GPU, one process per
 * GPU ([T] sections "ZeRO-1" and "ZeRO-2"; the pages tie ZeRO's cost to the
 * bandwidth between the ranks' devices: [T] section "ZeRO-3", the list of
 * what it is sensitive to, and [M] section 6).  Rank r keeps, in its own
 * GPU's memory and in arenas the caller allocates:
 *   GRAD    its 16-bit gradient replica, psi_pad elements (its backward's
 *           output; stage 1 also receives the all-reduced gradient here);
 *           at stage 3 one layer's gradient, the largest layer's length
 *   PARAM   its 16-bit parameter replica, psi_pad elements; at stage 3 its
 *           parameter shard, S elements
 *   STATES  fp32 master, m and v of its owned shard [rS, (r+1)S)
 *   SCRATCH the step's norm partials and counters
 *   GATHER  stage 3 only: the temporary gathered layer, the largest layer's
 *           length ([T] section "ZeRO-3": each layer's parameters are
 *           gathered into a temporary full buffer for its use)
 * Every rank exports its GRAD, PARAM and GATHER arenas as CUDA IPC records
 * (zero_dist_export), the caller exchanges the records (for instance with
 * torch.distributed all_gather_object) and every rank opens the others'
 * (zero_dist_open_peers).  zero_dist_step then launches, on this GPU, one
 * kernel over the owned shard that reads the N ranks' gradient slices (the
 * peers' through the peer mapping) with plain 16-byte loads, sums them in
 * rank order 0..N-1 in binary32, multiplies by fp32(1/N), rounds to bf16,
 * runs Adam (zero_adam_shard's equations) on the owned fp32 states, and
 * stores bf16(master) into the shard's range of every rank's PARAM replica
 * (stage 1: also the averaged gradient into every rank's GRAD replica): the
 * reduce-scatter, the update and the all-gather in one pass, the same bits
 * as the single-device step and the oracle.  At stage 3 the step goes layer
 * by layer (zero_dist_step_layer): every rank's GRAD buffer holds that
 * layer's gradient, the kernel covers the layer's part of the owned shard,
 * writes the rank's own PARAM shard and stores the result into that part of
 * every rank's GATHER buffer, so that once every rank has run the layer each
 * GATHER buffer holds the whole layer.  No bulk copy or multicast reads
 * another GPU's memory.
 *
 * Ordering between the ranks is the caller's, on the host: every rank's GRAD
 * replica of the step is complete before any rank calls zero_dist_step (for
 * instance: synchronise the stream of the backward, then a barrier), and no
 * rank reads its PARAM replica or writes its GRAD replica again before every
 * rank's step has completed (synchronise the step's stream, then a barrier).
 * zero_dist_load_master has the same contract as a step, and so does each
 * layer of a stage-3 step (its GRAD buffers filled before, its GATHER buffers
 * used and GRAD refilled only after every rank has run it).  No kernel of
 * this API waits on another rank.
 *
 * Errors as for the single-device context: status codes, the text in
 * zero_dist_last_error.  Stages 1, 2 and 3; DP returns ZERO_ENOTIMPL.
 */
typedef struct zero_dist zero_dist;

enum {
  ZERO_DIST_ARENA_GRAD = 0,
  ZERO_DIST_ARENA_PARAM = 1,
  ZERO_DIST_ARENA_STATES = 2,
  ZERO_DIST_ARENA_SCRATCH = 3,
  ZERO_DIST_ARENA_GATHER = 4,  /* stage 3 only (0 bytes otherwise) */
  ZERO_DIST_NUM_ARENAS = 5
};

/* Bytes of one rank's export record (three CUDA IPC handles -- GRAD, PARAM,
 * GATHER -- with the arenas' offsets in their allocations and their lengths;
 * an empty arena's entry is zero; zero padded). */
#define ZERO_DIST_HANDLE_BYTES 256

/* Plan rank `rank` of `world` ranks (1..ZERO_MAX_RANKS) at `stage` (1, 2 or
 * 3): the same partition and layers as zero_init (S = psi_pad / world).
 * Host only.  ZERO_EINVAL for bad arguments, ZERO_ENOTIMPL for DP. */
zero_status zero_dist_init(const zero_layout* layout, int32_t world, int32_t rank, int32_t stage,
                           zero_dist** out);

/* plan = {psi, psi_pad, shard}; arena_bytes[ZERO_DIST_NUM_ARENAS].  Either
 * may be NULL.  Host only. */
zero_status zero_dist_sizes(const zero_dist* d, int64_t plan[3], int64_t arena_bytes[ZERO_DIST_NUM_ARENAS]);

/* Flat offset of every tensor (cap >= n_tensors).  Host only. */
zero_status zero_dist_tensor_offsets(const zero_dist* d, int64_t* out, int32_t cap);

/* Bind this rank's arenas: device pointers on the current device, 256-byte
 * aligned, caller-owned, at least zero_dist_sizes bytes each (an arena of 0
 * bytes may be NULL).  GRAD and PARAM
 * must come from device allocations that CUDA IPC can export (cudaMalloc and
 * allocators built on it; not virtual-memory-managed pools).  Zeroes SCRATCH
 * (synchronously).  With world = 1 no peer needs opening. */
zero_status zero_dist_bind(zero_dist* d, void* const* arenas);

/* Write this rank's export record (ZERO_DIST_HANDLE_BYTES bytes) to `record`:
 * the IPC handles of the allocations holding its GRAD and PARAM arenas and
 * the arenas' offsets in them.  The allocations must stay alive while any
 * peer has them open. */
zero_status zero_dist_export(zero_dist* d, void* record);

/* Open the peers' arenas from `records`: world records in rank order, each
 * ZERO_DIST_HANDLE_BYTES bytes (this rank's own is ignored).  Each distinct
 * allocation is opened once (cudaIpcOpenMemHandle with lazy peer access) and
 * closed by zero_dist_destroy.  ZERO_EINVAL when a record does not describe
 * arenas of this layout's sizes, ZERO_ECUDA when a handle cannot be opened. */
zero_status zero_dist_open_peers(zero_dist* d, const void* records);

/* Adam hyper-parameters (as zero_set_hparams). */
zero_status zero_dist_set_hparams(zero_dist* d, const zero_adam_hparams* hp);

/* Initialise from fp32 master weights: master_full is a device array of
 * psi_pad fp32 values on this GPU (pads 0); the rank copies its shard into
 * STATES, sets m = v = 0 and the step counter to 0, and writes bf16(master)
 * of its shard into every rank's PARAM replica (so that, once every rank has
 * loaded, every replica holds all of them); at stage 3 into its own PARAM
 * shard.  Enqueued on `stream`. */
zero_status zero_dist_load_master(zero_dist* d, const float* master_full, void* stream);

/* One fused step (t = completed steps + 1) over this rank's shard, enqueued
 * on `stream`, as described above; records this rank's share of the
 * gradient norm (sum of squares and non-finite count of its shard's
 * averaged gradient) for zero_dist_read_partial.  The global norm is the
 * square root of the ranks' sums, added in rank order. */
zero_status zero_dist_step(zero_dist* d, void* stream);

/* One layer of a stage-3 step (t = completed steps + 1), enqueued on
 * `stream`: `layer` in layer order (zero_layers of a context with the same
 * layout lists them); every rank's GRAD buffer holds that layer's gradient
 * from element 0.  The rank updates the layer's part of its shard (none when
 * it owns no part of the layer) and stores the result into its PARAM shard
 * and into every rank's GATHER buffer at the part's offset in the layer.
 * The call with `last` != 0 completes the step: the step counter advances
 * and zero_dist_read_partial then gives the step's partial sums (all layers
 * of the step added).  Layers may come in any order ([T] section "ZeRO-3"
 * walks them from the last).  ZERO_ESTATE at stages 1 and 2, ZERO_EINVAL for
 * a layer out of range. */
zero_status zero_dist_step_layer(zero_dist* d, int32_t layer, int32_t last, void* stream);

/* Adam on this rank's shard from an already reduced 16-bit gradient shard
 * (grad_shard: S values on this GPU, 16-byte aligned) -- for a caller whose
 * reduce-scatter and all-gather are collective-library calls (NCCL): the
 * update writes bf16(master) into this rank's own PARAM replica at [rS,
 * (r+1)S) only, and advances the step counter. */
zero_status zero_dist_adam_shard(zero_dist* d, const void* grad_shard, void* stream);

/* Synchronise `stream` and read the last step's partial statistics (sum of
 * squares of this shard's averaged gradient, its non-finite count) and the
 * step counter (step may be NULL). */
zero_status zero_dist_read_partial(zero_dist* d, void* stream, double* sumsq, int64_t* nonfinite, int64_t* step);

/* The step's global statistics from the ranks' partials (host only, no
 * device work): norm = sqrt of sumsq[0] + ... + sumsq[world-1] added in rank
 * order in binary64, and the non-finite counts summed -- the same bits on
 * every rank that passes the same partials.  Not on the pages (the usual
 * mixed-precision norm and overflow report). */
zero_status zero_dist_combine_partials(int32_t world, const double* sumsq, const int64_t* nonfinite, double* norm,
                                       int64_t* nonfinite_total);

/* Local device pointer and length of ZERO_VIEW_MASTER / _EXP_AVG /
 * _EXP_AVG_SQ (the owned shard, S), ZERO_VIEW_PARAM / ZERO_VIEW_GRAD_BUF
 * (this rank's replicas, psi_pad; at stage 3 the parameter shard, S, and the
 * layer gradient buffer) or ZERO_VIEW_GATHER (stage 3: the gathered layer). */
zero_status zero_dist_view(const zero_dist* d, int32_t what, void** ptr, int64_t* n_elems);

/* Message of the last failure (d == NULL: of the calling thread's last
 * zero_dist_init). */
const char* zero_dist_last_error(const zero_dist* d);

/* Close the peers' mappings and release the context (the arenas stay the
 * caller's).  Does not wait for the device: the caller synchronises first,
 * and no peer may still run a step that writes this rank's replicas. */
void zero_dist_destroy(zero_dist* d);

#ifdef __cplusplus
}
#endif

#endif /* ZERO_SM_H */
