/*
 * zero_shard.h -- C ABI of libzero_shard.so, the B200 (sm_100a) ZeRO-DP
 * partitioned mixed-precision Adam shard step.
 *
 * What ZeRO-DP does, and so what this library computes:
 *   Each of Nd data-parallel processes owns one 1/Nd slice of the model state
 *   (fp32 master copy, Adam momentum and variance; stage 2 also the gradient,
 *   stage 3 also the fp16 parameters).  A reduce-scatter brings each owner the
 *   summed gradient of its slice, the owner updates only its slice, and an
 *   all-gather rebuilds the full fp16 parameters.
 *   Sources: anthology-of-the-sota note 103 on ZeRO (dmarx.github.io),
 *   sections "Method" and "Concepts"; "ZeRO memory optimization: training
 *   large models" (trishampatil.com), sections "ZeRO-1", "ZeRO-2", "ZeRO-3"
 *   and "Forward/Backward Under ZeRO-3"; "ZeRO: partitioning training state
 *   across GPUs" (upskillscore.com), section "How it works".
 *
 * On one GPU the Nd ranks are simulated: their fp16 gradient contributions
 * sit side by side in device memory and one fused kernel per call sums them
 * (the reduce-scatter), unscales by the loss scale, checks for inf/NaN,
 * optionally clips by the global L2 norm, applies Adam/AdamW to the owned
 * fp32 state and writes the fp16 cast straight into the full parameter
 * buffer at the owner's offset (the all-gather layout).
 *
 * Arithmetic (the pages give no update equations; textbook readings):
 *   s_i  = c_0,i + c_1,i + ... + c_{Nd-1},i      fp32, left to right by rank
 *   g_i  = s_i * (fp32)(1/S)      [(fp32)(1/(S*Nd)) when averaging; S is the
 *          dynamic loss scale of zero_opt_state when one is in use]
 *   skip the whole step if any g_i (i < Psi, pads excluded) is not finite
 *   norm = sqrt(sum_i (double)g_i^2); c = max/norm if norm > max else 1
 *   g^_i = g_i * c
 *   m = b1*m + (1-b1)*g^;  v = b2*v + (1-b2)*(g^*g^)
 *   p = (p - (lr*wd)*p) - lr*((m/bc1)/(sqrt(v/bc2) + eps))
 *   bc_k = (fp32)(1 - b_k^t), b_k^t kept as fp64 running products
 *   P_i = fp16 round-to-nearest-even of p
 * (Kingma & Ba 2015, Alg. 1; decoupled decay per Loshchilov & Hutter 2019.)
 * Every fp32 operation above is one IEEE-rounded operation (no fused
 * multiply-add), so results are deterministic and independent of the launch
 * geometry; only the norm's fp64 summation order depends on it.
 *
 * Conventions for every call:
 *   - Pointers documented "device" are CUDA device addresses on the device
 *     current when the call is made; "host" pointers are ordinary memory.
 *   - 16-bit data (gradients, parameters) is IEEE binary16 by default, or
 *     bfloat16 where a call's storage argument says so (ZERO_STORAGE_*),
 *     passed as void* / uint16_t bit patterns.  Below, "fp16" names that
 *     16-bit format.
 *   - The caller allocates and owns every device buffer (parameters, state,
 *     gradients, workspace).  The library allocates only the host-side plan
 *     object, never device memory, and never synchronises a stream.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  All device work of a call is enqueued on it, in order.
 *   - Arguments are validated before anything is launched; a failed check
 *     returns a non-zero status and enqueues nothing.  zero_last_error()
 *     then describes the failure (per calling thread).
 *   - A gradient overflow is NOT an error: the call returns ZERO_OK and the
 *     device-side result records overflow = 1.
 */
#ifndef ZERO_SHARD_H
#define ZERO_SHARD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ZERO_SHARD_ABI_VERSION 9

/* Every entry point is exported with default visibility; the library hides
 * everything else. */
#if defined(__GNUC__)
#define ZERO_API __attribute__((visibility("default")))
#else
#define ZERO_API
#endif

/* ---- status codes ------------------------------------------------------- */
typedef int32_t zero_status;
#define ZERO_OK 0
#define ZERO_ERR_INVALID_ARG 1 /* null / out-of-range argument, bad combination */
#define ZERO_ERR_ALIGNMENT 2   /* a pointer is not aligned to its element size  */
#define ZERO_ERR_CUDA 3        /* a CUDA runtime call or launch failed          */
#define ZERO_ERR_WORKSPACE 4   /* workspace missing or smaller than required    */
#define ZERO_ERR_TIMEOUT 5     /* a bounded device-side wait expired (reported in zero_step_result.status) */
#define ZERO_ERR_UNSUPPORTED 6 /* combination not available (e.g. clip + speculative) */

/* ---- enumerations --------------------------------------------------------- */
/* Skip-correct execution modes of zero_shard_step (overflow must be known
 * before any state changes):
 *   SPECULATIVE: one fused pass reads the live state slot and writes the other
 *     (ping-pong master/m/v); the slot index flips only if no overflow was
 *     seen, and on overflow the fp16 parameters are re-cast from the live
 *     master.  Minimal traffic (2*Nd + 26 bytes per owned parameter), +12
 *     bytes of memory per parameter.  No clipping.
 *   TWO_PASS: a statistics pass (overflow flag, norm) re-reads the gradients
 *     before the in-place update.  4*Nd + 26 bytes per parameter, no extra
 *     memory.
 *   STASH: the statistics pass also writes the reduced fp32 gradient to a
 *     caller buffer and the in-place update reads it back.  2*Nd + 34 bytes
 *     per parameter, +4 bytes of memory per parameter. */
#define ZERO_MODE_SPECULATIVE 0
#define ZERO_MODE_TWO_PASS 1
#define ZERO_MODE_STASH 2

/* Layout of the gradient contributions:
 *   FULL (stages 1 and 2: every rank holds a full-size gradient): rank r's
 *     contribution to flat parameter j is grads[r * grad_rank_stride + j],
 *     grad_rank_stride >= psi.
 *   PER_OWNER (stage 3: contributions arrive already partitioned): rank r's
 *     contribution to element i of owner (owner_first + k) is
 *     grads[(k * nd + r) * grad_rank_stride + i], grad_rank_stride >= L
 *     (0 means L).
 *   REDUCED (stage 2 with retention): the owners' reduced gradients as
 *     zero_reduce_scatter keeps them, one value per element: element i of
 *     owner (owner_first + k) is grads[k * L + i]; grad_rank_stride is
 *     ignored.  The step then sums nothing and otherwise runs unchanged
 *     (averaging still divides by the plan's nd). */
#define ZERO_GRADS_FULL 0
#define ZERO_GRADS_PER_OWNER 1
#define ZERO_GRADS_REDUCED 2

/* 16-bit format of the gradient contributions and of the parameters.  The
 * pages' mixed precision uses fp16; bfloat16 (the same 2 bytes, the upper half
 * of a binary32) is the alternative.  Widening is exact for both, narrowing
 * rounds to nearest even; the step's arithmetic is otherwise identical. */
#define ZERO_STORAGE_FP16 0
#define ZERO_STORAGE_BF16 1

/* ---- plan ------------------------------------------------------------------ */
/* Partition of Psi parameters over Nd owners ("ZeRO memory optimization",
 * trishampatil.com, sections "ZeRO-1/2/3"; upskillscore.com guide, "How it
 * works").  Every owner gets a slice of the same padded length
 * L = ceil(Psi / (Nd * A)) * A elements, so shard starts are A-aligned and
 * only the last non-empty shard is short of real elements; pads are never
 * read as data and never written to the parameters.  Buckets are the fixed
 * B-element ranges [k*B, min((k+1)*B, Psi)) of the flat buffer in which the
 * reduce-scatter is issued (the constant-size fused buffers of ZeRO-R,
 * anthology-of-the-sota note 103, "Method"). */
typedef struct zero_plan_desc {
    int64_t psi;                 /* parameters, >= 1 */
    int64_t align_elems;         /* A >= 1 (256 is the usual choice) */
    int64_t bucket_elems;        /* B >= 0; 0 = one bucket holding everything */
    const int64_t* tensor_sizes; /* host, optional: tensors laid back to back; must sum to psi */
    int32_t nd;                  /* data-parallel degree, >= 1 */
    int32_t stage;               /* 0 (plain DP, accounting only), 1, 2 or 3 */
    int32_t n_tensors;           /* entries in tensor_sizes (0 if NULL) */
    int32_t reserved;            /* must be 0 */
} zero_plan_desc;

typedef struct zero_plan_s zero_plan_t; /* opaque, host only */

typedef struct zero_plan_info {
    int64_t psi, psi_pad, shard_len, align_elems, bucket_elems, n_buckets, n_segments;
    int32_t nd, stage;
} zero_plan_info;

/* One piece of a tensor held by one owner (a tensor can straddle owners). */
typedef struct zero_segment {
    int64_t tensor, owner, offset_in_tensor, length, offset_in_shard;
} zero_segment;

/* Builds the plan (host only, no device touched).  *out must later be
 * released with zero_plan_destroy.  Errors: INVALID_ARG for psi < 1, nd < 1,
 * A < 1, B < 0, stage outside 0..3, or tensor sizes that do not sum to psi. */
ZERO_API zero_status zero_plan(const zero_plan_desc* desc, zero_plan_t** out);
ZERO_API zero_status zero_plan_query(const zero_plan_t* plan, zero_plan_info* out);
/* Owner's flat range [start, start + real_len), 0 <= real_len <= L. */
ZERO_API zero_status zero_plan_shard(const zero_plan_t* plan, int32_t owner, int64_t* start, int64_t* real_len);
/* Bucket k's flat range, 0 <= k < n_buckets. */
ZERO_API zero_status zero_plan_bucket(const zero_plan_t* plan, int64_t k, int64_t* start, int64_t* len);
/* Copies up to cap tensor pieces (tensor order, then owner order) into out
 * (host); *n_out receives the total number.  out may be NULL when cap == 0. */
ZERO_API zero_status zero_plan_segments(const zero_plan_t* plan, zero_segment* out, int64_t cap, int64_t* n_out);
ZERO_API void zero_plan_destroy(zero_plan_t* plan);

/* ---- accounting --------------------------------------------------------------- */
/* Model-state bytes per device and communication volume per step.
 * "ZeRO memory optimization" (trishampatil.com): "The Real Problem" (2 Psi
 * fp16 params + 2 Psi fp16 grads + 12 Psi fp32 Adam state = 16 Psi) and the
 * table under "The Full Progression, in One View": stage 0 (plain DP) 16 Psi,
 * stage 1 4 Psi + 12 Psi/Nd, stage 2 2 Psi + 14 Psi/Nd, stage 3 16 Psi/Nd;
 * communication 2 Psi, 2 Psi, 2 Psi, 3 Psi elements per process per step
 * (stage 3 adds a second parameter all-gather, upskillscore.com guide, "How
 * it works").  The *_padded fields replace Psi/Nd by the padded shard length
 * L of alignment A; comm_bytes counts 2 bytes per fp16 element;
 * comm_elems_ring ((Nd-1)/Nd of each collective) is a derived extra. */
typedef struct zero_state_report {
    double params_bytes, grads_bytes, optim_bytes, total_bytes;
    int64_t params_bytes_padded, grads_bytes_padded, optim_bytes_padded, total_bytes_padded;
    double reduction;       /* 16 Psi / total_bytes */
    double comm_elems;      /* per process per step */
    double comm_bytes;
    double comm_elems_ring;
} zero_state_report;

ZERO_API zero_status zero_state_bytes(int64_t psi, int32_t nd, int32_t stage, int64_t align_elems,
                             zero_state_report* out);

/* ---- device-side state -------------------------------------------------------- */
/* Optimizer bookkeeping, resident in device memory (caller allocates >= 64
 * bytes, 8-byte aligned; zero_opt_state_init fills it).  Only the library's
 * kernels update it, so a step never needs a host synchronisation. */
typedef struct zero_opt_state {
    int64_t t;        /* steps applied (skipped steps do not count) */
    double beta1_pow; /* beta1^t, fp64 running product */
    double beta2_pow; /* beta2^t */
    int64_t skipped;  /* steps skipped on overflow */
    int32_t cur;      /* SPECULATIVE: ping-pong slot (0/1) holding the live state */
    int32_t reserved;
    /* Dynamic loss scaling (mixed-precision training, Micikevicius et al.
     * 2018, section 3.2), in use when loss_scale > 0: it then replaces
     * zero_hparams.loss_scale; a skipped step multiplies it by
     * backoff_factor, growth_interval consecutive applied steps multiply it
     * by growth_factor, and good_steps counts the applied steps since the
     * last change.  zero_opt_state_init leaves it off (loss_scale = 0). */
    float loss_scale;
    int32_t good_steps;
    float growth_factor;
    float backoff_factor;
    int32_t growth_interval;
    int32_t reserved2;
} zero_opt_state; /* 64 bytes */

/* Per-call outcome, written to device memory when args->result != NULL. */
typedef struct zero_step_result {
    double grad_norm;  /* global L2 norm of the unscaled reduced gradient;
                          NaN in SPECULATIVE mode and on overflow */
    int64_t t;         /* zero_opt_state.t after the call */
    int64_t skipped;   /* zero_opt_state.skipped after the call */
    float clip_coef;   /* coefficient applied (1 when not clipping) */
    int32_t overflow;  /* 1: a non-finite gradient was seen, nothing was updated */
    int32_t status;    /* ZERO_OK, or ZERO_ERR_TIMEOUT if a pipeline wait inside a
                          kernel gave up (a fault, never expected): SPECULATIVE
                          then keeps the previous state as on overflow; in
                          TWO_PASS / STASH the update is incomplete */
    float loss_scale;  /* dynamic loss scale for the next step (0: static scaling) */
} zero_step_result;

/* ---- the step ---------------------------------------------------------------------- */
typedef struct zero_hparams {
    float lr, beta1, beta2, eps, weight_decay;
    float loss_scale;      /* S > 0; contributions carry the loss scaled by S */
    float max_grad_norm;   /* > 0: clip to this global norm; <= 0: no clipping */
    int32_t average_over_nd; /* 1: divide the sum by Nd as well */
    int32_t mode;          /* ZERO_MODE_* */
    int32_t reserved;      /* must be 0 */
} zero_hparams;

/* Buffers of one call.  The call updates owners owner_first ..
 * owner_first + owner_count - 1 (all Nd owners of a plan: the whole simulated
 * data-parallel group; one owner: a single rank's view).
 *   master/exp_avg/exp_avg_sq[k]: device fp32.  Element i of owner
 *     (owner_first + j) lives at [j * L + i]; only i < real_len is touched.
 *     Slot [1] is required by SPECULATIVE only (and ignored otherwise).
 *     16-byte aligned pointers take the vectorised path.
 *   params: device fp16, the full assembled buffer of psi elements: owner o
 *     writes params[o * L + i].  Positions of other owners are untouched.
 *   grads: device fp16 contributions in grad_layout (ZERO_GRADS_*).
 *   grad_stash: STASH mode only: device fp32 laid out like master.
 *   opt_state: device zero_opt_state; result: device zero_step_result or NULL.
 *   workspace: device scratch of at least zero_workspace_bytes() bytes,
 *     256-byte aligned; contents need no initialisation and are clobbered.
 *   timing_events: optional pair of cudaEvent_t (as void*) recorded on the
 *     stream immediately before and after the parameter-update kernel(s), so
 *     a caller can time the dominant kernel alone; NULL entries = none.
 *   peers: NULL, or the peer tables of the fused reduce-scatter + update +
 *     all-gather (zero_peer_args below); grads and grad_rank_stride are then
 *     ignored. */
typedef struct zero_peer_args zero_peer_args;
typedef struct zero_step_args {
    const void* grads;
    int64_t grad_rank_stride;
    int32_t grad_layout;
    int32_t owner_first;
    int32_t owner_count;
    int32_t storage;        /* ZERO_STORAGE_FP16 or ZERO_STORAGE_BF16 (grads and params) */
    float* master[2];
    float* exp_avg[2];
    float* exp_avg_sq[2];
    void* params;
    float* grad_stash;
    void* opt_state;
    void* result;
    void* workspace;
    size_t workspace_bytes;
    void* timing_events[2];
    const zero_peer_args* peers;   /* host pointer, may be NULL */
} zero_step_args;

/* ---- fused reduce-scatter + update + all-gather over peer memory ------------- */
/* With one process per GPU, a step reads every rank's contribution to its own
 * shard (the reduce-scatter) and ends with every rank holding every owner's
 * new 16-bit parameters (the all-gather) -- "ZeRO: partitioning training
 * state across GPUs" (upskillscore.com), "How it works"; "ZeRO memory
 * optimization" (trishampatil.com), the figure under "Forward/Backward Under
 * ZeRO-3".  With peer tables the step's kernels do both themselves, in the
 * same pass as the arithmetic: they load rank r's contribution straight from
 * rank_grads[r] (this GPU's memory or another GPU's, mapped into this
 * process with zero_ipc_open) and store each new parameter into params and
 * into every param_dests[d] (the other ranks' full parameter buffers).
 * Nothing waits on another GPU inside a kernel: the caller orders the ranks
 * with stream-ordered collectives -- one after the gradients are written and
 * before zero_shard_step_begin (every contribution is complete), the vote
 * all-reduce between begin and end, and one after end (every rank's
 * parameters are complete and its gradient buffer is free again).
 *   rank_grads[r], r < nd: device, rank r's 16-bit gradient buffer in the
 *     FULL layout (the element at flat index f at [f]); the call reads
 *     [o * L, o * L + real_len_o) of it for each owner o of the call.
 *   param_dests[d], d < n_param_dests: device, full parameter buffers (psi
 *     elements, the all-gather layout) written like params.
 *   Entries past nd / n_param_dests are ignored.  The arithmetic and the
 *   results are exactly those of the strided call with the same data.
 * Errors (besides zero_shard_step's): UNSUPPORTED if nd > ZERO_MAX_PEERS or
 * grad_layout is not FULL; INVALID_ARG for a NULL entry or n_param_dests
 * outside [0, ZERO_MAX_PEERS]; ALIGNMENT for an entry not 2-byte aligned
 * (16-byte aligned entries keep the vectorised path). */
#define ZERO_MAX_PEERS 64
struct zero_peer_args {
    const void* rank_grads[ZERO_MAX_PEERS];
    void* param_dests[ZERO_MAX_PEERS];
    int32_t n_param_dests;
    int32_t reserved;        /* must be 0 */
};

/* A device buffer exported for mapping into another process (CUDA IPC).
 * handle: the cudaIpcMemHandle_t of the allocation that holds the buffer;
 * offset: the buffer's byte offset inside that allocation. */
typedef struct zero_ipc_handle {
    unsigned char handle[64];
    int64_t offset;
    int32_t device;          /* ordinal of the exporting device */
    int32_t reserved;
} zero_ipc_handle;

/* Exports the device buffer at dev_ptr (anywhere inside a cudaMalloc
 * allocation) into *out.  Errors: INVALID_ARG for a null argument or a
 * pointer that is not device memory; CUDA. */
ZERO_API zero_status zero_ipc_export(const void* dev_ptr, zero_ipc_handle* out);
/* Maps a buffer exported by another process into this one, with peer access
 * enabled when it lives on another GPU, and returns its address in *dev_ptr.
 * Mapping the same allocation again reuses the mapping (reference counted).
 * Errors: INVALID_ARG; CUDA (e.g. a handle exported by this same process,
 * which CUDA refuses to open). */
ZERO_API zero_status zero_ipc_open(const zero_ipc_handle* h, void** dev_ptr);
/* Releases a mapping made by zero_ipc_open (the address it returned).
 * Errors: INVALID_ARG for an address zero_ipc_open did not return; CUDA. */
ZERO_API zero_status zero_ipc_close(void* dev_ptr);

/* Writes {t = 0, beta1_pow = beta2_pow = 1, skipped = 0, cur = 0, static
 * loss scaling} into the device zero_opt_state at opt_state, on stream. */
ZERO_API zero_status zero_opt_state_init(void* opt_state, void* stream);
/* The same with dynamic loss scaling switched on, starting at initial_scale.
 * Errors: INVALID_ARG unless initial_scale > 0 and finite, growth_factor >= 1,
 * 0 < backoff_factor <= 1 and growth_interval >= 1. */
ZERO_API zero_status zero_opt_state_init_dynamic(void* opt_state, float initial_scale, float growth_factor,
                                                 float backoff_factor, int32_t growth_interval, void* stream);

/* Bytes of scratch a zero_shard_step call with these arguments needs (the
 * workspace fields of args are ignored).  A few hundred bytes in SPECULATIVE
 * mode; in TWO_PASS / STASH also 16 KiB of fp64 norm partials per bucket. */
ZERO_API zero_status zero_workspace_bytes(const zero_plan_t* plan, const zero_hparams* hp,
                                 const zero_step_args* args, size_t* bytes);

/* One ZeRO-DP step for the owners in args (reduce-scatter sum + unscale +
 * overflow check + optional clip + Adam + fp16 cast into the all-gather
 * layout), enqueued on stream without host synchronisation.  On overflow
 * nothing changes: master/m/v, params (see SPECULATIVE note below) and
 * opt_state.t keep their values and opt_state.skipped grows by one.
 * SPECULATIVE note: on a skipped step params is rewritten as the fp16 cast of
 * the unchanged live master, which equals its previous contents whenever
 * params holds that cast (true after any step of this library, and after
 * zero_cast_params).
 * The overflow flag and the norm are global over every owner of the call.
 * Errors: INVALID_ARG (null pointers, owner range outside the plan, bad
 * hyper-parameters or layout), ALIGNMENT (pointer not aligned to its element
 * size), UNSUPPORTED (clipping in SPECULATIVE mode), WORKSPACE, CUDA. */
ZERO_API zero_status zero_shard_step(const zero_plan_t* plan, const zero_hparams* hp,
                            const zero_step_args* args, void* stream);

/* Everything zero_shard_step (and its two halves, zero_shard_step_begin and
 * _end) would do for these arguments except enqueueing work: the same
 * validation, then each kernel the call would launch is loaded and its
 * launch geometry (SM count, blocks per SM, shared-memory limit) resolved
 * and cached for the current device.  Launches nothing, records no timing
 * event, touches no device memory and changes no optimizer state, so the
 * next zero_shard_step is the first step.  Call it before capturing steps
 * into a CUDA graph: the captured calls then neither load a kernel nor query
 * the device.  Returns the status zero_shard_step would return for these
 * arguments, minus the launch-time CUDA errors (nothing is launched).  Not a
 * page's operation: a host-side convenience of this library. */
ZERO_API zero_status zero_shard_step_prepare(const zero_plan_t* plan, const zero_hparams* hp,
                                             const zero_step_args* args);

/* ---- split step: one owner per process -------------------------------------- */
/* When each owner runs in its own process (one GPU each), a step's global
 * decisions -- skip on a non-finite gradient anywhere, the global clip norm --
 * need every owner's gradient.  zero_shard_step_begin and _end split the step
 * around one sum-all-reduce of a 16-byte "vote" that the library keeps in the
 * workspace at byte offset ZERO_VOTE_OFFSET: two fp64 values, {this call's
 * sum of squares of the unscaled reduced gradient (0 in SPECULATIVE mode),
 * 1 if this call saw a non-finite gradient else 0}.  The caller adds the
 * votes of all processes (e.g. an NCCL fp64 sum over the group, in place on
 * the stream between the two calls); any non-zero second value then skips
 * the step everywhere, and the summed first value gives the global norm.
 *   SPECULATIVE: begin = fused update into the spare slot + vote; end =
 *     commit (or re-cast on skip).  TWO_PASS / STASH: begin = statistics
 *     pass + vote; end = decision + in-place update.
 * begin + end with no reduction in between equal zero_shard_step over the
 * call's owners; arguments, workspace and errors are those of
 * zero_shard_step, and both calls must receive the same arguments.  The
 * exchange of gradient slices before begin (each owner gathers the Nd
 * contributions to its shard: the reduce-scatter's input) and the
 * all-gather of the fp16 shards after end are the caller's collectives. */
#define ZERO_VOTE_OFFSET 128
ZERO_API zero_status zero_shard_step_begin(const zero_plan_t* plan, const zero_hparams* hp,
                                           const zero_step_args* args, void* stream);
ZERO_API zero_status zero_shard_step_end(const zero_plan_t* plan, const zero_hparams* hp,
                                         const zero_step_args* args, void* stream);

/* Size of the device scratch array that zero_shard_step_static_scratch uses
 * (1 MiB on every GPU that loads the library, kept until the process exits). */
#define ZERO_STATIC_SCRATCH_BYTES (1 << 20)

/* zero_shard_step for callers that cannot allocate device memory.  This entry
 * point has no counterpart on the ZeRO pages; it exists for code that runs
 * where a cudaMalloc is not available or not allowed -- inside a framework
 * whose caching allocator owns the whole device and forbids raw allocations
 * beside it, in plug-in or embedded runtimes that are handed buffers but no
 * allocator, or in step loops where an allocation (which may synchronise the
 * device) is not acceptable.
 *
 * Behaviour, arguments and errors are those of zero_shard_step, except that
 * args->workspace and args->workspace_bytes are ignored: the scratch (the
 * per-step header and the fp64 norm partials) lives in one static device
 * array of ZERO_STATIC_SCRATCH_BYTES inside the library.  No call allocates
 * or frees device memory.
 *   - Limit: SPECULATIVE calls need 256 bytes; TWO_PASS and STASH calls need
 *     256 bytes plus 8 per statistics block (at most 2048 blocks per
 *     bucket), i.e. up to 63 full-size buckets.  A call needing more returns
 *     ZERO_ERR_WORKSPACE before anything is launched (zero_workspace_bytes
 *     tells the size in advance).
 *   - The first call on a device resolves the array's device address with
 *     that device current and caches it for the current CUDA context; make
 *     that first call before any stream capture begins.  The address lives
 *     as long as that context: after cudaDeviceReset (or any teardown of
 *     the context) the next call, in the new context, resolves it again.
 *   - Every call on a device shares the one array, which keeps the last
 *     call's contents.  Each call rewrites the header and every partial it
 *     reads before reading it, so nothing has to start at zero.  Calls whose
 *     GPU work overlaps (unordered streams, or host threads racing on one
 *     device) race on the array and corrupt each other's overflow flag and
 *     norm: order them, e.g. on one stream. */
ZERO_API zero_status zero_shard_step_static_scratch(const zero_plan_t* plan, const zero_hparams* hp,
                                                    const zero_step_args* args, void* stream);

/* Reduce-scatter with retention (ZeRO stage 2, P_os+g): the owner of a slice
 * keeps the rank-order sum of that slice's gradients, after which no rank
 * needs its full gradient buffer for that slice any more.  Stage 2 as
 * described in "ZeRO: partitioning training state across GPUs"
 * (upskillscore.com), "How it works", and "ZeRO memory optimization"
 * (trishampatil.com), "ZeRO-2".
 *   For the owners owner_first .. owner_first + owner_count - 1 of args and
 *   the flat range of bucket `bucket` of the plan (bucket < 0: the owners'
 *   whole range; a plan without buckets has the one bucket 0), writes
 *   grad_shards[k * L + i] = the rank-order fp32 sum of the Nd
 *   contributions to element i of owner (owner_first + k), rounded once to
 *   nearest even in args->storage's 16-bit format.  Pads (i >= real_len)
 *   and elements outside the bucket are not written.
 *   The contributions come from args->grads in args->grad_layout (FULL or
 *   PER_OWNER) or through args->peers; every other field of args is
 *   ignored.  grad_shards: device, owner_count * L 16-bit values; a
 *   16-byte aligned buffer (with 16-byte aligned contributions) takes the
 *   vectorised path.
 *   The step consumes the result with grad_layout = ZERO_GRADS_REDUCED.  A
 *   sum beyond the format's range is kept as inf and skips that step.
 *   Bucket by bucket, a caller can reduce each bucket as soon as every rank
 *   has produced it and then reuse the ranks' buffers for it.
 * Errors: INVALID_ARG (null pointers, owner range, layout, bucket outside
 * [0, n_buckets)), ALIGNMENT, UNSUPPORTED (peer-table limits), CUDA. */
ZERO_API zero_status zero_reduce_scatter(const zero_plan_t* plan, const zero_step_args* args, int64_t bucket,
                                         void* grad_shards, void* stream);

/* Gather-assembly (the stage-3 all-gather seen by one rank): for every owner
 * r whose shard_ptrs[r] (host array of nd device pointers) is not NULL,
 * copies its fp16 shard [0, real_len_r) into params_full[r * L ...].
 * "ZeRO memory optimization" (trishampatil.com), "Forward/Backward Under
 * ZeRO-3": a process gathers the parameter shards it does not own. */
ZERO_API zero_status zero_gather_params(const zero_plan_t* plan, const void* const* shard_ptrs,
                               void* params_full, void* stream);

/* On-demand gather of a tensor range, for stage 3: a layer's parameters are
 * gathered when the forward or backward pass reaches them and released after
 * use ("ZeRO memory optimization", trishampatil.com, "ZeRO-3" and the figure
 * under "Forward/Backward Under ZeRO-3").  Tensors first_tensor ..
 * first_tensor + n_tensors - 1 of the plan's tensor list (the plan must have
 * one) are assembled from the owners' fp16 shards (shard_ptrs: host array of
 * nd device pointers, [L] each): the element at flat index f comes from
 * shard f / L at f % L.  compact = 0: into `out` (device fp16, Psi elements)
 * at the flat index; a NULL shard is then skipped (its part is already in
 * place).  compact = 1: tensors back to back from out[0] (device fp16, the
 * range's element count); every needed shard must be given.  *elements
 * (host, may be NULL) receives the number of elements copied -- the gather's
 * communication volume when the shards live on other processes. */
ZERO_API zero_status zero_gather_tensors(const zero_plan_t* plan, int32_t first_tensor, int32_t n_tensors,
                                         const void* const* shard_ptrs, void* out, int32_t compact,
                                         int64_t* elements, void* stream);

/* zero_gather_tensors moved by the GPU's copy engines instead of a kernel:
 * the same pieces, arguments, results and errors, with one device-to-device
 * cudaMemcpyAsync per run of pieces that continue each other in both the
 * shard and the destination (the consecutive tensors one owner holds).  No
 * SM runs the copy, so it proceeds beside kernels that occupy every SM on
 * other streams (a layer's compute while the next layer is prefetched),
 * where a copy kernel would wait for SMs; alone it is slower than the
 * kernel.  Shards on other GPUs (mapped with zero_ipc_open) are reached the
 * same way, over NVLink. */
ZERO_API zero_status zero_gather_tensors_dma(const zero_plan_t* plan, int32_t first_tensor, int32_t n_tensors,
                                             const void* const* shard_ptrs, void* out, int32_t compact,
                                             int64_t* elements, void* stream);

/* params[(owner_first + j) * L + i] = cast(master[j * L + i]) for the owners
 * owner_first .. owner_first + owner_count - 1, in the 16-bit format
 * `storage` (ZERO_STORAGE_*): establishes the 16-bit copy of a freshly
 * initialised fp32 master (device pointers). */
ZERO_API zero_status zero_cast_params(const zero_plan_t* plan, const float* master, void* params,
                             int32_t owner_first, int32_t owner_count, int32_t storage, void* stream);

/* ---- diagnostics ---------------------------------------------------------------- */
ZERO_API int32_t zero_abi_version(void);
ZERO_API const char* zero_strerror(zero_status status);
/* Message of the last failed call on this thread ("" if none). */
ZERO_API const char* zero_last_error(void);
/* Number of kernels this library has launched in this process. */
ZERO_API uint64_t zero_launch_count(void);
/* Names of the kernels this library launched last in this process (up to the
 * last 64 launches, from all threads), oldest first, as the compiler emits
 * them (mangled C++ names, e.g. containing "zs_update_pipe_kernel"): writes
 * up to `max` pointers into `names` (host array) and returns how many.  The
 * strings belong to the CUDA runtime and stay valid while the library is
 * loaded.  Returns -1 if max < 0, or if max > 0 and names is NULL.  For
 * diagnostics and tests: which update kernel a call's shape rules chose. */
ZERO_API int32_t zero_recent_kernels(const char** names, int32_t max);
/* Budget, in SM clock cycles, of each bounded wait inside the pipelined
 * update kernel (default 2^31, about a second).  A wait that exceeds it makes
 * the step report status ZERO_ERR_TIMEOUT instead of hanging.  A negative
 * value makes every such wait expire at once (a test hook for that path: the
 * kernel then copies and updates nothing).  The final wait for the kernel's
 * own copies in flight always keeps the default budget.  0 restores the
 * default.  Returns the previous value.  Process-wide; affects steps
 * enqueued afterwards. */
ZERO_API int64_t zero_set_wait_budget(int64_t cycles);

#ifdef __cplusplus
}
#endif

#endif /* ZERO_SHARD_H */
