// zs_internal.h -- types shared by the host API (api.cpp, plan.cpp) and the
// kernels (kernels.cu) of libzero_shard.so.  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <vector>

#include <cuda_runtime.h>

#include "zero_shard.h"

struct zero_plan_s {
    int64_t psi = 0;
    int64_t shard_len = 0; // L
    int64_t psi_pad = 0;   // Nd * L
    int64_t align = 1;     // A
    int64_t bucket = 0;    // B (0: one bucket)
    int64_t n_buckets = 1;
    int32_t nd = 1;
    int32_t stage = 0;
    std::vector<zero_segment> segments; // tensor -> owner pieces (optional)
    std::vector<int64_t> tensor_offset;  // flat offset of each tensor, plus psi at the end
};

namespace zs {

// ---- error reporting (plan.cpp) ---------------------------------------------
zero_status fail(zero_status s, const char* fmt, ...);
void clear_error();
void count_launches(uint64_t n);
void record_launch(const void* kernel); // for zero_recent_kernels
long long wait_budget_cycles();  // current budget of a bounded pipeline wait

// A prepare call (zero_shard_step_prepare) runs the step's host logic with
// every launch replaced by loading the kernel: launch geometry is resolved
// and cached, nothing is enqueued.  Per calling thread.
bool preparing();
struct PrepareScope {
    PrepareScope();
    ~PrepareScope();
};

// ---- launch geometry ------------------------------------------------------------
constexpr int kThreads = 256;          // threads per block of the streaming kernels
constexpr int kMaxSegs = 64;           // segments per launch (kernel parameter table)
constexpr int kStatsMaxBlocks = 2048;  // fp64 norm partials per statistics launch
constexpr size_t kHeaderBytes = 256;   // workspace header, before the partials

// A contiguous run of n elements processed by one kernel launch.  Element e
// (0 <= e < n) reads rank r's fp16 contribution at grads[g_off + r*g_rstride + e],
// the fp32 state at [s_off + e] and writes the fp16 parameter at params[p_off + e].
struct Seg {
    int64_t g_off;
    int64_t g_rstride;
    int64_t s_off;
    int64_t p_off;
    int64_t n;
};

struct SegList {
    int32_t count;
    int32_t pad;
    Seg seg[kMaxSegs];
};

// Per-step scalars in the device workspace.  Written by the prep kernel from
// the optimizer state, completed by the finalize / commit kernels.
struct WsHeader {
    unsigned int overflow; // any non-finite reduced gradient seen (atomicOr)
    int32_t skip;          // pre-pass modes: the step is skipped
    int32_t cur;           // live ping-pong slot at the start of the step
    float bc1, bc2;        // bias corrections of the step being applied
    float clip;            // clip coefficient applied by the update
    unsigned int error;    // a bounded pipeline wait gave up (atomicOr)
    double b1p_next, b2p_next;
    double sumsq, norm;
    int64_t t_next;
    float inv;      // unscale factor of this step: fp32 1/(S [* Nd]), S static or dynamic
    int32_t pad2;
    unsigned char pad1[ZERO_VOTE_OFFSET - 80];
    double vote[2]; // split step: {sum of squares, non-finite seen}, at ZERO_VOTE_OFFSET
};
static_assert(sizeof(WsHeader) <= kHeaderBytes, "workspace header too large");
static_assert(offsetof(WsHeader, vote) == ZERO_VOTE_OFFSET, "vote must sit at ZERO_VOTE_OFFSET");

// Source of the reduced gradient in the update kernel.
enum UpdateSrc : int {
    kSrcGradsSpeculative = 0, // fused reduce, overflow flag, ping-pong state
    kSrcGradsInPlace = 1,     // TWO_PASS: re-reduce; skip decided beforehand
    kSrcStash = 2,            // STASH: read the fp32 reduced gradient
};

struct UpdateArgs {
    const uint16_t* grads;
    const float* stash;
    float* master[2];
    float* exp_avg[2];
    float* exp_avg_sq[2];
    uint16_t* params;
    WsHeader* ws;
    int32_t nd;
    float inv;                         // fp32 1/S (or 1/(S*Nd))
    float lr, beta1, beta2, eps, lr_wd;
    float one_minus_beta1, one_minus_beta2;
    zero_step_result* result; // receives status = ZERO_ERR_TIMEOUT on a pipeline fault (may be null)
    long long wait_budget;    // cycles per bounded pipeline wait
    int32_t bf16;             // 16-bit storage of gradients and parameters: 0 fp16, 1 bf16
};

struct StatsArgs {
    const uint16_t* grads;
    float* stash; // nullptr unless STASH
    WsHeader* ws;
    double* partials;
    const zero_opt_state* st; // the dynamic loss scale, when in use
    double scale_mult;        // Nd when averaging, else 1
    int32_t nd;
    float inv;                // static unscale factor
    int32_t bf16;             // 16-bit storage of the contributions: 0 fp16, 1 bf16
};

// Peer tables of a fused reduce-scatter + update + all-gather call (kernel
// parameter, 1 KiB): rank r's contribution to flat element f is at
// grads[r][f]; each new parameter is stored at params[p] and dests[d][p].
constexpr int kMaxPeers = ZERO_MAX_PEERS;
struct PeerTable {
    const uint16_t* grads[kMaxPeers];
    uint16_t* dests[kMaxPeers];
    int32_t n_dests;
    int32_t pad;
};

struct GatherEntry {
    const uint16_t* src;
    int64_t dst_off;
    int64_t n;
    int64_t vec; // 1: src and dst + dst_off 16-byte aligned, copied in 8-element vectors
};

struct GatherList {
    int32_t count;
    int32_t pad;
    GatherEntry e[kMaxSegs];
    int64_t first[kMaxSegs + 1]; // first unit of each piece, then the total (filled by launch_gather)
};

// ---- launchers (kernels.cu); each returns the launch's cudaError_t ----------
cudaError_t launch_opt_init(zero_opt_state* st, float scale, float growth, float backoff, int32_t interval,
                            cudaStream_t s);
cudaError_t launch_prep(const zero_opt_state* st, WsHeader* ws, float beta1, float beta2, float static_inv,
                        double scale_mult, cudaStream_t s);
// peers: nullptr for the strided addressing of UpdateArgs / StatsArgs
cudaError_t launch_update(int src, bool vec, const UpdateArgs& a, const SegList& segs,
                          const PeerTable* peers, cudaStream_t s);
// blocks (= fp64 partials written) of one statistics launch over segs
int stats_blocks(bool vec, const SegList& segs);
cudaError_t launch_stats(bool vec, const StatsArgs& a, const SegList& segs, const PeerTable* peers,
                         cudaStream_t s);
cudaError_t launch_finalize(WsHeader* ws, const double* partials, int64_t n_partials,
                            float max_grad_norm, zero_opt_state* st, zero_step_result* res,
                            cudaStream_t s);
cudaError_t launch_vote_local(WsHeader* ws, const double* partials, int64_t n, cudaStream_t s);
cudaError_t launch_vote_apply(WsHeader* ws, bool speculative, float max_norm, zero_opt_state* st,
                              zero_step_result* res, cudaStream_t s);
cudaError_t launch_commit(bool vec, const UpdateArgs& a, const SegList& segs, bool bookkeeping,
                          zero_opt_state* st, zero_step_result* res, const PeerTable* peers, cudaStream_t s);
cudaError_t launch_cast(bool vec, bool bf16, const float* master, uint16_t* params, const SegList& segs,
                        cudaStream_t s);
// streaming_stores: evict-first stores (compact per-layer buffers) or plain
// ones (a full parameter buffer)
cudaError_t launch_gather(uint16_t* dst, const GatherList& g, bool streaming_stores, cudaStream_t s);
// out[seg.s_off + e] = 16-bit rounding of the rank-order sum of nd contributions
cudaError_t launch_reduce(bool vec, bool bf16, const uint16_t* grads, uint16_t* out, int nd, const SegList& segs,
                          const PeerTable* peers, cudaStream_t s);

} // namespace zs
