// plan.cpp -- host side of libzero_shard.so: partition planner, tensor
// segments, per-stage accounting, error reporting and diagnostics.
//
// ZeRO-DP shards the flat model state into Nd contiguous owner slices
// ("ZeRO memory optimization: training large models", trishampatil.com,
// sections "ZeRO-1", "ZeRO-2", "ZeRO-3"; upskillscore.com guide "ZeRO:
// partitioning training state across GPUs", "How it works").
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <new>

#include "zs_internal.h"

namespace zs {

static thread_local char g_last_error[512] = "";
static std::atomic<uint64_t> g_launches{0};
constexpr int64_t kDefaultWaitBudget = 1ll << 31; // about a second at B200 clocks
static std::atomic<int64_t> g_wait_budget{kDefaultWaitBudget};

long long wait_budget_cycles() { return (long long)g_wait_budget.load(std::memory_order_relaxed); }

zero_status fail(zero_status s, const char* fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return s;
}

void clear_error() { g_last_error[0] = '\0'; }

void count_launches(uint64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

// The entry points of the last kRecentKernels launches, a ring in launch order.
constexpr int kRecentKernels = 64;
static std::mutex g_recent_mu;
static const void* g_recent[kRecentKernels];
static uint64_t g_recent_total = 0;

void record_launch(const void* kernel)
{
    std::lock_guard<std::mutex> lk(g_recent_mu);
    g_recent[g_recent_total % kRecentKernels] = kernel;
    ++g_recent_total;
}

static thread_local bool t_preparing = false;
bool preparing() { return t_preparing; }
PrepareScope::PrepareScope() { t_preparing = true; }
PrepareScope::~PrepareScope() { t_preparing = false; }

} // namespace zs

using zs::fail;

extern "C" {

int32_t zero_abi_version(void) { return ZERO_SHARD_ABI_VERSION; }

const char* zero_strerror(zero_status s)
{
    switch (s) {
    case ZERO_OK: return "ok";
    case ZERO_ERR_INVALID_ARG: return "invalid argument";
    case ZERO_ERR_ALIGNMENT: return "misaligned pointer";
    case ZERO_ERR_CUDA: return "CUDA error";
    case ZERO_ERR_WORKSPACE: return "workspace missing or too small";
    case ZERO_ERR_TIMEOUT: return "timeout";
    case ZERO_ERR_UNSUPPORTED: return "unsupported combination";
    default: return "unknown status";
    }
}

const char* zero_last_error(void) { return zs::g_last_error; }

uint64_t zero_launch_count(void) { return zs::g_launches.load(std::memory_order_relaxed); }

int32_t zero_recent_kernels(const char** names, int32_t max)
{
    if (max < 0 || (max > 0 && !names))
        return -1;
    std::lock_guard<std::mutex> lk(zs::g_recent_mu);
    const uint64_t held = zs::g_recent_total < (uint64_t)zs::kRecentKernels ? zs::g_recent_total
                                                                             : (uint64_t)zs::kRecentKernels;
    const uint64_t n = held < (uint64_t)max ? held : (uint64_t)max;
    for (uint64_t i = 0; i < n; ++i) {
        const void* k = zs::g_recent[(zs::g_recent_total - n + i) % zs::kRecentKernels];
        const char* name = nullptr;
        if (cudaFuncGetName(&name, k) != cudaSuccess || !name)
            name = "?";
        names[i] = name;
    }
    return (int32_t)n;
}

int64_t zero_set_wait_budget(int64_t cycles)
{
    return zs::g_wait_budget.exchange(cycles ? cycles : zs::kDefaultWaitBudget);
}

// Shard length: the smallest multiple of A whose Nd copies cover Psi.
zero_status zero_plan(const zero_plan_desc* d, zero_plan_t** out)
{
    zs::clear_error();
    if (!d || !out)
        return fail(ZERO_ERR_INVALID_ARG, "zero_plan: null desc or out");
    *out = nullptr;
    if (d->psi < 1 || d->nd < 1 || d->align_elems < 1 || d->bucket_elems < 0)
        return fail(ZERO_ERR_INVALID_ARG, "zero_plan: need psi >= 1, nd >= 1, align >= 1, bucket >= 0 "
                    "(got %lld, %d, %lld, %lld)", (long long)d->psi, d->nd,
                    (long long)d->align_elems, (long long)d->bucket_elems);
    if (d->stage < 0 || d->stage > 3)
        return fail(ZERO_ERR_INVALID_ARG, "zero_plan: stage %d not in 0..3", d->stage);
    if (d->reserved != 0)
        return fail(ZERO_ERR_INVALID_ARG, "zero_plan: reserved field must be 0");
    if (d->n_tensors < 0 || (d->n_tensors > 0 && !d->tensor_sizes))
        return fail(ZERO_ERR_INVALID_ARG, "zero_plan: bad tensor list");
    const int64_t nd = d->nd, a = d->align_elems;
    if (a > (INT64_MAX / 4) / nd)
        return fail(ZERO_ERR_INVALID_ARG, "zero_plan: nd * align overflows");

    auto* p = new (std::nothrow) zero_plan_s;
    if (!p)
        return fail(ZERO_ERR_INVALID_ARG, "zero_plan: out of host memory");
    const int64_t group = nd * a;
    p->psi = d->psi;
    p->nd = d->nd;
    p->stage = d->stage;
    p->align = a;
    p->shard_len = ((d->psi + group - 1) / group) * a;
    p->psi_pad = nd * p->shard_len;
    p->bucket = d->bucket_elems;
    p->n_buckets = d->bucket_elems > 0 ? (d->psi + d->bucket_elems - 1) / d->bucket_elems : 1;

    if (d->n_tensors > 0) {
        int64_t total = 0;
        for (int32_t t = 0; t < d->n_tensors; ++t) {
            if (d->tensor_sizes[t] < 0) {
                delete p;
                return fail(ZERO_ERR_INVALID_ARG, "zero_plan: tensor %d has negative size", t);
            }
            total += d->tensor_sizes[t];
        }
        if (total != d->psi) {
            delete p;
            return fail(ZERO_ERR_INVALID_ARG, "zero_plan: tensor sizes sum to %lld, psi is %lld",
                        (long long)total, (long long)d->psi);
        }
        // Walk the tensors in order; a tensor is cut wherever it crosses the
        // end of an owner's slice.
        int64_t base = 0;
        const int64_t L = p->shard_len;
        for (int32_t t = 0; t < d->n_tensors; ++t) {
            const int64_t size = d->tensor_sizes[t];
            p->tensor_offset.push_back(base);
            for (int64_t done = 0; done < size;) {
                const int64_t flat = base + done;
                const int64_t owner = flat / L;
                const int64_t room = (owner + 1) * L - flat;
                const int64_t len = size - done < room ? size - done : room;
                p->segments.push_back({t, owner, done, len, flat - owner * L});
                done += len;
            }
            base += size;
        }
        p->tensor_offset.push_back(base);
    }
    *out = p;
    return ZERO_OK;
}

zero_status zero_plan_query(const zero_plan_t* p, zero_plan_info* out)
{
    zs::clear_error();
    if (!p || !out)
        return fail(ZERO_ERR_INVALID_ARG, "zero_plan_query: null argument");
    out->psi = p->psi;
    out->psi_pad = p->psi_pad;
    out->shard_len = p->shard_len;
    out->align_elems = p->align;
    out->bucket_elems = p->bucket;
    out->n_buckets = p->n_buckets;
    out->n_segments = (int64_t)p->segments.size();
    out->nd = p->nd;
    out->stage = p->stage;
    return ZERO_OK;
}

zero_status zero_plan_shard(const zero_plan_t* p, int32_t owner, int64_t* start, int64_t* real_len)
{
    zs::clear_error();
    if (!p || !start || !real_len)
        return fail(ZERO_ERR_INVALID_ARG, "zero_plan_shard: null argument");
    if (owner < 0 || owner >= p->nd)
        return fail(ZERO_ERR_INVALID_ARG, "zero_plan_shard: owner %d not in [0, %d)", owner, p->nd);
    const int64_t s = (int64_t)owner * p->shard_len;
    int64_t n = p->psi - s;
    n = n < 0 ? 0 : (n > p->shard_len ? p->shard_len : n);
    *start = s;
    *real_len = n;
    return ZERO_OK;
}

zero_status zero_plan_bucket(const zero_plan_t* p, int64_t k, int64_t* start, int64_t* len)
{
    zs::clear_error();
    if (!p || !start || !len)
        return fail(ZERO_ERR_INVALID_ARG, "zero_plan_bucket: null argument");
    if (k < 0 || k >= p->n_buckets)
        return fail(ZERO_ERR_INVALID_ARG, "zero_plan_bucket: bucket %lld not in [0, %lld)",
                    (long long)k, (long long)p->n_buckets);
    if (p->bucket <= 0) {
        *start = 0;
        *len = p->psi;
        return ZERO_OK;
    }
    const int64_t s = k * p->bucket;
    const int64_t e = s + p->bucket < p->psi ? s + p->bucket : p->psi;
    *start = s;
    *len = e - s;
    return ZERO_OK;
}

zero_status zero_plan_segments(const zero_plan_t* p, zero_segment* out, int64_t cap, int64_t* n_out)
{
    zs::clear_error();
    if (!p || !n_out || cap < 0 || (cap > 0 && !out))
        return fail(ZERO_ERR_INVALID_ARG, "zero_plan_segments: bad argument");
    const int64_t n = (int64_t)p->segments.size();
    for (int64_t i = 0; i < n && i < cap; ++i)
        out[i] = p->segments[(size_t)i];
    *n_out = n;
    return ZERO_OK;
}

void zero_plan_destroy(zero_plan_t* p) { delete p; }

// Per-device model-state bytes and per-step communication of each stage.
// Storage per parameter: fp16 parameter 2 B, fp16 gradient 2 B, fp32 Adam
// state (master copy, momentum, variance) 12 B ("ZeRO memory optimization",
// trishampatil.com, "The Real Problem").  Stage s shards, cumulatively, the
// optimizer state (s >= 1), the gradient (s >= 2) and the parameters (s >= 3)
// (same page, table under "The Full Progression, in One View").  A process
// sends Psi elements per collective: reduce-scatter + all-gather, plus a second
// all-gather in stage 3 (upskillscore.com guide, "How it works").
zero_status zero_state_bytes(int64_t psi, int32_t nd, int32_t stage, int64_t align_elems,
                             zero_state_report* r)
{
    zs::clear_error();
    if (!r || psi < 1 || nd < 1 || align_elems < 1 || stage < 0 || stage > 3)
        return fail(ZERO_ERR_INVALID_ARG, "zero_state_bytes: need psi, nd, align >= 1 and stage 0..3");
    const int64_t group = (int64_t)nd * align_elems;
    const int64_t L = ((psi + group - 1) / group) * align_elems;
    struct Part { double bytes_per_param; bool sharded; };
    const Part parts[3] = {{2.0, stage >= 3}, {2.0, stage >= 2}, {12.0, stage >= 1}};
    double b[3];
    int64_t bp[3];
    for (int k = 0; k < 3; ++k) {
        // k Psi / Nd, in the order the formula is written
        const double whole = parts[k].bytes_per_param * (double)psi;
        b[k] = parts[k].sharded ? whole / (double)nd : whole;
        bp[k] = (int64_t)parts[k].bytes_per_param * (parts[k].sharded ? L : psi);
    }
    r->params_bytes = b[0];
    r->grads_bytes = b[1];
    r->optim_bytes = b[2];
    r->total_bytes = b[0] + b[1] + b[2];
    r->params_bytes_padded = bp[0];
    r->grads_bytes_padded = bp[1];
    r->optim_bytes_padded = bp[2];
    r->total_bytes_padded = bp[0] + bp[1] + bp[2];
    r->reduction = 16.0 * (double)psi / r->total_bytes;
    const double collectives = stage >= 3 ? 3.0 : 2.0;
    r->comm_elems = collectives * (double)psi;
    r->comm_bytes = 2.0 * r->comm_elems;
    r->comm_elems_ring = r->comm_elems * (double)(nd - 1) / (double)nd;
    return ZERO_OK;
}

} // extern "C"
