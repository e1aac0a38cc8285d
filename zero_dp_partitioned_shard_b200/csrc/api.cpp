// api.cpp -- C ABI entry points of libzero_shard.so that touch the device:
// argument validation, launch planning and the per-mode kernel sequences.
// Nothing here allocates device memory or synchronises a stream.
#include <cmath>
#include <cstring>
#include <vector>

#include "zs_internal.h"

using zs::fail;

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The kernel launches of one zero_shard_step call.
struct LaunchPlan {
    bool vec = false;                               // 16-byte vector path
    std::vector<std::vector<zs::SegList>> buckets;  // grad-reading launches, bucket by bucket
    std::vector<zs::SegList> whole;                 // the call's full range
    int64_t n_partials = 0;                         // fp64 norm partials of all statistics launches
};

void push_seg(std::vector<zs::SegList>& lists, const zs::Seg& s)
{
    if (s.n <= 0)
        return;
    if (lists.empty() || lists.back().count == zs::kMaxSegs) {
        zs::SegList l;
        std::memset(&l, 0, sizeof l);
        lists.push_back(l);
    }
    lists.back().seg[lists.back().count++] = s;
}

// Segments covering flat range [lo, hi) of the owners starting at o0.
void segments_of(const zero_plan_s& p, int layout, int64_t stride, int32_t o0, int64_t lo,
                 int64_t hi, std::vector<zs::SegList>& out)
{
    // per-owner blocks hold nd contributions (PER_OWNER) or one (REDUCED)
    const int64_t per_owner = layout == ZERO_GRADS_REDUCED ? 1 : p.nd;
    const int64_t L = p.shard_len;
    if (lo >= hi)
        return;
    if (layout == ZERO_GRADS_FULL) {
        // every array is addressed by the flat index, so owners run together
        push_seg(out, zs::Seg{lo, stride, lo - (int64_t)o0 * L, lo, hi - lo});
        return;
    }
    for (int64_t o = lo / L; o * L < hi; ++o) {
        const int64_t i0 = (lo > o * L ? lo : o * L) - o * L;
        const int64_t i1 = (hi < (o + 1) * L ? hi : (o + 1) * L) - o * L;
        const int64_t j = o - o0;
        push_seg(out, zs::Seg{j * per_owner * stride + i0, stride, j * L + i0, o * L + i0, i1 - i0});
    }
}

bool segs_vec_ok(const std::vector<zs::SegList>& lists)
{
    for (const auto& l : lists)
        for (int i = 0; i < l.count; ++i)
            if ((l.seg[i].g_off | l.seg[i].s_off | l.seg[i].p_off | l.seg[i].g_rstride) & 7)
                return false;
    return true;
}

int64_t effective_stride(const zero_plan_s& p, const zero_step_args& a)
{
    if (a.peers) // one buffer per rank: the stride is not used
        return 0;
    if (a.grad_layout == ZERO_GRADS_REDUCED) // one value per element, owners back to back
        return p.shard_len;
    if (a.grad_layout == ZERO_GRADS_PER_OWNER && a.grad_rank_stride == 0)
        return p.shard_len;
    return a.grad_rank_stride;
}

// Checks of where a call's gradient contributions come from and which owners
// it covers (zero_shard_step and zero_reduce_scatter).  reduced_ok: the
// REDUCED layout is accepted (the step's input, not the reduce-scatter's).
zero_status validate_source(const zero_plan_s* p, const zero_step_args* a, bool reduced_ok)
{
    if (a->storage != ZERO_STORAGE_FP16 && a->storage != ZERO_STORAGE_BF16)
        return fail(ZERO_ERR_INVALID_ARG, "unknown 16-bit storage format %d", a->storage);
    if (a->owner_first < 0 || a->owner_count < 1 || a->owner_first > p->nd - a->owner_count)
        return fail(ZERO_ERR_INVALID_ARG, "owner range [%d, %d + %d) outside [0, %d)",
                    a->owner_first, a->owner_first, a->owner_count, p->nd);
    const bool reduced = a->grad_layout == ZERO_GRADS_REDUCED;
    if (a->grad_layout != ZERO_GRADS_FULL && a->grad_layout != ZERO_GRADS_PER_OWNER && !(reduced && reduced_ok))
        return fail(ZERO_ERR_INVALID_ARG, "grad_layout %d not accepted here", a->grad_layout);
    if (a->peers) {
        const zero_peer_args& q = *a->peers;
        if (a->grad_layout != ZERO_GRADS_FULL)
            return fail(ZERO_ERR_UNSUPPORTED, "peer tables need the FULL gradient layout");
        if (p->nd > ZERO_MAX_PEERS)
            return fail(ZERO_ERR_UNSUPPORTED, "peer tables hold at most %d ranks (nd = %d)", ZERO_MAX_PEERS, p->nd);
        if (q.n_param_dests < 0 || q.n_param_dests > ZERO_MAX_PEERS)
            return fail(ZERO_ERR_INVALID_ARG, "n_param_dests %d outside [0, %d]", q.n_param_dests, ZERO_MAX_PEERS);
        if (q.reserved != 0)
            return fail(ZERO_ERR_INVALID_ARG, "reserved fields must be 0");
        for (int r = 0; r < p->nd; ++r) {
            if (!q.rank_grads[r])
                return fail(ZERO_ERR_INVALID_ARG, "rank_grads[%d] is null", r);
            if (!aligned(q.rank_grads[r], 2))
                return fail(ZERO_ERR_ALIGNMENT, "rank_grads[%d] must be 2-byte aligned", r);
        }
        for (int d = 0; d < q.n_param_dests; ++d) {
            if (!q.param_dests[d])
                return fail(ZERO_ERR_INVALID_ARG, "param_dests[%d] is null", d);
            if (!aligned(q.param_dests[d], 2))
                return fail(ZERO_ERR_ALIGNMENT, "param_dests[%d] must be 2-byte aligned", d);
        }
        return ZERO_OK;
    }
    const int64_t stride = effective_stride(*p, *a);
    if (a->grad_layout == ZERO_GRADS_FULL && p->nd > 1 && stride < p->psi)
        return fail(ZERO_ERR_INVALID_ARG, "FULL layout needs grad_rank_stride >= psi (%lld < %lld)",
                    (long long)stride, (long long)p->psi);
    if (a->grad_layout == ZERO_GRADS_PER_OWNER && stride < p->shard_len)
        return fail(ZERO_ERR_INVALID_ARG, "PER_OWNER layout needs grad_rank_stride >= L (%lld < %lld)",
                    (long long)stride, (long long)p->shard_len);
    if (!a->grads)
        return fail(ZERO_ERR_INVALID_ARG, "null grads");
    if (!aligned(a->grads, 2))
        return fail(ZERO_ERR_ALIGNMENT, "16-bit buffers must be 2-byte aligned");
    return ZERO_OK;
}

zero_status validate(const zero_plan_s* p, const zero_hparams* hp, const zero_step_args* a)
{
    if (!p || !hp || !a)
        return fail(ZERO_ERR_INVALID_ARG, "zero_shard_step: null plan, hparams or args");
    if (hp->mode < ZERO_MODE_SPECULATIVE || hp->mode > ZERO_MODE_STASH)
        return fail(ZERO_ERR_INVALID_ARG, "unknown mode %d", hp->mode);
    if (hp->reserved != 0)
        return fail(ZERO_ERR_INVALID_ARG, "reserved fields must be 0");
    if (!(hp->loss_scale > 0.0f) || !std::isfinite(hp->loss_scale))
        return fail(ZERO_ERR_INVALID_ARG, "loss_scale must be finite and > 0");
    if (!std::isfinite(hp->lr) || !std::isfinite(hp->weight_decay) || !std::isfinite(hp->eps) ||
        hp->eps < 0.0f || !std::isfinite(hp->max_grad_norm))
        return fail(ZERO_ERR_INVALID_ARG, "lr, weight_decay, eps, max_grad_norm must be finite, eps >= 0");
    if (!(hp->beta1 >= 0.0f && hp->beta1 < 1.0f) || !(hp->beta2 >= 0.0f && hp->beta2 < 1.0f))
        return fail(ZERO_ERR_INVALID_ARG, "betas must lie in [0, 1)");
    if (hp->average_over_nd != 0 && hp->average_over_nd != 1)
        return fail(ZERO_ERR_INVALID_ARG, "average_over_nd must be 0 or 1");
    if (hp->mode == ZERO_MODE_SPECULATIVE && hp->max_grad_norm > 0.0f)
        return fail(ZERO_ERR_UNSUPPORTED, "global-norm clipping needs the norm before any update: "
                    "use TWO_PASS or STASH mode");
    zero_status s = validate_source(p, a, true);
    if (s != ZERO_OK)
        return s;
    if (!a->master[0] || !a->exp_avg[0] || !a->exp_avg_sq[0] || !a->params || !a->opt_state)
        return fail(ZERO_ERR_INVALID_ARG, "null device buffer (master, exp_avg, exp_avg_sq, params, opt_state)");
    const bool spec = hp->mode == ZERO_MODE_SPECULATIVE;
    if (spec && (!a->master[1] || !a->exp_avg[1] || !a->exp_avg_sq[1]))
        return fail(ZERO_ERR_INVALID_ARG, "SPECULATIVE mode needs the second state slot");
    if (hp->mode == ZERO_MODE_STASH && !a->grad_stash)
        return fail(ZERO_ERR_INVALID_ARG, "STASH mode needs grad_stash");
    for (int k = 0; k < (spec ? 2 : 1); ++k)
        if (!aligned(a->master[k], 4) || !aligned(a->exp_avg[k], 4) || !aligned(a->exp_avg_sq[k], 4))
            return fail(ZERO_ERR_ALIGNMENT, "fp32 state buffers must be 4-byte aligned");
    if (!aligned(a->params, 2))
        return fail(ZERO_ERR_ALIGNMENT, "16-bit buffers must be 2-byte aligned");
    if (a->grad_stash && !aligned(a->grad_stash, 4))
        return fail(ZERO_ERR_ALIGNMENT, "grad_stash must be 4-byte aligned");
    if (!aligned(a->opt_state, 8) || (a->result && !aligned(a->result, 8)))
        return fail(ZERO_ERR_ALIGNMENT, "opt_state / result must be 8-byte aligned");
    return ZERO_OK;
}

LaunchPlan plan_launches(const zero_plan_s& p, const zero_hparams& hp, const zero_step_args& a)
{
    LaunchPlan lp;
    const int64_t L = p.shard_len;
    const int64_t stride = effective_stride(p, a);
    const int64_t lo = (int64_t)a.owner_first * L;
    int64_t hi = (int64_t)(a.owner_first + a.owner_count) * L;
    if (hi > p.psi)
        hi = p.psi;

    if (p.bucket > 0) {
        for (int64_t k = 0; k < p.n_buckets; ++k) {
            const int64_t b0 = k * p.bucket > lo ? k * p.bucket : lo;
            const int64_t b1 = (k + 1) * p.bucket < hi ? (k + 1) * p.bucket : hi;
            if (b0 >= b1)
                continue;
            lp.buckets.emplace_back();
            segments_of(p, a.grad_layout, stride, a.owner_first, b0, b1, lp.buckets.back());
        }
    } else if (lo < hi) {
        lp.buckets.emplace_back();
        segments_of(p, a.grad_layout, stride, a.owner_first, lo, hi, lp.buckets.back());
    }
    segments_of(p, a.grad_layout, stride, a.owner_first, lo, hi, lp.whole);
    if (lp.whole.empty()) {
        zs::SegList empty;
        std::memset(&empty, 0, sizeof empty);
        lp.whole.push_back(empty);
    }
    const bool spec = hp.mode == ZERO_MODE_SPECULATIVE;
    bool vec = (L % 8 == 0) && (p.bucket % 8 == 0) && (stride % 8 == 0) && aligned(a.params, 16);
    if (a.peers) {
        for (int r = 0; r < p.nd; ++r)
            vec = vec && aligned(a.peers->rank_grads[r], 16);
        for (int d = 0; d < a.peers->n_param_dests; ++d)
            vec = vec && aligned(a.peers->param_dests[d], 16);
    } else {
        vec = vec && aligned(a.grads, 16);
    }
    for (int k = 0; k < (spec ? 2 : 1); ++k)
        vec = vec && aligned(a.master[k], 16) && aligned(a.exp_avg[k], 16) && aligned(a.exp_avg_sq[k], 16);
    if (hp.mode == ZERO_MODE_STASH)
        vec = vec && aligned(a.grad_stash, 16);
    vec = vec && segs_vec_ok(lp.whole);
    for (const auto& b : lp.buckets)
        vec = vec && segs_vec_ok(b);
    lp.vec = vec;
    for (const auto& b : lp.buckets)
        for (const auto& l : b)
            lp.n_partials += zs::stats_blocks(vec, l);
    return lp;
}

// The peer table of a call (kernel parameter), or nullptr without peer tables.
const zs::PeerTable* make_peer_table(const zero_plan_s& p, const zero_step_args& a, zs::PeerTable* pt)
{
    if (!a.peers)
        return nullptr;
    std::memset(pt, 0, sizeof *pt);
    for (int r = 0; r < p.nd; ++r)
        pt->grads[r] = static_cast<const uint16_t*>(a.peers->rank_grads[r]);
    for (int d = 0; d < a.peers->n_param_dests; ++d)
        pt->dests[d] = static_cast<uint16_t*>(a.peers->param_dests[d]);
    pt->n_dests = a.peers->n_param_dests;
    return pt;
}

size_t workspace_need(const zero_hparams& hp, const LaunchPlan& lp)
{
    if (hp.mode == ZERO_MODE_SPECULATIVE)
        return zs::kHeaderBytes;
    return zs::kHeaderBytes + (size_t)lp.n_partials * sizeof(double);
}

zero_status cuda_fail(cudaError_t e, const char* what)
{
    return fail(ZERO_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

} // namespace

extern "C" {

zero_status zero_opt_state_init(void* opt_state, void* stream)
{
    zs::clear_error();
    if (!opt_state)
        return fail(ZERO_ERR_INVALID_ARG, "zero_opt_state_init: null opt_state");
    if (!aligned(opt_state, 8))
        return fail(ZERO_ERR_ALIGNMENT, "zero_opt_state_init: opt_state must be 8-byte aligned");
    cudaError_t e = zs::launch_opt_init(static_cast<zero_opt_state*>(opt_state), 0.0f, 2.0f, 0.5f, 2000,
                                        static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ZERO_OK : cuda_fail(e, "zero_opt_state_init");
}

zero_status zero_opt_state_init_dynamic(void* opt_state, float initial_scale, float growth_factor,
                                        float backoff_factor, int32_t growth_interval, void* stream)
{
    zs::clear_error();
    if (!opt_state)
        return fail(ZERO_ERR_INVALID_ARG, "zero_opt_state_init_dynamic: null opt_state");
    if (!aligned(opt_state, 8))
        return fail(ZERO_ERR_ALIGNMENT, "zero_opt_state_init_dynamic: opt_state must be 8-byte aligned");
    if (!(initial_scale > 0.0f) || !std::isfinite(initial_scale) || !(growth_factor >= 1.0f) ||
        !std::isfinite(growth_factor) || !(backoff_factor > 0.0f && backoff_factor <= 1.0f) ||
        growth_interval < 1)
        return fail(ZERO_ERR_INVALID_ARG, "zero_opt_state_init_dynamic: need scale > 0, growth >= 1, "
                    "0 < backoff <= 1, interval >= 1");
    cudaError_t e = zs::launch_opt_init(static_cast<zero_opt_state*>(opt_state), initial_scale, growth_factor,
                                        backoff_factor, growth_interval, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ZERO_OK : cuda_fail(e, "zero_opt_state_init_dynamic");
}

zero_status zero_workspace_bytes(const zero_plan_t* plan, const zero_hparams* hp,
                                 const zero_step_args* args, size_t* bytes)
{
    zs::clear_error();
    if (!bytes)
        return fail(ZERO_ERR_INVALID_ARG, "zero_workspace_bytes: null bytes");
    zero_status s = validate(plan, hp, args);
    if (s != ZERO_OK)
        return s;
    *bytes = workspace_need(*hp, plan_launches(*plan, *hp, *args));
    return ZERO_OK;
}

// The step's kernel sequence.  PHASE_ALL is zero_shard_step; PHASE_BEGIN and
// PHASE_END are its two halves around the caller's reduction of the vote.
enum StepPhase { PHASE_ALL, PHASE_BEGIN, PHASE_END };

static zero_status run_step(const zero_plan_t* plan, const zero_hparams* hp, const zero_step_args* args,
                            void* stream, StepPhase phase)
{
    zs::clear_error();
    zero_status s = validate(plan, hp, args);
    if (s != ZERO_OK)
        return s;
    const zero_plan_s& p = *plan;
    const zero_hparams& h = *hp;
    const zero_step_args& a = *args;
    const LaunchPlan lp = plan_launches(p, h, a);
    const size_t need = workspace_need(h, lp);
    if (!a.workspace || a.workspace_bytes < need)
        return fail(ZERO_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                    a.workspace ? a.workspace_bytes : (size_t)0);
    if (!aligned(a.workspace, 256))
        return fail(ZERO_ERR_ALIGNMENT, "workspace must be 256-byte aligned");

    auto* st = static_cast<zero_opt_state*>(a.opt_state);
    auto* res = static_cast<zero_step_result*>(a.result);
    auto* ws = static_cast<zs::WsHeader*>(a.workspace);
    auto* partials = reinterpret_cast<double*>(static_cast<char*>(a.workspace) + zs::kHeaderBytes);
    cudaStream_t str = static_cast<cudaStream_t>(stream);
    auto* ev0 = static_cast<cudaEvent_t>(a.timing_events[0]);
    auto* ev1 = static_cast<cudaEvent_t>(a.timing_events[1]);

    zs::UpdateArgs u;
    std::memset(&u, 0, sizeof u);
    u.grads = static_cast<const uint16_t*>(a.grads);
    u.stash = a.grad_stash;
    for (int k = 0; k < 2; ++k) {
        u.master[k] = a.master[k];
        u.exp_avg[k] = a.exp_avg[k];
        u.exp_avg_sq[k] = a.exp_avg_sq[k];
    }
    u.params = static_cast<uint16_t*>(a.params);
    u.ws = ws;
    u.result = res;
    u.wait_budget = zs::wait_budget_cycles();
    u.bf16 = a.storage == ZERO_STORAGE_BF16 ? 1 : 0;
    u.nd = a.grad_layout == ZERO_GRADS_REDUCED ? 1 : p.nd; // contributions per element
    double scale = (double)h.loss_scale;
    if (h.average_over_nd)
        scale *= (double)p.nd;
    u.inv = (float)(1.0 / scale);
    u.lr = h.lr;
    u.beta1 = h.beta1;
    u.beta2 = h.beta2;
    u.eps = h.eps;
    // fp32 constants, each rounded once on the host
    u.lr_wd = h.lr * h.weight_decay;
    u.one_minus_beta1 = 1.0f - h.beta1;
    u.one_minus_beta2 = 1.0f - h.beta2;

    // peer tables: one gradient buffer per rank, extra parameter destinations
    zs::PeerTable peer_table;
    const zs::PeerTable* peers = make_peer_table(p, a, &peer_table);

    const bool spec = h.mode == ZERO_MODE_SPECULATIVE;
    const bool first_half = phase != PHASE_END;
    const bool second_half = phase != PHASE_BEGIN;
    cudaError_t e;
    const double scale_mult = h.average_over_nd ? (double)p.nd : 1.0;
    if (first_half && (e = zs::launch_prep(st, ws, h.beta1, h.beta2, u.inv, scale_mult, str)) != cudaSuccess)
        return cuda_fail(e, "prep launch");

    if (spec) {
        if (first_half) {
            if (ev0 && !zs::preparing() && (e = cudaEventRecord(ev0, str)) != cudaSuccess)
                return cuda_fail(e, "timing event");
            // Buckets are only the granularity at which gradients become
            // ready; nothing orders them inside one call, so the update walks
            // the whole range in as few launches as the segment table allows.
            for (const auto& l : lp.whole)
                if (l.count > 0 &&
                    (e = zs::launch_update(zs::kSrcGradsSpeculative, lp.vec, u, l, peers, str)) != cudaSuccess)
                    return cuda_fail(e, "update launch");
            if (ev1 && !zs::preparing() && (e = cudaEventRecord(ev1, str)) != cudaSuccess)
                return cuda_fail(e, "timing event");
            if (phase == PHASE_BEGIN && (e = zs::launch_vote_local(ws, partials, 0, str)) != cudaSuccess)
                return cuda_fail(e, "vote launch");
        }
        if (second_half) {
            if (phase == PHASE_END &&
                (e = zs::launch_vote_apply(ws, true, h.max_grad_norm, st, res, str)) != cudaSuccess)
                return cuda_fail(e, "vote launch");
            for (size_t i = 0; i < lp.whole.size(); ++i)
                if ((e = zs::launch_commit(lp.vec, u, lp.whole[i], i == 0, st, res, peers, str)) != cudaSuccess)
                    return cuda_fail(e, "commit launch");
        }
        return ZERO_OK;
    }

    // pre-pass modes: statistics bucket by bucket, decision, in-place update
    if (first_half) {
        zs::StatsArgs sa;
        sa.grads = u.grads;
        sa.stash = h.mode == ZERO_MODE_STASH ? a.grad_stash : nullptr;
        sa.ws = ws;
        sa.nd = u.nd;
        sa.inv = u.inv;
        sa.st = st;
        sa.scale_mult = scale_mult;
        sa.bf16 = u.bf16;
        int64_t n_partials = 0;
        for (const auto& b : lp.buckets) {
            for (const auto& l : b) {
                sa.partials = partials + n_partials;
                if ((e = zs::launch_stats(lp.vec, sa, l, peers, str)) != cudaSuccess)
                    return cuda_fail(e, "statistics launch");
                n_partials += zs::stats_blocks(lp.vec, l);
            }
        }
        if (phase == PHASE_ALL) {
            if ((e = zs::launch_finalize(ws, partials, n_partials, h.max_grad_norm, st, res, str)) != cudaSuccess)
                return cuda_fail(e, "finalize launch");
        } else if ((e = zs::launch_vote_local(ws, partials, n_partials, str)) != cudaSuccess) {
            return cuda_fail(e, "vote launch");
        }
    }
    if (second_half) {
        if (phase == PHASE_END &&
            (e = zs::launch_vote_apply(ws, false, h.max_grad_norm, st, res, str)) != cudaSuccess)
            return cuda_fail(e, "vote launch");
        const int src = h.mode == ZERO_MODE_STASH ? zs::kSrcStash : zs::kSrcGradsInPlace;
        if (ev0 && !zs::preparing() && (e = cudaEventRecord(ev0, str)) != cudaSuccess)
            return cuda_fail(e, "timing event");
        for (const auto& l : lp.whole)
            if (l.count > 0 && (e = zs::launch_update(src, lp.vec, u, l, peers, str)) != cudaSuccess)
                return cuda_fail(e, "update launch");
        if (ev1 && !zs::preparing() && (e = cudaEventRecord(ev1, str)) != cudaSuccess)
            return cuda_fail(e, "timing event");
    }
    return ZERO_OK;
}

zero_status zero_reduce_scatter(const zero_plan_t* plan, const zero_step_args* args, int64_t bucket,
                                void* grad_shards, void* stream)
{
    zs::clear_error();
    if (!plan || !args || !grad_shards)
        return fail(ZERO_ERR_INVALID_ARG, "zero_reduce_scatter: null plan, args or grad_shards");
    const zero_plan_s& p = *plan;
    const zero_step_args& a = *args;
    zero_status s = validate_source(&p, &a, false);
    if (s != ZERO_OK)
        return s;
    if (!aligned(grad_shards, 2))
        return fail(ZERO_ERR_ALIGNMENT, "grad_shards must be 2-byte aligned");
    const int64_t nb = p.bucket > 0 ? p.n_buckets : 1;
    if (bucket >= nb)
        return fail(ZERO_ERR_INVALID_ARG, "bucket %lld outside [0, %lld)", (long long)bucket, (long long)nb);
    const int64_t L = p.shard_len;
    int64_t lo = (int64_t)a.owner_first * L;
    int64_t hi = (int64_t)(a.owner_first + a.owner_count) * L;
    hi = hi < p.psi ? hi : p.psi;
    if (bucket >= 0 && p.bucket > 0) {
        lo = lo > bucket * p.bucket ? lo : bucket * p.bucket;
        hi = hi < (bucket + 1) * p.bucket ? hi : (bucket + 1) * p.bucket;
    }
    if (lo >= hi)
        return ZERO_OK;
    const int64_t stride = effective_stride(p, a);
    std::vector<zs::SegList> lists;
    segments_of(p, a.grad_layout, stride, a.owner_first, lo, hi, lists);
    bool vec = (L % 8 == 0) && (stride % 8 == 0) && aligned(grad_shards, 16) && segs_vec_ok(lists);
    if (a.peers) {
        for (int r = 0; r < p.nd; ++r)
            vec = vec && aligned(a.peers->rank_grads[r], 16);
    } else {
        vec = vec && aligned(a.grads, 16);
    }
    zs::PeerTable peer_table;
    const zs::PeerTable* peers = make_peer_table(p, a, &peer_table);
    for (const auto& l : lists) {
        cudaError_t e = zs::launch_reduce(vec, a.storage == ZERO_STORAGE_BF16, static_cast<const uint16_t*>(a.grads),
                                          static_cast<uint16_t*>(grad_shards), p.nd, l, peers,
                                          static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess)
            return cuda_fail(e, "reduce launch");
    }
    return ZERO_OK;
}

zero_status zero_shard_step(const zero_plan_t* plan, const zero_hparams* hp,
                            const zero_step_args* args, void* stream)
{
    return run_step(plan, hp, args, stream, PHASE_ALL);
}

zero_status zero_shard_step_begin(const zero_plan_t* plan, const zero_hparams* hp,
                                  const zero_step_args* args, void* stream)
{
    return run_step(plan, hp, args, stream, PHASE_BEGIN);
}

zero_status zero_shard_step_end(const zero_plan_t* plan, const zero_hparams* hp,
                                const zero_step_args* args, void* stream)
{
    return run_step(plan, hp, args, stream, PHASE_END);
}

zero_status zero_shard_step_prepare(const zero_plan_t* plan, const zero_hparams* hp,
                                    const zero_step_args* args)
{
    // the host logic of a whole step and of its two halves, each launch
    // replaced by loading its kernel (the geometry is cached on the way)
    zs::PrepareScope scope;
    zero_status s = run_step(plan, hp, args, nullptr, PHASE_ALL);
    if (s == ZERO_OK)
        s = run_step(plan, hp, args, nullptr, PHASE_BEGIN);
    if (s == ZERO_OK)
        s = run_step(plan, hp, args, nullptr, PHASE_END);
    return s;
}

// Launches copies of shard pieces, at most kMaxSegs per launch; compact
// (small, reused layer buffers) copies use evict-first stores.
static zero_status launch_pieces(std::vector<zs::GatherEntry>& entries, uint16_t* dst, bool compact,
                                 cudaStream_t str, const char* what)
{
    for (size_t i = 0; i < entries.size(); i += zs::kMaxSegs) {
        zs::GatherList g;
        std::memset(&g, 0, sizeof g);
        for (size_t k = i; k < entries.size() && g.count < zs::kMaxSegs; ++k)
            g.e[g.count++] = entries[k];
        cudaError_t e = zs::launch_gather(dst, g, compact, str);
        if (e != cudaSuccess)
            return cuda_fail(e, what);
    }
    return ZERO_OK;
}

static zs::GatherEntry piece(const void* src, int64_t src_off, const void* dst, int64_t dst_off, int64_t n)
{
    const uint16_t* s = static_cast<const uint16_t*>(src) + src_off;
    const uint16_t* d = static_cast<const uint16_t*>(dst) + dst_off;
    return zs::GatherEntry{s, dst_off, n, (aligned(s, 16) && aligned(d, 16)) ? 1 : 0};
}

zero_status zero_gather_params(const zero_plan_t* plan, const void* const* shard_ptrs,
                               void* params_full, void* stream)
{
    zs::clear_error();
    if (!plan || !shard_ptrs || !params_full)
        return fail(ZERO_ERR_INVALID_ARG, "zero_gather_params: null argument");
    const zero_plan_s& p = *plan;
    if (!aligned(params_full, 2))
        return fail(ZERO_ERR_ALIGNMENT, "zero_gather_params: params_full must be 2-byte aligned");
    std::vector<zs::GatherEntry> entries;
    for (int32_t r = 0; r < p.nd; ++r) {
        if (!shard_ptrs[r])
            continue;
        if (!aligned(shard_ptrs[r], 2))
            return fail(ZERO_ERR_ALIGNMENT, "zero_gather_params: shard %d must be 2-byte aligned", r);
        const int64_t start = (int64_t)r * p.shard_len;
        int64_t n = p.psi - start;
        n = n < 0 ? 0 : (n > p.shard_len ? p.shard_len : n);
        if (n > 0)
            entries.push_back(piece(shard_ptrs[r], 0, params_full, start, n));
    }
    return launch_pieces(entries, static_cast<uint16_t*>(params_full), false, static_cast<cudaStream_t>(stream),
                         "gather launch");
}

// The pieces (owner shard range -> destination offset) of a tensor range.
static zero_status tensor_pieces(const zero_plan_t* plan, int32_t first_tensor, int32_t n_tensors,
                                 const void* const* shard_ptrs, void* out, int32_t compact, const char* who,
                                 std::vector<zs::GatherEntry>* entries, int64_t* n_elems)
{
    if (!plan || !shard_ptrs || !out)
        return fail(ZERO_ERR_INVALID_ARG, "%s: null argument", who);
    const zero_plan_s& p = *plan;
    const int32_t nt = (int32_t)p.tensor_offset.size() - 1;
    if (nt < 1)
        return fail(ZERO_ERR_INVALID_ARG, "%s: the plan was built without a tensor list", who);
    if (first_tensor < 0 || n_tensors < 0 || first_tensor > nt - n_tensors)
        return fail(ZERO_ERR_INVALID_ARG, "%s: tensors [%d, %d + %d) outside [0, %d)", who,
                    first_tensor, first_tensor, n_tensors, nt);
    if (compact != 0 && compact != 1)
        return fail(ZERO_ERR_INVALID_ARG, "%s: compact must be 0 or 1", who);
    if (!aligned(out, 2))
        return fail(ZERO_ERR_ALIGNMENT, "%s: out must be 2-byte aligned", who);
    const int64_t base = p.tensor_offset[(size_t)first_tensor];
    *n_elems = 0;
    for (const zero_segment& sg : p.segments) {
        if (sg.tensor < first_tensor || sg.tensor >= first_tensor + n_tensors)
            continue;
        const void* sh = shard_ptrs[sg.owner];
        const int64_t flat = p.tensor_offset[(size_t)sg.tensor] + sg.offset_in_tensor;
        if (!sh) {
            if (compact)
                return fail(ZERO_ERR_INVALID_ARG, "%s: tensor %lld needs owner %lld's shard", who,
                            (long long)sg.tensor, (long long)sg.owner);
            continue; // in place: this owner's part is already there
        }
        if (!aligned(sh, 2))
            return fail(ZERO_ERR_ALIGNMENT, "%s: shard %lld must be 2-byte aligned", who, (long long)sg.owner);
        entries->push_back(piece(sh, sg.offset_in_shard, out, compact ? flat - base : flat, sg.length));
        *n_elems += sg.length;
    }
    return ZERO_OK;
}

zero_status zero_gather_tensors(const zero_plan_t* plan, int32_t first_tensor, int32_t n_tensors,
                                const void* const* shard_ptrs, void* out, int32_t compact,
                                int64_t* elements, void* stream)
{
    zs::clear_error();
    std::vector<zs::GatherEntry> entries;
    int64_t n_elems = 0;
    zero_status s = tensor_pieces(plan, first_tensor, n_tensors, shard_ptrs, out, compact, "zero_gather_tensors",
                                  &entries, &n_elems);
    if (s != ZERO_OK)
        return s;
    if (elements)
        *elements = n_elems;
    return launch_pieces(entries, static_cast<uint16_t*>(out), compact != 0, static_cast<cudaStream_t>(stream),
                         "gather launch");
}

zero_status zero_gather_tensors_dma(const zero_plan_t* plan, int32_t first_tensor, int32_t n_tensors,
                                    const void* const* shard_ptrs, void* out, int32_t compact,
                                    int64_t* elements, void* stream)
{
    zs::clear_error();
    std::vector<zs::GatherEntry> entries;
    int64_t n_elems = 0;
    zero_status s = tensor_pieces(plan, first_tensor, n_tensors, shard_ptrs, out, compact,
                                  "zero_gather_tensors_dma", &entries, &n_elems);
    if (s != ZERO_OK)
        return s;
    if (elements)
        *elements = n_elems;
    // pieces that continue each other in both the shard and the destination
    // (consecutive tensors of one owner) move as one copy
    uint16_t* dst = static_cast<uint16_t*>(out);
    cudaStream_t str = static_cast<cudaStream_t>(stream);
    for (size_t i = 0; i < entries.size();) {
        const uint16_t* src = entries[i].src;
        const int64_t off = entries[i].dst_off;
        int64_t n = entries[i].n;
        size_t j = i + 1;
        while (j < entries.size() && entries[j].src == src + n && entries[j].dst_off == off + n)
            n += entries[j++].n;
        const cudaError_t e = cudaMemcpyAsync(dst + off, src, (size_t)n * 2, cudaMemcpyDeviceToDevice, str);
        if (e != cudaSuccess)
            return cuda_fail(e, "zero_gather_tensors_dma copy");
        i = j;
    }
    return ZERO_OK;
}

zero_status zero_cast_params(const zero_plan_t* plan, const float* master, void* params,
                             int32_t owner_first, int32_t owner_count, int32_t storage, void* stream)
{
    zs::clear_error();
    if (!plan || !master || !params)
        return fail(ZERO_ERR_INVALID_ARG, "zero_cast_params: null argument");
    if (storage != ZERO_STORAGE_FP16 && storage != ZERO_STORAGE_BF16)
        return fail(ZERO_ERR_INVALID_ARG, "zero_cast_params: unknown 16-bit storage format %d", storage);
    const zero_plan_s& p = *plan;
    if (owner_first < 0 || owner_count < 1 || owner_first > p.nd - owner_count)
        return fail(ZERO_ERR_INVALID_ARG, "zero_cast_params: owner range outside the plan");
    if (!aligned(master, 4) || !aligned(params, 2))
        return fail(ZERO_ERR_ALIGNMENT, "zero_cast_params: misaligned buffer");
    const int64_t lo = (int64_t)owner_first * p.shard_len;
    int64_t hi = (int64_t)(owner_first + owner_count) * p.shard_len;
    hi = hi > p.psi ? p.psi : hi;
    std::vector<zs::SegList> lists;
    segments_of(p, ZERO_GRADS_FULL, 0, owner_first, lo, hi, lists);
    const bool vec = (p.shard_len % 8 == 0) && aligned(master, 16) && aligned(params, 16) &&
                     segs_vec_ok(lists);
    for (const auto& l : lists) {
        cudaError_t e = zs::launch_cast(vec, storage == ZERO_STORAGE_BF16, master, static_cast<uint16_t*>(params), l,
                                        static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess)
            return cuda_fail(e, "cast launch");
    }
    return ZERO_OK;
}

} // extern "C"
