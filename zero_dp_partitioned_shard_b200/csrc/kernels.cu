// kernels.cu -- sm_100a kernels of libzero_shard.so.
//
// The step is HBM-bound streaming work (about 20 fp32 operations, one square
// root and three divisions per parameter against 2*Nd + 26 bytes), so it uses
// no tensor cores.  The update runs as a bulk-copy pipeline (warp-specialised:
// one producer warp streams tiles into a shared-memory ring with
// cp.async.bulk -- for more than 16 contributions as 2-D tensor-map boxes of
// all rank rows -- and eight consumer warps compute from it; for 5 to 11
// contributions the results go back through the ring and leave by the
// producer's bulk stores) for up to 64 contributions (16 through peer
// tables) and for the stash, and on the register path below otherwise.
// Design points of the register path, which the statistics, reduce, commit
// and cast kernels share:
//   * one thread owns 8 consecutive parameters per iteration: every access is
//     a 16-byte vector (fp16 x8 or fp32 x4) and a warp touches 512 contiguous
//     bytes of each stream; loads bypass L1 and are marked evict-first, since
//     every byte is read exactly once;
//   * the Nd rank contributions of a chunk are loaded in groups of 8 before
//     any is added, so up to 8 * 16 B of gradient plus 96 B of optimizer state
//     are in flight per thread; the adds then run in rank order;
//   * persistent grid-stride launches sized to (SM count x resident blocks);
//   * the overflow flag is a warp vote followed by one atomicOr per warp that
//     saw a non-finite value; the fp64 norm partials are reduced per block in a
//     fixed shuffle pattern and summed in a fixed order by a one-block kernel,
//     so results are bit-reproducible for a given launch geometry.
// No kernel waits on another block, a flag or a peer: ordering between the
// kernels of a step is plain stream order.  With peer tables the same kernels
// load the contributions from each rank's own buffer (possibly another GPU's
// memory) and store every new parameter into each rank's parameter buffer:
// the reduce-scatter and the all-gather ride on the update's own loads and
// stores.
//
// Arithmetic per parameter (ZeRO leaves the optimizer's maths unchanged; the
// pages name Adam with fp32 master, momentum and variance -- "ZeRO memory
// optimization: training large models", trishampatil.com, "The Real Problem"
// -- and the equations are the textbook Adam/AdamW of Kingma & Ba 2015, Alg. 1
// and Loshchilov & Hutter 2019): every fp32 operation is an explicitly rounded
// intrinsic (no contraction into FMA), division and square root are the
// IEEE-rounded __fdiv_rn / __fsqrt_rn, and the fp16 cast is round-to-nearest-
// even with subnormals kept.
#include <cuda.h> // CUtensorMap and the tensor-map encoder's types (the encoder is looked up at run time)
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <map>
#include <mutex>
#include <type_traits>
#include <unordered_map>
#include <utility>

#include "zs_internal.h"
#include "zs_launch.h"

namespace zs {

// ---------------------------------------------------------------------------
// device helpers
// ---------------------------------------------------------------------------

struct AdamK {
    float beta1, beta2, omb1, omb2, lr, lr_wd, eps, bc1, bc2, clip;
};

// m = b1*m + (1-b1)*g; v = b2*v + (1-b2)*g^2;
// p = (p - lr_wd*p) - lr * ((m/bc1) / (sqrt(v/bc2) + eps))
__device__ __forceinline__ void adam_update(float g, float& p, float& m, float& v, const AdamK& k)
{
    const float m_new = __fadd_rn(__fmul_rn(k.beta1, m), __fmul_rn(k.omb1, g));
    const float v_new = __fadd_rn(__fmul_rn(k.beta2, v), __fmul_rn(k.omb2, __fmul_rn(g, g)));
    const float m_hat = __fdiv_rn(m_new, k.bc1);
    const float v_hat = __fdiv_rn(v_new, k.bc2);
    const float denom = __fadd_rn(__fsqrt_rn(v_hat), k.eps);
    const float step = __fmul_rn(k.lr, __fdiv_rn(m_hat, denom));
    p = __fsub_rn(__fsub_rn(p, __fmul_rn(k.lr_wd, p)), step);
    m = m_new;
    v = v_new;
}

// 16-bit storage formats: BF = false is IEEE binary16, BF = true is
// bfloat16 (the upper half of a binary32, so widening is a shift).  Narrowing
// rounds to nearest even in both.
template <bool BF>
__device__ __forceinline__ void unpack_h8(const uint4& x, float f[8])
{
    if (BF) {
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            f[2 * q] = __uint_as_float(w[q] << 16);
            f[2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
        }
    } else {
        const __half2* h = reinterpret_cast<const __half2*>(&x);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 t = __half22float2(h[q]);
            f[2 * q] = t.x;
            f[2 * q + 1] = t.y;
        }
    }
}

template <bool BF>
__device__ __forceinline__ uint32_t pack_h2(float a, float b)
{
    if (BF) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&h);
    }
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

template <bool BF>
__device__ __forceinline__ uint4 pack_h8(const float f[8])
{
    return make_uint4(pack_h2<BF>(f[0], f[1]), pack_h2<BF>(f[2], f[3]), pack_h2<BF>(f[4], f[5]),
                      pack_h2<BF>(f[6], f[7]));
}

__device__ __forceinline__ uint4 ld_stream(const uint16_t* p)
{
    return __ldcs(reinterpret_cast<const uint4*>(p));
}

__device__ __forceinline__ void ld_f8(const float* p, float f[8])
{
    const float4 a = __ldcs(reinterpret_cast<const float4*>(p));
    const float4 b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

__device__ __forceinline__ void st_f8(float* p, const float f[8])
{
    __stcs(reinterpret_cast<float4*>(p), make_float4(f[0], f[1], f[2], f[3]));
    __stcs(reinterpret_cast<float4*>(p) + 1, make_float4(f[4], f[5], f[6], f[7]));
}

template <bool BF>
__device__ __forceinline__ float h2f(uint16_t h)
{
    return BF ? __uint_as_float((uint32_t)h << 16) : __half2float(__ushort_as_half(h));
}

template <bool BF>
__device__ __forceinline__ uint16_t f2h(float f)
{
    return BF ? __bfloat16_as_ushort(__float2bfloat16_rn(f)) : __half_as_ushort(__float2half_rn(f));
}

// Where rank r's contributions to a run of elements start: the rank buffers
// side by side at a fixed stride (one process holding the whole group), or one
// buffer per rank through the peer table (each possibly another GPU's memory,
// reached by plain loads over NVLink).
struct StridedRanks {
    const uint16_t* g;
    int64_t rstride;
    __device__ __forceinline__ const uint16_t* at(int r) const { return g + (int64_t)r * rstride; }
};

struct TableRanks {
    const uint16_t* const* tbl;
    int64_t off;
    __device__ __forceinline__ const uint16_t* at(int r) const { return tbl[r] + off; }
};

struct NoPeers {};
template <bool PEER>
using PeerParam = typename std::conditional<PEER, PeerTable, NoPeers>::type;

template <bool PEER>
__device__ __forceinline__ auto ranks_at(const uint16_t* grads, const PeerParam<PEER>& pt, const Seg& sg, int64_t e)
{
    if constexpr (PEER)
        return TableRanks{pt.grads, sg.g_off + e};
    else
        return StridedRanks{grads + sg.g_off + e, sg.g_rstride};
}

// New parameters go to params and, with peer tables, to every other rank's
// parameter buffer as well (the all-gather as stores).
template <bool PEER>
__device__ __forceinline__ void store_params8(uint16_t* params, const PeerParam<PEER>& pt, int64_t off, uint4 v)
{
    __stcs(reinterpret_cast<uint4*>(params + off), v);
    if constexpr (PEER)
        for (int d = 0; d < pt.n_dests; ++d)
            __stcs(reinterpret_cast<uint4*>(pt.dests[d] + off), v);
}

template <bool PEER>
__device__ __forceinline__ void store_param1(uint16_t* params, const PeerParam<PEER>& pt, int64_t off, uint16_t v)
{
    params[off] = v;
    if constexpr (PEER)
        for (int d = 0; d < pt.n_dests; ++d)
            pt.dests[d][off] = v;
}

// Rank-order sum of the Nd contributions of 8 consecutive parameters: the
// loads of the first G ranks are issued together, then those of each further
// group of 8, and every group is added in rank order.  G = 8 suits the update
// kernel, which also holds master/m/v in registers; the statistics pass has
// the registers to keep all 16 contributions of a 16-rank step in flight
// (measured 1.00 of the copy bandwidth against 0.94-0.97 with G = 8).
template <bool BF, int G = 8, class Ranks>
__device__ __forceinline__ void rank_sum8(const Ranks& rk, int nd, float s[8])
{
    {
        uint4 x[G];
#pragma unroll
        for (int u = 0; u < G; ++u)
            if (u < nd)
                x[u] = ld_stream(rk.at(u));
        unpack_h8<BF>(x[0], s);
#pragma unroll
        for (int u = 1; u < G; ++u) {
            if (u < nd) {
                float f[8];
                unpack_h8<BF>(x[u], f);
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    s[q] = __fadd_rn(s[q], f[q]);
            }
        }
    }
    for (int r = G; r < nd; r += 8) {
        uint4 x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (r + u < nd)
                x[u] = ld_stream(rk.at(r + u));
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            if (r + u < nd) {
                float f[8];
                unpack_h8<BF>(x[u], f);
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    s[q] = __fadd_rn(s[q], f[q]);
            }
        }
    }
}

template <bool BF, class Ranks>
__device__ __forceinline__ float rank_sum1(const Ranks& rk, int nd)
{
    float s = h2f<BF>(rk.at(0)[0]);
    for (int r = 1; r < nd; ++r)
        s = __fadd_rn(s, h2f<BF>(rk.at(r)[0]));
    return s;
}

// Programmatic dependent launch (stream-ordered, no flags): a kernel launched
// with programmatic serialization may start while its predecessor in the
// stream drains; griddepcontrol.wait returns once that predecessor has
// completed and its writes are visible.  Both are no-ops for a kernel
// launched without the attribute.
__device__ __forceinline__ void wait_for_predecessor() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void flag_nonfinite(bool bad, unsigned int* flag)
{
    // every lane of the warp reaches this point (grid-stride loops only)
    const unsigned int any = __ballot_sync(0xffffffffu, bad);
    if (any && (threadIdx.x & 31) == 0)
        atomicOr(flag, 1u);
}

// Walks this thread's share of a launch: the 8-element chunks of every
// segment as one index space (segments back to back, grid-stride, so a launch
// over many short segments keeps the whole grid busy instead of ending each
// segment in a partial wave), then the < 8-element tail of each segment on
// the lowest thread ids.  Without VEC every element is a scalar unit.
template <bool VEC, typename ChunkFn, typename ElemFn>
__device__ __forceinline__ void walk_segments(const SegList& segs, ChunkFn&& chunk, ElemFn&& elem)
{
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t nthr = (int64_t)gridDim.x * blockDim.x;
    const int shift = VEC ? 3 : 0;
    int64_t total = 0;
    for (int s = 0; s < segs.count; ++s)
        total += segs.seg[s].n >> shift;
    int si = 0;
    int64_t base = 0;
    for (int64_t u = tid; u < total; u += nthr) {
        while (u >= base + (segs.seg[si].n >> shift)) {
            base += segs.seg[si].n >> shift;
            ++si;
        }
        if (VEC)
            chunk(segs.seg[si], (u - base) << 3);
        else
            elem(segs.seg[si], u - base);
    }
    if (VEC) {
        for (int s = 0; s < segs.count; ++s) {
            const Seg& sg = segs.seg[s];
            const int64_t e = ((sg.n >> 3) << 3) + tid;
            if (e < sg.n)
                elem(sg, e);
        }
    }
}

// Unscale factor of a step: fp32 1/(S [* Nd]) with S the dynamic loss scale
// when one is in use (computed exactly as the host computes the static one).
__device__ __forceinline__ float step_inv(const zero_opt_state* st, float static_inv, double scale_mult)
{
    const float S = st->loss_scale;
    return S > 0.0f ? __double2float_rn(__ddiv_rn(1.0, __dmul_rn((double)S, scale_mult))) : static_inv;
}

// Dynamic loss scaling after a step (nothing when static): back off on a
// skipped step, grow after growth_interval consecutive applied steps.
__device__ __forceinline__ void advance_loss_scale(zero_opt_state* st, bool skipped)
{
    if (!(st->loss_scale > 0.0f))
        return;
    if (skipped) {
        st->loss_scale = __fmul_rn(st->loss_scale, st->backoff_factor);
        st->good_steps = 0;
    } else if (++st->good_steps >= st->growth_interval) {
        st->loss_scale = __fmul_rn(st->loss_scale, st->growth_factor);
        st->good_steps = 0;
    }
}

// The clip coefficient is 1 when the step has no pre-pass (speculative): the
// update kernels then skip the multiply by it, which would change no value.
__device__ __forceinline__ AdamK load_consts(const UpdateArgs& a, const WsHeader* ws, bool clip)
{
    AdamK k;
    k.beta1 = a.beta1;
    k.beta2 = a.beta2;
    k.omb1 = a.one_minus_beta1;
    k.omb2 = a.one_minus_beta2;
    k.lr = a.lr;
    k.lr_wd = a.lr_wd;
    k.eps = a.eps;
    k.bc1 = ws->bc1;
    k.bc2 = ws->bc2;
    k.clip = clip ? ws->clip : 1.0f;
    return k;
}

// ---------------------------------------------------------------------------
// K0: optimizer-state init and per-step prep (one thread)
// ---------------------------------------------------------------------------

__global__ void zs_opt_init_kernel(zero_opt_state* st, float scale, float growth, float backoff, int32_t interval)
{
    st->t = 0;
    st->beta1_pow = 1.0;
    st->beta2_pow = 1.0;
    st->skipped = 0;
    st->cur = 0;
    st->reserved = 0;
    st->loss_scale = scale; // 0: static scaling
    st->good_steps = 0;
    st->growth_factor = growth;
    st->backoff_factor = backoff;
    st->growth_interval = interval;
    st->reserved2 = 0;
}

// Bias corrections of the step about to be applied, from the fp64 running
// products beta^t: bc = (fp32)(1 - beta^(t+1)).
__global__ void zs_prep_kernel(const zero_opt_state* st, WsHeader* ws, float beta1, float beta2, float static_inv,
                               double scale_mult)
{
    ws->inv = step_inv(st, static_inv, scale_mult); // the update kernels' unscale factor
    const double b1 = __dmul_rn(st->beta1_pow, (double)beta1);
    const double b2 = __dmul_rn(st->beta2_pow, (double)beta2);
    ws->overflow = 0u;
    ws->error = 0u;
    ws->skip = 0;
    ws->cur = st->cur & 1;
    ws->bc1 = __double2float_rn(__dsub_rn(1.0, b1));
    ws->bc2 = __double2float_rn(__dsub_rn(1.0, b2));
    ws->clip = 1.0f;
    ws->b1p_next = b1;
    ws->b2p_next = b2;
    ws->sumsq = 0.0;
    ws->norm = __longlong_as_double(0x7ff8000000000000LL);
    ws->t_next = st->t + 1;
}

// ---------------------------------------------------------------------------
// K1: fused reduce + unscale (+ overflow) + clip + Adam + fp16 cast
// ---------------------------------------------------------------------------

// One element, scalar loads and stores; returns true if its gradient is not
// finite (only meaningful when the reduced gradient is computed here).
template <int SRC, bool BF, bool PEER>
__device__ __forceinline__ bool update_scalar(const UpdateArgs& a, const PeerParam<PEER>& pt, const Seg& sg,
                                              int64_t e, const AdamK& k, float inv, const float* p_in,
                                              const float* m_in, const float* v_in, float* p_out, float* m_out,
                                              float* v_out)
{
    const int64_t so = sg.s_off + e;
    float g;
    if (SRC == kSrcStash)
        g = a.stash[so];
    else
        g = __fmul_rn(rank_sum1<BF>(ranks_at<PEER>(a.grads, pt, sg, e), a.nd), inv);
    float p = p_in[so], m = m_in[so], v = v_in[so];
    adam_update(SRC == kSrcGradsSpeculative ? g : __fmul_rn(g, k.clip), p, m, v, k);
    p_out[so] = p;
    m_out[so] = m;
    v_out[so] = v;
    store_param1<PEER>(a.params, pt, sg.p_off + e, f2h<BF>(p));
    return !isfinite(g);
}

template <int SRC, bool VEC, bool BF, bool PEER>
__global__ void __launch_bounds__(kThreads, 2)
zs_update_kernel(const UpdateArgs a, const __grid_constant__ SegList segs, const __grid_constant__ PeerParam<PEER> pt)
{
    constexpr bool kSpec = SRC == kSrcGradsSpeculative;
    wait_for_predecessor(); // bias corrections, slot, skip and clip come from the kernels before
    allow_dependents();
    const WsHeader* ws = a.ws;
    if (!kSpec && ws->skip)
        return; // uniform across the grid: the whole step is skipped
    const int cur = kSpec ? ws->cur : 0;
    const int nxt = kSpec ? cur ^ 1 : 0;
    const AdamK k = load_consts(a, ws, !kSpec);
    const float inv = ws->inv;
    // slot selection by value: indexing the parameter arrays with a runtime
    // index would force a local-memory copy of the whole argument struct
    const float* __restrict__ p_in = cur ? a.master[1] : a.master[0];
    const float* __restrict__ m_in = cur ? a.exp_avg[1] : a.exp_avg[0];
    const float* __restrict__ v_in = cur ? a.exp_avg_sq[1] : a.exp_avg_sq[0];
    float* p_out = nxt ? a.master[1] : a.master[0];
    float* m_out = nxt ? a.exp_avg[1] : a.exp_avg[0];
    float* v_out = nxt ? a.exp_avg_sq[1] : a.exp_avg_sq[0];

    bool bad = false;
    walk_segments<VEC>(
        segs,
        [&](const Seg& sg, int64_t e) {
            const int64_t so = sg.s_off + e;
            float p[8], m[8], v[8], g[8];
            ld_f8(p_in + so, p);
            ld_f8(m_in + so, m);
            ld_f8(v_in + so, v);
            if (SRC == kSrcStash) {
                ld_f8(a.stash + so, g);
            } else {
                rank_sum8<BF>(ranks_at<PEER>(a.grads, pt, sg, e), a.nd, g);
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    g[q] = __fmul_rn(g[q], inv);
            }
            if (kSpec) {
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    bad |= !isfinite(g[q]);
            }
#pragma unroll
            for (int q = 0; q < 8; ++q)
                adam_update(kSpec ? g[q] : __fmul_rn(g[q], k.clip), p[q], m[q], v[q], k);
            st_f8(p_out + so, p);
            st_f8(m_out + so, m);
            st_f8(v_out + so, v);
            store_params8<PEER>(a.params, pt, sg.p_off + e, pack_h8<BF>(p));
        },
        [&](const Seg& sg, int64_t e) {
            bad |= update_scalar<SRC, BF, PEER>(a, pt, sg, e, k, inv, p_in, m_in, v_in, p_out, m_out, v_out);
        });
    if (kSpec)
        flag_nonfinite(bad, &a.ws->overflow);
}

// ---------------------------------------------------------------------------
// K1, bulk-copy pipeline: the same per-element arithmetic, with the operands
// staged through shared memory.  One producer thread streams each tile of
// master/m/v and of the Nd rank contributions (or the stash) into a ring of
// shared-memory stages with 1-D cp.async.bulk copies that complete on an
// mbarrier; eight consumer warps wait for a stage, compute from shared memory,
// store straight to global memory and release the stage.  Loads in flight no
// longer depend on registers or occupancy: (stages - 1) tiles per CTA are
// always on their way.  Every wait is bounded; a wait that expires sets the
// workspace error word and the result's status, and the kernel exits after
// waiting (bounded) for its own copies.
// ---------------------------------------------------------------------------

constexpr int kPipeConsumerWarps = 8;
constexpr int kPipeConsumers = kPipeConsumerWarps * 32;
constexpr int kPipeThreads = kPipeConsumers + 32; // + the producer warp
constexpr long long kDrainBudgetCycles = 1ll << 31; // ~1 s: far beyond any memory latency
constexpr int kPipeHeaderBytes = 1024;           // mbarriers + tile table, before the ring

__device__ __forceinline__ uint32_t smem_addr(const void* p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok)
                 : "r"(smem_addr(bar)), "r"(parity)
                 : "memory");
    return ok != 0;
}

// Wait for the phase of the given parity; false if `budget` cycles ran out
// (a negative budget expires at once).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, long long budget)
{
    if (budget < 0)
        return false;
    if (mbar_test(bar, parity))
        return true;
    const long long t0 = clock64();
    while (!mbar_test(bar, parity))
        if (clock64() - t0 > budget)
            return false;
    return true;
}

// L2 policy of the 1-D pipeline's copies: evict first, like its streaming
// stores.  Each byte is read once, so the lines it would keep in L2 are better
// left to the dirty lines of the stores.  Measured on one B200 against the
// default policy: GPT-2 1.5B-shaped Nd = 8 update 0.970-0.972 -> 0.974-0.975
// of the copy bandwidth, and the 24-layer clip step (stash mode) 13.58 ->
// 13.37-13.39 ms; with plain stores instead of evict-first ones the same
// policy cost 3 % everywhere.  The tensor-map instantiations keep the default
// policy: with evict-first copies Nd = 64 fell from 1.01-1.03 to 0.90-0.91.
__device__ __forceinline__ uint64_t evict_first_policy()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// global -> shared bulk copy of `bytes` (multiple of 16, both ends 16-byte
// aligned) completing as transaction bytes on `bar`; with HINT under L2 policy
// `pol`, else under the default policy.  No multicast.
template <bool HINT>
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar, uint64_t pol)
{
    if constexpr (HINT)
        asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
                     " [%0], [%1], %2, [%3], %4;"
                     ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(pol)
                     : "memory");
    else
        asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                     ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar))
                     : "memory");
}

// global -> shared copy of one box of a 2-D tensor map (the box's top-left
// element at column x, row y) completing as transaction bytes on `bar`.  The
// whole box always lands in shared memory; elements past the map's extent
// arrive as zeros.  x * 2 bytes must be a multiple of 16 (the host checks it
// before the launch).  No multicast.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int32_t x, int32_t y, uint64_t* bar)
{
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3}], [%4];"
                 ::"r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
                 : "memory");
}

// shared -> global bulk copy of `bytes` (multiple of 16, both ends 16-byte
// aligned) under L2 policy `pol`, tracked by the issuing thread's bulk-async
// groups.
__device__ __forceinline__ void bulk_store(void* dst, const void* src, uint32_t bytes, uint64_t pol)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group.L2::cache_hint [%0], [%1], %2, %3;"
                 ::"l"(dst), "r"(smem_addr(src)), "r"(bytes), "l"(pol)
                 : "memory");
}

template <int N>
__device__ __forceinline__ void sts_f(float* p, const float f[N])
{
    if (N == 8) {
        reinterpret_cast<float4*>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
        reinterpret_cast<float4*>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
    } else if (N == 4) {
        *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
    } else if (N == 2) {
        *reinterpret_cast<float2*>(p) = make_float2(f[0], f[1]);
    } else {
        p[0] = f[0];
    }
}

template <int N, bool BF>
__device__ __forceinline__ void sts_h(uint16_t* p, const float f[N])
{
    if (N == 8) {
        *reinterpret_cast<uint4*>(p) = pack_h8<BF>(f);
    } else if (N == 4) {
        *reinterpret_cast<uint2*>(p) = make_uint2(pack_h2<BF>(f[0], f[1]), pack_h2<BF>(f[2], f[3]));
    } else if (N == 2) {
        *reinterpret_cast<unsigned int*>(p) = pack_h2<BF>(f[0], f[1]);
    } else {
        p[0] = f2h<BF>(f[0]);
    }
}

// The tensor map of a pipelined launch that moves the rank rows of a tile
// with 2-D copies (TM), or nothing.
struct NoMap {};
template <bool TM>
using TmapParam = typename std::conditional<TM, CUtensorMap, NoMap>::type;
constexpr int kBoxCols = 256; // columns (elements) of one 2-D box; a tile of T elements takes T / 256 boxes

template <int N>
__device__ __forceinline__ void lds_f(const float* p, float f[N])
{
    if (N == 8) {
        const float4 x = reinterpret_cast<const float4*>(p)[0];
        const float4 y = reinterpret_cast<const float4*>(p)[1];
        f[0] = x.x; f[1] = x.y; f[2] = x.z; f[3] = x.w;
        f[4] = y.x; f[5] = y.y; f[6] = y.z; f[7] = y.w;
    } else if (N == 4) {
        const float4 x = *reinterpret_cast<const float4*>(p);
        f[0] = x.x; f[1] = x.y; f[2] = x.z; f[3] = x.w;
    } else if (N == 2) {
        const float2 x = *reinterpret_cast<const float2*>(p);
        f[0] = x.x; f[1] = x.y;
    } else {
        f[0] = p[0];
    }
}

template <int N, bool BF>
__device__ __forceinline__ void lds_h(const uint16_t* p, float f[N])
{
    if (N == 8) {
        unpack_h8<BF>(*reinterpret_cast<const uint4*>(p), f);
    } else if (N == 4) {
        const uint2 x = *reinterpret_cast<const uint2*>(p);
        const uint32_t w[2] = {x.x, x.y};
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            f[2 * q] = h2f<BF>((uint16_t)(w[q] & 0xFFFFu));
            f[2 * q + 1] = h2f<BF>((uint16_t)(w[q] >> 16));
        }
    } else if (N == 2) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
        f[0] = h2f<BF>((uint16_t)(w & 0xFFFFu));
        f[1] = h2f<BF>((uint16_t)(w >> 16));
    } else {
        f[0] = h2f<BF>(p[0]);
    }
}

template <int N>
__device__ __forceinline__ void stg_f(float* p, const float f[N])
{
    if (N == 8)
        st_f8(p, f);
    else if (N == 4)
        __stcs(reinterpret_cast<float4*>(p), make_float4(f[0], f[1], f[2], f[3]));
    else if (N == 2)
        __stcs(reinterpret_cast<float2*>(p), make_float2(f[0], f[1]));
    else
        __stcs(p, f[0]);
}

template <int N, bool BF>
__device__ __forceinline__ void stg_h(uint16_t* p, const float f[N])
{
    if (N == 8) {
        __stcs(reinterpret_cast<uint4*>(p), pack_h8<BF>(f));
    } else if (N == 4) {
        __stcs(reinterpret_cast<uint2*>(p), make_uint2(pack_h2<BF>(f[0], f[1]), pack_h2<BF>(f[2], f[3])));
    } else if (N == 2) {
        __stcs(reinterpret_cast<unsigned int*>(p), pack_h2<BF>(f[0], f[1]));
    } else {
        p[0] = f2h<BF>(f[0]);
    }
}

// Segment of tile g, through the per-CTA tile table.  A thread's tiles only
// move forward (g += gridDim.x), so it keeps the segment of its previous tile
// and advances from there: over a whole launch at most `count` steps, instead
// of a scan of the table per tile (which, with one segment per owner of a
// 64-owner call and 256-element tiles, cost as much as the arithmetic).
__device__ __forceinline__ int next_tile_segment(const int64_t* first_tile, int count, int64_t g, int si)
{
    while (si + 1 < count && g >= first_tile[si + 1])
        ++si;
    return si;
}

// TM: the Nd rank rows of a tile arrive as T / 256 two-dimensional boxes of
// [256 columns x Nd rows] from a tensor map over the contributions (one copy
// per box instead of one per rank); in shared memory box b holds rank r's
// columns at (b * Nd + r) * 256.  Without TM each rank row is one 1-D copy
// and rank r's row starts at r * T.
// BST: the consumers write a tile's results into the stage -- master/m/v over
// their own input slots, the 16-bit parameters into a region of T * 2 bytes
// after the source rows -- and the producer warp stores the tile with bulk
// copies before it refills the stage.  Otherwise each consumer stores its own
// results to global memory.
template <int SRC, int EPT, bool BF, bool PEER, bool TM, bool BST, int MINB = 2>
__global__ void __launch_bounds__(kPipeThreads, MINB)
zs_update_pipe_kernel(const UpdateArgs a, const __grid_constant__ SegList segs, int stages,
                      const __grid_constant__ PeerParam<PEER> pt, const __grid_constant__ TmapParam<TM> tmap)
{
    static_assert(!TM || (SRC != kSrcStash && !PEER && (kPipeConsumers * EPT) % kBoxCols == 0),
                  "2-D boxes carry local rank rows of whole 256-column boxes");
    static_assert(!BST || (!TM && !PEER && SRC != kSrcStash), "bulk stores: 1-D contributions, no peer tables");
    constexpr bool kSpec = SRC == kSrcGradsSpeculative;
    constexpr int T = kPipeConsumers * EPT; // elements per tile
    wait_for_predecessor();
    allow_dependents();
    WsHeader* ws = a.ws;
    if (!kSpec && ws->skip)
        return; // uniform: the whole step is skipped

    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + stages;
    int64_t* first_tile = reinterpret_cast<int64_t*>(smem + 256); // [count + 1]
    unsigned char* ring = smem + kPipeHeaderBytes;
    const int src_bytes = SRC == kSrcStash ? 4 : 2 * a.nd;        // per element
    const int params_off = T * (12 + src_bytes);                   // BST: the tile's 16-bit results
    const int stage_bytes = T * (12 + src_bytes) + (BST ? T * 2 : 0);

    if (threadIdx.x == 0) {
        int64_t acc = 0;
        for (int s = 0; s < segs.count; ++s) {
            first_tile[s] = acc;
            acc += ((segs.seg[s].n >> 3) * 8 + T - 1) / T;
        }
        first_tile[segs.count] = acc;
        for (int i = 0; i < stages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kPipeConsumerWarps);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    const int64_t n_tiles = first_tile[segs.count];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cur = kSpec ? ws->cur : 0;
    const int nxt = kSpec ? cur ^ 1 : 0;
    const float* p_in = cur ? a.master[1] : a.master[0];
    const float* m_in = cur ? a.exp_avg[1] : a.exp_avg[0];
    const float* v_in = cur ? a.exp_avg_sq[1] : a.exp_avg_sq[0];
    float* p_out = nxt ? a.master[1] : a.master[0];
    float* m_out = nxt ? a.exp_avg[1] : a.exp_avg[0];
    float* v_out = nxt ? a.exp_avg_sq[1] : a.exp_avg_sq[0];
    bool failed = false;

    if (warp == kPipeConsumerWarps) {
        // ---- producer warp: lane 0 claims a free stage and announces its
        // bytes; the tile's copies (3 state arrays + the source rows) are then
        // issued by all 32 lanes at once ----
        const int n_copies = 3 + (SRC == kSrcStash ? 1 : (TM ? 1 : a.nd));
        constexpr bool kHint = !TM; // evict-first copies, except with tensor maps
        const uint64_t pol = kHint ? evict_first_policy() : 0;
        // BST: lane 0, which acquired the stage's empty barrier, stores the
        // results of tile gw from the stage and waits until the copies have
        // read shared memory, so that the stage can take new copies
        int si_out = 0; // segment of the tile being stored
        auto store_tile = [&](const unsigned char* sbuf, int64_t gw) {
            if (lane == 0) {
                si_out = next_tile_segment(first_tile, segs.count, gw, si_out);
                const Seg& sw = segs.seg[si_out];
                const int64_t w0 = (gw - first_tile[si_out]) * T;
                const int64_t wv = (sw.n >> 3) * 8;
                const uint32_t wn = (uint32_t)(wv - w0 < T ? wv - w0 : T);
                bulk_store(p_out + sw.s_off + w0, sbuf, wn * 4, pol);
                bulk_store(m_out + sw.s_off + w0, sbuf + T * 4, wn * 4, pol);
                bulk_store(v_out + sw.s_off + w0, sbuf + T * 8, wn * 4, pol);
                bulk_store(a.params + sw.p_off + w0, sbuf + params_off, wn * 2, pol);
                asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
            }
            __syncwarp();
        };
        int it = 0;
        int si = 0; // segment of the current tile
        for (int64_t g = blockIdx.x; g < n_tiles; g += gridDim.x, ++it) {
            const int st = it % stages;
            bool ok = true;
            if (lane == 0)
                ok = mbar_wait(&empty[st], ((it / stages) & 1) ^ 1, a.wait_budget);
            if (!__shfl_sync(0xffffffffu, ok, 0)) {
                failed = true;
                break;
            }
            if constexpr (BST)
                if (it >= stages) // the stage's previous tile
                    store_tile(ring + (size_t)st * stage_bytes, g - (int64_t)stages * gridDim.x);
            si = next_tile_segment(first_tile, segs.count, g, si);
            const Seg& sg = segs.seg[si];
            const int64_t e0 = (g - first_tile[si]) * T;
            const int64_t nv = (sg.n >> 3) * 8;
            const uint32_t n = (uint32_t)(nv - e0 < T ? nv - e0 : T);
            unsigned char* buf = ring + (size_t)st * stage_bytes;
            if (lane == 0) // 2-D boxes always deliver whole boxes, also past the tile's last element
                mbar_arrive_expect_tx(&full[st], TM ? n * 12u + (uint32_t)(T * src_bytes) : n * (12u + (uint32_t)src_bytes));
            __syncwarp();
            const int64_t so = sg.s_off + e0;
            for (int j = lane; j < n_copies; j += 32) {
                if (j < 3) {
                    const float* src = j == 0 ? p_in : (j == 1 ? m_in : v_in);
                    bulk_load<kHint>(buf + j * (T * 4), src + so, n * 4, &full[st], pol);
                } else if (SRC == kSrcStash) {
                    bulk_load<kHint>(buf + T * 12, a.stash + so, n * 4, &full[st], pol);
                } else if constexpr (TM) {
                    // the tile's contributions start at column f % stride of
                    // row f / stride (rank 0 of the segment's owner)
                    const int64_t f = sg.g_off + e0;
                    const int32_t x = (int32_t)(f % sg.g_rstride), y = (int32_t)(f / sg.g_rstride);
#pragma unroll
                    for (int b = 0; b < T / kBoxCols; ++b)
                        tma_load_2d(buf + T * 12 + (size_t)b * kBoxCols * src_bytes, &tmap, x + b * kBoxCols, y,
                                    &full[st]);
                } else {
                    const int r = j - 3;
                    bulk_load<kHint>(buf + T * 12 + r * (T * 2), ranks_at<PEER>(a.grads, pt, sg, e0).at(r), n * 2,
                                     &full[st], pol);
                }
            }
        }
        if constexpr (BST) {
            // the last tile of each stage, once its consumers are done
            for (int j = it - stages < 0 ? 0 : it - stages; j < it && !failed; ++j) {
                const int st = j % stages;
                bool ok = true;
                if (lane == 0)
                    ok = mbar_wait(&empty[st], (j / stages) & 1, a.wait_budget);
                if (!__shfl_sync(0xffffffffu, ok, 0)) {
                    failed = true;
                    break;
                }
                store_tile(ring + (size_t)st * stage_bytes, blockIdx.x + (int64_t)j * gridDim.x);
            }
            if (lane == 0) // the stores are complete before the CTA exits
                asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
        }
        // every copy issued lands before the producer may leave the CTA
        if (lane == 0) {
            const int issued = it;
            for (int st = 0; st < stages && st < issued; ++st) {
                const int last = issued - 1 - ((issued - 1 - st) % stages); // last use of stage st
                const long long drain = a.wait_budget > kDrainBudgetCycles ? a.wait_budget : kDrainBudgetCycles;
                if (!mbar_wait(&full[st], (last / stages) & 1, drain))
                    failed = true;
            }
        }
    } else {
        // ---- consumers ----
        const AdamK k = load_consts(a, ws, !kSpec);
        const float inv = ws->inv;
        const int c = threadIdx.x; // 0 .. kPipeConsumers-1
        bool bad = false;
        int it = 0;
        int si = 0; // segment of the current tile
        for (int64_t g = blockIdx.x; g < n_tiles; g += gridDim.x, ++it) {
            const int st = it % stages;
            const bool ok = mbar_wait(&full[st], (it / stages) & 1, a.wait_budget);
            if (!__all_sync(0xffffffffu, ok)) {
                failed = true;
                break;
            }
            si = next_tile_segment(first_tile, segs.count, g, si);
            const Seg& sg = segs.seg[si];
            const int64_t e0 = (g - first_tile[si]) * T;
            const int64_t nv = (sg.n >> 3) * 8;
            const int n = (int)(nv - e0 < T ? nv - e0 : T);
            const int i0 = c * EPT; // this thread's first element in the tile
            if (i0 < n) {
                const unsigned char* buf = ring + (size_t)st * stage_bytes;
                float p[EPT], m[EPT], v[EPT], gr[EPT];
                lds_f<EPT>(reinterpret_cast<const float*>(buf) + i0, p);
                lds_f<EPT>(reinterpret_cast<const float*>(buf + T * 4) + i0, m);
                lds_f<EPT>(reinterpret_cast<const float*>(buf + T * 8) + i0, v);
                if (SRC == kSrcStash) {
                    lds_f<EPT>(reinterpret_cast<const float*>(buf + T * 12) + i0, gr);
                } else {
                    // rank r's EPT elements: TM boxes hold 256 columns per
                    // rank row; 1-D copies hold T
                    const int rstep = TM ? kBoxCols : T;
                    const uint16_t* gs = reinterpret_cast<const uint16_t*>(buf + T * 12) +
                                         (TM ? (i0 / kBoxCols) * kBoxCols * a.nd + i0 % kBoxCols : i0);
                    lds_h<EPT, BF>(gs, gr);
                    for (int r = 1; r < a.nd; ++r) {
                        float f[EPT];
                        lds_h<EPT, BF>(gs + r * rstep, f);
#pragma unroll
                        for (int q = 0; q < EPT; ++q)
                            gr[q] = __fadd_rn(gr[q], f[q]);
                    }
#pragma unroll
                    for (int q = 0; q < EPT; ++q)
                        gr[q] = __fmul_rn(gr[q], inv);
                }
                if (kSpec) {
#pragma unroll
                    for (int q = 0; q < EPT; ++q)
                        bad |= !isfinite(gr[q]);
                }
#pragma unroll
                for (int q = 0; q < EPT; ++q)
                    adam_update(kSpec ? gr[q] : __fmul_rn(gr[q], k.clip), p[q], m[q], v[q], k);
                if constexpr (BST) {
                    // this thread's own slots (it alone read them), made
                    // visible to the producer's bulk copies
                    unsigned char* wbuf = ring + (size_t)st * stage_bytes;
                    sts_f<EPT>(reinterpret_cast<float*>(wbuf) + i0, p);
                    sts_f<EPT>(reinterpret_cast<float*>(wbuf + T * 4) + i0, m);
                    sts_f<EPT>(reinterpret_cast<float*>(wbuf + T * 8) + i0, v);
                    sts_h<EPT, BF>(reinterpret_cast<uint16_t*>(wbuf + params_off) + i0, p);
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                } else {
                    const int64_t so = sg.s_off + e0 + i0;
                    stg_f<EPT>(p_out + so, p);
                    stg_f<EPT>(m_out + so, m);
                    stg_f<EPT>(v_out + so, v);
                    stg_h<EPT, BF>(a.params + sg.p_off + e0 + i0, p);
                    if constexpr (PEER)
                        for (int d = 0; d < pt.n_dests; ++d)
                            stg_h<EPT, BF>(pt.dests[d] + sg.p_off + e0 + i0, p);
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&empty[st]);
        }
        // the < 8-element tail of each segment, scalar
        const int64_t gtid = (int64_t)blockIdx.x * kPipeConsumers + c;
        if (!failed) {
            for (int si = 0; si < segs.count; ++si) {
                const Seg& sg = segs.seg[si];
                const int64_t e = (sg.n >> 3) * 8 + gtid;
                if (e < sg.n)
                    bad |= update_scalar<SRC, BF, PEER>(a, pt, sg, e, k, inv, p_in, m_in, v_in, p_out, m_out, v_out);
            }
        }
        if (kSpec)
            flag_nonfinite(bad, &ws->overflow);
    }
    if (failed) {
        atomicOr(&ws->error, 1u);
        if (a.result)
            a.result->status = ZERO_ERR_TIMEOUT;
    }
}

// ---------------------------------------------------------------------------
// K2: statistics pre-pass -- overflow flag, fp64 sum of squares per block,
//     optionally the fp32 reduced gradient (stash)
// ---------------------------------------------------------------------------

template <bool VEC, bool STASH, bool BF, bool PEER>
__global__ void __launch_bounds__(kThreads, 2)
zs_stats_kernel(const StatsArgs a, const __grid_constant__ SegList segs, const __grid_constant__ PeerParam<PEER> pt)
{
    // The buckets of a step are independent: the next statistics launch may
    // start as soon as this one is resident.  Each launch waits for its
    // predecessor only before publishing its flag and partial sums, so launches
    // overlap at their boundaries while completion stays ordered (the flag was
    // reset by the prep kernel that heads the chain).
    allow_dependents();
    // The loss scale comes from the optimizer state: only the previous
    // step's last kernels wrote it, and they completed before this step began.
    const float inv = step_inv(a.st, a.inv, a.scale_mult);
    double acc = 0.0;
    bool bad = false;
    walk_segments<VEC>(
        segs,
        [&](const Seg& sg, int64_t e) {
            float g[8];
            rank_sum8<BF, 16>(ranks_at<PEER>(a.grads, pt, sg, e), a.nd, g);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                g[q] = __fmul_rn(g[q], inv);
                bad |= !isfinite(g[q]);
                const double d = (double)g[q];
                acc = __dadd_rn(acc, __dmul_rn(d, d));
            }
            if (STASH)
                st_f8(a.stash + sg.s_off + e, g);
        },
        [&](const Seg& sg, int64_t e) {
            const float g = __fmul_rn(rank_sum1<BF>(ranks_at<PEER>(a.grads, pt, sg, e), a.nd), inv);
            bad |= !isfinite(g);
            const double d = (double)g;
            acc = __dadd_rn(acc, __dmul_rn(d, d));
            if (STASH)
                a.stash[sg.s_off + e] = g;
        });
    wait_for_predecessor();
    flag_nonfinite(bad, &a.ws->overflow);

    // fixed-pattern block reduction of the fp64 partial sums
    __shared__ double warp_sum[kThreads / 32];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        acc = __dadd_rn(acc, __shfl_down_sync(0xffffffffu, acc, off));
    if ((threadIdx.x & 31) == 0)
        warp_sum[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x < 32) {
        double w = threadIdx.x < kThreads / 32 ? warp_sum[threadIdx.x] : 0.0;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            w = __dadd_rn(w, __shfl_down_sync(0xffffffffu, w, off));
        if (threadIdx.x == 0)
            a.partials[blockIdx.x] = w;
    }
}

// ---------------------------------------------------------------------------
// K3: finalize (one block) -- norm, clip coefficient, skip, bookkeeping
// ---------------------------------------------------------------------------

constexpr int kFinalizeThreads = 1024;

__device__ __forceinline__ double block_sum_partials(const double* partials, int64_t n)
{
    // fixed order: thread i sums partials i, i + 1024, ... ; then a fixed tree
    double acc = 0.0;
    for (int64_t i = threadIdx.x; i < n; i += kFinalizeThreads)
        acc = __dadd_rn(acc, partials[i]);
    __shared__ double warp_sum[kFinalizeThreads / 32];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        acc = __dadd_rn(acc, __shfl_down_sync(0xffffffffu, acc, off));
    if ((threadIdx.x & 31) == 0)
        warp_sum[threadIdx.x >> 5] = acc;
    __syncthreads();
    double w = 0.0;
    if (threadIdx.x < 32) {
        w = warp_sum[threadIdx.x];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            w = __dadd_rn(w, __shfl_down_sync(0xffffffffu, w, off));
    }
    return w; // valid in thread 0
}

// The step's global decision from the gradient's sum of squares and the
// overflow vote: norm, clip coefficient, skip, optimizer bookkeeping, result.
__device__ __forceinline__ void decide_step(WsHeader* ws, double sumsq, bool skip, float max_norm,
                                            zero_opt_state* st, zero_step_result* res)
{
    const double norm = __dsqrt_rn(sumsq);
    float clip = 1.0f;
    if (!skip && max_norm > 0.0f && norm > (double)max_norm)
        clip = __double2float_rn(__ddiv_rn((double)max_norm, norm));
    ws->skip = skip ? 1 : 0;
    ws->clip = clip;
    ws->sumsq = sumsq;
    ws->norm = norm;
    if (!skip) {
        st->t = ws->t_next;
        st->beta1_pow = ws->b1p_next;
        st->beta2_pow = ws->b2p_next;
    } else {
        st->skipped += 1;
    }
    // No reader of this step's scale is left: the statistics launches are
    // complete and the update reads the prep kernel's snapshot.
    advance_loss_scale(st, skip);
    if (res) {
        res->grad_norm = skip ? __longlong_as_double(0x7ff8000000000000LL) : norm;
        res->t = st->t;
        res->skipped = st->skipped;
        res->clip_coef = clip;
        res->overflow = skip ? 1 : 0;
        res->status = ZERO_OK;
        res->loss_scale = st->loss_scale;
    }
}

__global__ void __launch_bounds__(kFinalizeThreads)
zs_finalize_kernel(WsHeader* ws, const double* partials, int64_t n, float max_norm,
                   zero_opt_state* st, zero_step_result* res)
{
    wait_for_predecessor();
    allow_dependents();
    const double w = block_sum_partials(partials, n);
    if (threadIdx.x == 0)
        decide_step(ws, w, ws->overflow != 0u, max_norm, st, res);
}

// Split step, first half's end: this call's share of the global vote --
// its sum of squares (0 without a statistics pass) and whether it saw a
// non-finite gradient -- as two fp64 values that callers running one owner
// per process add up across processes (one sum-all-reduce of 16 bytes).
__global__ void __launch_bounds__(kFinalizeThreads)
zs_vote_local_kernel(WsHeader* ws, const double* partials, int64_t n)
{
    wait_for_predecessor();
    allow_dependents();
    const double w = block_sum_partials(partials, n);
    if (threadIdx.x == 0) {
        ws->vote[0] = w;
        ws->vote[1] = ws->overflow != 0u ? 1.0 : 0.0;
    }
}

// Split step, second half's start: the (now global) vote decides the step.
// Speculative: only the overflow flag, which the commit kernel then applies.
__global__ void zs_vote_apply_kernel(WsHeader* ws, int speculative, float max_norm, zero_opt_state* st,
                                     zero_step_result* res)
{
    wait_for_predecessor();
    allow_dependents();
    const bool skip = ws->vote[1] != 0.0;
    if (speculative)
        ws->overflow = skip ? 1u : 0u;
    else
        decide_step(ws, ws->vote[0], skip, max_norm, st, res);
}

// ---------------------------------------------------------------------------
// K5: speculative commit -- flip the live slot, or on overflow re-cast the
//     fp16 parameters from the unchanged live master; also zero_cast_params
// ---------------------------------------------------------------------------

template <bool VEC, bool BF, bool PEER>
__device__ __forceinline__ void cast_segments(const float* master, uint16_t* params, const SegList& segs,
                                              const PeerParam<PEER>& pt)
{
    walk_segments<VEC>(
        segs,
        [&](const Seg& sg, int64_t e) {
            float p[8];
            ld_f8(master + sg.s_off + e, p);
            store_params8<PEER>(params, pt, sg.p_off + e, pack_h8<BF>(p));
        },
        [&](const Seg& sg, int64_t e) { store_param1<PEER>(params, pt, sg.p_off + e, f2h<BF>(master[sg.s_off + e])); });
}

template <bool VEC, bool BF, bool PEER>
__global__ void __launch_bounds__(kThreads)
zs_commit_kernel(const UpdateArgs a, const __grid_constant__ SegList segs, int bookkeeping,
                 zero_opt_state* st, zero_step_result* res, const __grid_constant__ PeerParam<PEER> pt)
{
    wait_for_predecessor();
    const WsHeader* ws = a.ws;
    const bool fault = ws->error != 0u;
    const bool over = ws->overflow != 0u || fault;
    const int cur = ws->cur;
    if (bookkeeping && blockIdx.x == 0 && threadIdx.x == 0) {
        if (!over) {
            st->t = ws->t_next;
            st->beta1_pow = ws->b1p_next;
            st->beta2_pow = ws->b2p_next;
            st->cur = cur ^ 1;
        } else {
            st->skipped += 1;
        }
        if (!fault) // the update that read this step's scale has completed
            advance_loss_scale(st, over);
        if (res) {
            res->grad_norm = __longlong_as_double(0x7ff8000000000000LL);
            res->t = st->t;
            res->skipped = st->skipped;
            res->clip_coef = 1.0f;
            res->overflow = ws->overflow != 0u ? 1 : 0;
            res->status = fault ? ZERO_ERR_TIMEOUT : ZERO_OK;
            res->loss_scale = st->loss_scale;
        }
    }
    if (!over)
        return;
    cast_segments<VEC, BF, PEER>(cur ? a.master[1] : a.master[0], a.params, segs, pt);
}

template <bool VEC, bool BF>
__global__ void __launch_bounds__(kThreads)
zs_cast_kernel(const float* master, uint16_t* params, const __grid_constant__ SegList segs)
{
    cast_segments<VEC, BF, false>(master, params, segs, NoPeers{});
}

// ---------------------------------------------------------------------------
// Reduce-scatter with retention (stage 2): the owners' reduced gradients,
// the rank-order fp32 sum rounded once to the 16-bit format, kept at the
// state offsets for a later step to read as its single contribution
// ---------------------------------------------------------------------------

template <bool VEC, bool BF, bool PEER>
__global__ void __launch_bounds__(kThreads, 2)
zs_reduce_kernel(const uint16_t* grads, uint16_t* out, int nd, const __grid_constant__ SegList segs,
                 const __grid_constant__ PeerParam<PEER> pt)
{
    walk_segments<VEC>(
        segs,
        [&](const Seg& sg, int64_t e) {
            float sum[8];
            rank_sum8<BF>(ranks_at<PEER>(grads, pt, sg, e), nd, sum);
            __stcs(reinterpret_cast<uint4*>(out + sg.s_off + e), pack_h8<BF>(sum));
        },
        [&](const Seg& sg, int64_t e) {
            out[sg.s_off + e] = f2h<BF>(rank_sum1<BF>(ranks_at<PEER>(grads, pt, sg, e), nd));
        });
}

// ---------------------------------------------------------------------------
// launch geometry (the helpers shared with gather.cu are in zs_launch.h)
// ---------------------------------------------------------------------------

struct DevInfo {
    int sms = 0;
};

static std::mutex g_mu;
static std::unordered_map<int, DevInfo> g_dev;
static std::map<std::pair<const void*, int>, int> g_occ; // (kernel, device or shape key) -> blocks per SM

cudaError_t device_sms(int* sms)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_dev.find(dev);
    if (it == g_dev.end()) {
        DevInfo d;
        e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess)
            return e;
        it = g_dev.emplace(dev, d).first;
    }
    *sms = it->second.sms;
    return cudaSuccess;
}

cudaError_t blocks_per_sm(const void* kernel, int* occ)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    const std::pair<const void*, int> key(kernel, dev);
    {
        std::lock_guard<std::mutex> lk(g_mu);
        auto it = g_occ.find(key);
        if (it != g_occ.end()) {
            *occ = it->second;
            return cudaSuccess;
        }
    }
    int o = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, kernel, kThreads, 0);
    if (e != cudaSuccess)
        return e;
    o = o < 1 ? 1 : o;
    std::lock_guard<std::mutex> lk(g_mu);
    g_occ[key] = o;
    *occ = o;
    return cudaSuccess;
}

// units of work of a launch (8-element chunks when vectorised), all segments
static int64_t seg_work(const SegList& s, bool vec)
{
    int64_t w = 0;
    for (int i = 0; i < s.count; ++i)
        w += vec ? (s.seg[i].n + 7) >> 3 : s.seg[i].n;
    return w;
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------

cudaError_t launch_opt_init(zero_opt_state* st, float scale, float growth, float backoff, int32_t interval,
                            cudaStream_t s)
{
    return launch_plain(zs_opt_init_kernel, 1, 1, 0, s, st, scale, growth, backoff, interval);
}

cudaError_t launch_prep(const zero_opt_state* st, WsHeader* ws, float beta1, float beta2, float static_inv,
                        double scale_mult, cudaStream_t s)
{
    return launch_plain(zs_prep_kernel, 1, 1, 0, s, st, ws, beta1, beta2, static_inv, scale_mult);
}

// The peer table as the kernel parameter of a PEER / non-PEER instantiation.
template <bool PEER>
static PeerParam<PEER> peer_param(const PeerTable* peers)
{
    if constexpr (PEER)
        return *peers;
    else
        return NoPeers{};
}

template <int SRC, bool VEC, bool BF, bool PEER>
static cudaError_t launch_update_t(const UpdateArgs& a, const SegList& segs, const PeerTable* peers, cudaStream_t s)
{
    auto kernel = zs_update_kernel<SRC, VEC, BF, PEER>;
    int blocks = 0;
    cudaError_t e = grid_for(kernel, seg_work(segs, VEC), 0, &blocks);
    if (e != cudaSuccess)
        return e;
    return launch_overlapped(kernel, blocks, kThreads, 0, s, a, segs, peer_param<PEER>(peers));
}

template <int SRC, bool BF>
static cudaError_t launch_update_v(bool vec, const UpdateArgs& a, const SegList& segs, const PeerTable* peers,
                                   cudaStream_t s)
{
    if (peers)
        return vec ? launch_update_t<SRC, true, BF, true>(a, segs, peers, s)
                   : launch_update_t<SRC, false, BF, true>(a, segs, peers, s);
    return vec ? launch_update_t<SRC, true, BF, false>(a, segs, peers, s)
               : launch_update_t<SRC, false, BF, false>(a, segs, peers, s);
}

template <int SRC>
static cudaError_t launch_update_regs(bool vec, const UpdateArgs& a, const SegList& segs, const PeerTable* peers,
                                      cudaStream_t s)
{
    return a.bf16 ? launch_update_v<SRC, true>(vec, a, segs, peers, s)
                  : launch_update_v<SRC, false>(vec, a, segs, peers, s);
}

// Shape of the pipelined update for a given source: elements per consumer
// thread (tile = 256 x EPT), ring stages and CTAs per SM.  Chosen by
// measurement on one B200 (1B-parameter streams, 30- and 200-launch runs,
// the latter with the SM clock held near 1.5 GHz by the power cap), every
// shape bit-identical to the register path:
//   * contributions, Nd <= 8: EPT 4, 2 stages, 3 CTAs per SM -- 0.92 (Nd 1),
//     0.93 (2), 0.97 (4), 1.00 (8) of the copy bandwidth, against 0.79-0.95
//     for the register path and 0.90-1.00 for deeper 2-CTA rings;
//   * contributions, Nd <= 16: EPT 4, 2 stages, 2 CTAs (3 no longer fit):
//     1.02 at Nd = 16 against 0.94-0.97 for the register path;
//   * the 4-byte stash: EPT 8, 2 stages, 2 CTAs -- 0.96 against 0.89 for a
//     3-stage ring and 0.92 for the register path.
//   * contributions, 17 <= Nd <= 64: the Nd rank rows of a tile as 2-D
//     tensor-map boxes of [256 columns x Nd rows] (one copy per box instead
//     of one per rank, which at Nd = 32-64 had made the copy issue, not HBM,
//     the limit: 0.60-0.64), 2 stages: 2 boxes per tile while two CTAs fit
//     (Nd = 24: 3 CTAs, 1.01-1.04; Nd = 32: 2 CTAs, 0.99-1.01; Nd = 48:
//     2 CTAs, 1.05), else 1 box per tile and 3 CTAs (Nd = 64: 1.00-1.02),
//     against 0.91-0.99 for the register path.
// A shallow ring with more CTAs per SM beat every deeper one: the same bytes
// in flight per SM, spread over more independent producers.  Beyond Nd = 64
// the register path takes over.
// Stores (1-D contributions without peer tables): for 5 <= Nd <= 11 the
// results leave through the stage and the producer's bulk copies (BST).  A/B
// at 1B parameters, fractions of the copy bandwidth without -> with: Nd 5
// 0.97 -> 0.98, 6 0.97 -> 1.00, 7 0.97 -> 1.01, 8 0.97-0.98 -> 1.01 (256M:
// 0.94 -> 1.02, 2B: 0.97 -> 1.02), 9-11 0.96-0.97 -> 1.03-1.04.  Elsewhere
// the consumers store directly: at Nd = 4 bulk stores read 0.93 against
// 0.99, at Nd = 12 the results region leaves room for 2 CTAs only (0.93
// against 0.98), at Nd = 16 0.99 against 1.05, at Nd = 1 0.87 against 0.98,
// for the stash 0.91 against 0.98 and through peer tables 0.95 against 0.98:
// the producer may refill a stage only once its stores have read it, which
// costs more than it gains on streams with a larger share of writes.
struct PipeShape {
    int ept = 0, stages = 0, ctas_per_sm = 0, smem = 0;
    bool tm = false;  // rank rows by 2-D tensor-map boxes
    bool bst = false; // results stored by the producer's bulk copies
    bool occ3 = false; // peer tables: the build bounded to 3 CTAs per SM
};

constexpr int kPipeMaxNd = 16;    // 1-D copies of the rank rows up to here
constexpr int kPipeMaxNdTm = 64;  // 2-D tensor-map boxes of all Nd rank rows up to here
constexpr int kBulkStMinNd = 5, kBulkStMaxNd = 11; // bulk stores for these Nd (1-D, no peer tables)
// Peer tables: the kernel that stores into every destination needs 74
// registers, which leave room for 2 CTAs per SM; a build bounded to 3 CTAs
// (61 registers) is used up to this Nd.  One-GPU emulation, 512M parameters,
// fraction of the copy bandwidth, 2-CTA -> 3-CTA build: Nd 1 0.86 -> 0.99,
// Nd 2 0.87 -> 0.98, Nd 3 0.92 -> 0.96, Nd 4 0.97 -> 0.93, Nd 8 0.97 -> 0.92.
constexpr int kPeerOcc3MaxNd = 3;

static bool pipe_shape(int src, int nd, bool peers, PipeShape* ps)
{
    const bool stash = src == kSrcStash;
    if (!stash && nd > kPipeMaxNdTm)
        return false;
    int e = 12 + (stash ? 4 : 2 * nd); // bytes per element of one stage
    PipeShape p;
    if (stash) {
        p.ept = 8, p.stages = 2, p.ctas_per_sm = 2;
    } else if (nd <= kPipeMaxNd) {
        p.ept = 4, p.stages = 2, p.ctas_per_sm = 3;
        p.bst = !peers && nd >= kBulkStMinNd && nd <= kBulkStMaxNd;
        p.occ3 = peers && nd <= kPeerOcc3MaxNd;
        e += p.bst ? 2 : 0; // the 16-bit results region
    } else {
        // 2-D boxes of all Nd rank rows: two 256-column boxes per tile while a
        // 2-stage ring of them still fits two CTAs per SM (Nd <= 50), else one
        const int two_boxes = kPipeHeaderBytes + 2 * kPipeConsumers * 2 * e;
        p.ept = 2 * (two_boxes + 1024) <= 228 * 1024 ? 2 : 1;
        p.stages = 2, p.ctas_per_sm = 3, p.tm = true;
    }
    // CTAs per SM that the shared memory allows (228 KB per SM, 1 KB of it
    // reserved per CTA); the launch also checks the occupancy it gets
    for (;;) {
        p.smem = kPipeHeaderBytes + p.stages * kPipeConsumers * p.ept * e;
        if (p.ctas_per_sm * (p.smem + 1024) <= 228 * 1024 || p.ctas_per_sm == 1)
            break;
        --p.ctas_per_sm;
    }
    if (p.smem > 220 * 1024 + kPipeHeaderBytes)
        return false;
    *ps = p;
    return true;
}

static std::map<std::pair<const void*, int>, int> g_smem_set; // (kernel, device) -> bytes allowed

// cuTensorMapEncodeTiled, looked up once from the driver through the runtime
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_tiled()
{
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

// The tensor map of the rank rows a launch reads: a 2-D array of 16-bit
// values whose row stride is the segments' rank stride, rows = ranks (of all
// owners in the per-owner layout), boxes of [256 columns x Nd rows].  Its
// extent is exactly the columns and rows the segments address, so a box's
// overhang past a segment's end reads no memory (it arrives as zeros).
// Returns false (and the launch takes the register path) unless every box
// coordinate the kernel will use is a multiple of 8 columns (16 bytes) and
// the map encodes.
static bool rank_rows_map(const UpdateArgs& a, const SegList& segs, CUtensorMap* map)
{
    const EncodeTiledFn encode = encode_tiled();
    if (!encode || segs.count < 1 || a.nd < 1 || a.nd > 256 || (reinterpret_cast<uintptr_t>(a.grads) & 15))
        return false;
    const int64_t stride = segs.seg[0].g_rstride;
    if (stride <= 0 || stride % 8)
        return false;
    int64_t cols = 0, rows = 0;
    for (int i = 0; i < segs.count; ++i) {
        const Seg& sg = segs.seg[i];
        if (sg.g_rstride != stride || sg.g_off < 0)
            return false;
        const int64_t x0 = sg.g_off % stride, y0 = sg.g_off / stride;
        // tiles start at x0 + (multiples of 256): all on 16-byte columns
        if (x0 % 8 || x0 + sg.n > stride)
            return false;
        cols = cols > x0 + sg.n ? cols : x0 + sg.n;
        rows = rows > y0 + a.nd ? rows : y0 + a.nd;
    }
    if (cols < 1 || cols > INT32_MAX - 2 * kBoxCols || rows > INT32_MAX)
        return false;
    const cuuint64_t dim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t stride_bytes[1] = {(cuuint64_t)stride * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kBoxCols, (cuuint32_t)a.nd};
    const cuuint32_t elem_strides[2] = {1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<uint16_t*>(a.grads), dim, stride_bytes, box,
                  elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool TM>
static bool tmap_param(const UpdateArgs& a, const SegList& segs, TmapParam<TM>* out)
{
    if constexpr (TM)
        return rank_rows_map(a, segs, out);
    else
        return true;
}

template <int SRC, int EPT, bool BF, bool PEER, bool TM, bool BST = false, int MINB = 2>
static cudaError_t launch_pipe_t(const UpdateArgs& a, const SegList& segs, const PipeShape& ps,
                                 const PeerTable* peers, cudaStream_t s)
{
    auto kernel = zs_update_pipe_kernel<SRC, EPT, BF, PEER, TM, BST, MINB>;
    TmapParam<TM> tmap;
    if (!tmap_param<TM>(a, segs, &tmap))
        return cudaErrorNotSupported; // the caller falls back to the register path
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || (e = device_sms(&sms)) != cudaSuccess)
        return e;
    const std::pair<const void*, int> key(reinterpret_cast<const void*>(kernel), dev);
    {
        std::lock_guard<std::mutex> lk(g_mu);
        auto it = g_smem_set.find(key);
        if (it == g_smem_set.end() || it->second < ps.smem) {
            e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 220 * 1024 + kPipeHeaderBytes);
            if (e != cudaSuccess)
                return e;
            g_smem_set[key] = 220 * 1024 + kPipeHeaderBytes;
        }
    }
    int occ = 0;
    {
        const std::pair<const void*, int> okey(reinterpret_cast<const void*>(kernel), dev * 4096 + ps.smem / 256);
        std::lock_guard<std::mutex> lk(g_mu);
        auto it = g_occ.find(okey);
        if (it != g_occ.end())
            occ = it->second;
    }
    if (occ == 0) {
        // blocks per SM that fit at this shape (registers, threads, shared memory)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, kPipeThreads, ps.smem);
        if (e != cudaSuccess)
            return e;
        occ = occ < 1 ? 1 : occ;
        std::lock_guard<std::mutex> lk(g_mu);
        g_occ[std::pair<const void*, int>(reinterpret_cast<const void*>(kernel), dev * 4096 + ps.smem / 256)] = occ;
    }
    int64_t tiles = 0;
    const int T = kPipeConsumers * EPT;
    for (int i = 0; i < segs.count; ++i)
        tiles += ((segs.seg[i].n >> 3) * 8 + T - 1) / T;
    int64_t grid = (int64_t)sms * (ps.ctas_per_sm < occ ? ps.ctas_per_sm : occ);
    grid = tiles < grid ? tiles : grid;
    grid = grid < 1 ? 1 : grid;
    return launch_overlapped(kernel, (unsigned)grid, kPipeThreads, ps.smem, s, a, segs, ps.stages,
                             peer_param<PEER>(peers), tmap);
}

template <int SRC, bool BF, bool PEER>
static cudaError_t launch_pipe_f(const UpdateArgs& a, const SegList& segs, const PipeShape& ps,
                                 const PeerTable* peers, cudaStream_t s)
{
    // pipe_shape chooses 8 (the stash) or 4 (contributions, 1-D rows) elements
    // per thread, or 1 or 2 (contributions by 2-D boxes)
    if (ps.tm) {
        if constexpr (SRC != kSrcStash && !PEER)
            return ps.ept == 2 ? launch_pipe_t<SRC, 2, BF, PEER, true>(a, segs, ps, peers, s)
                               : launch_pipe_t<SRC, 1, BF, PEER, true>(a, segs, ps, peers, s);
        // one tensor map cannot span the separate buffers of a peer table,
        // and the 1-D kernel's tile does not fit a 2-D shape's ring
        return cudaErrorNotSupported;
    }
    if (ps.ept != 8 && ps.ept != 4)
        return cudaErrorNotSupported;
    if constexpr (PEER && SRC != kSrcStash)
        if (ps.occ3 && ps.ept == 4)
            return launch_pipe_t<SRC, 4, BF, PEER, false, false, 3>(a, segs, ps, peers, s);
    if (ps.bst) {
        if constexpr (SRC != kSrcStash && !PEER)
            if (ps.ept == 4)
                return launch_pipe_t<SRC, 4, BF, PEER, false, true>(a, segs, ps, peers, s);
        return cudaErrorNotSupported;
    }
    return ps.ept == 8 ? launch_pipe_t<SRC, 8, BF, PEER, false>(a, segs, ps, peers, s)
                       : launch_pipe_t<SRC, 4, BF, PEER, false>(a, segs, ps, peers, s);
}

// With peer tables the producer copies rank r's rows from table entry r (a
// buffer of this GPU or another GPU's, by plain 1-D bulk copies: no
// multicast), and the consumers store the new parameters into every
// destination.
template <int SRC>
static cudaError_t launch_pipe(const UpdateArgs& a, const SegList& segs, const PipeShape& ps,
                               const PeerTable* peers, cudaStream_t s)
{
    if (peers)
        return a.bf16 ? launch_pipe_f<SRC, true, true>(a, segs, ps, peers, s)
                      : launch_pipe_f<SRC, false, true>(a, segs, ps, peers, s);
    return a.bf16 ? launch_pipe_f<SRC, true, false>(a, segs, ps, nullptr, s)
                  : launch_pipe_f<SRC, false, false>(a, segs, ps, nullptr, s);
}

// The bulk-copy pipeline takes the stash source and up to 64 contributions
// (see pipe_shape for the measurements), or up to 16 through peer tables
// (1-D row copies only); the register path takes larger Nd, and any launch
// whose layout a tensor map cannot describe with 16-byte aligned columns.  A launch that leaves each CTA fewer than 64 tiles pays
// several percent for the ring's fill and drain: from Nd = 4 up, where the
// register path is close at full speed, such launches take the register path
// (16M elements at Nd = 8, 37 tiles per CTA: 0.95 against 0.85 of the copy
// bandwidth).  With Nd <= 3 the pipeline wins at every size (16M elements at
// Nd = 1: 0.89 against 0.77).
constexpr int64_t kPipeMinTilesPerCta = 64;

static bool use_pipeline(int src, int nd, int64_t elems, const PipeShape& ps, int sms, bool peers)
{
    if (src == kSrcStash || nd <= 3)
        return true;
    if (peers && nd > kPipeMaxNd)
        return false;
    const int64_t tiles = elems / ((int64_t)kPipeConsumers * ps.ept);
    return nd <= kPipeMaxNdTm && tiles >= kPipeMinTilesPerCta * (int64_t)sms * ps.ctas_per_sm;
}

cudaError_t launch_update(int src, bool vec, const UpdateArgs& a, const SegList& segs, const PeerTable* peers,
                          cudaStream_t s)
{
    PipeShape ps;
    int sms = 0;
    if (vec && pipe_shape(src, a.nd, peers != nullptr, &ps) && device_sms(&sms) == cudaSuccess &&
        use_pipeline(src, a.nd, seg_work(segs, true) * 8, ps, sms, peers != nullptr)) {
        cudaError_t e;
        switch (src) {
        case kSrcGradsSpeculative: e = launch_pipe<kSrcGradsSpeculative>(a, segs, ps, peers, s); break;
        case kSrcGradsInPlace: e = launch_pipe<kSrcGradsInPlace>(a, segs, ps, peers, s); break;
        default: e = launch_pipe<kSrcStash>(a, segs, ps, peers, s); break;
        }
        if (e != cudaErrorNotSupported) // a shape or tensor map this launch cannot take: register path
            return e;
    }
    switch (src) {
    case kSrcGradsSpeculative: return launch_update_regs<kSrcGradsSpeculative>(vec, a, segs, peers, s);
    case kSrcGradsInPlace: return launch_update_regs<kSrcGradsInPlace>(vec, a, segs, peers, s);
    default: return launch_update_regs<kSrcStash>(vec, a, segs, peers, s);
    }
}

int stats_blocks(bool vec, const SegList& segs)
{
    // a function of the work alone (not of the device), so the workspace size
    // and the fp64 summation order are the same on every GPU
    const int64_t want = (seg_work(segs, vec) + kThreads - 1) / kThreads;
    return (int)(want < 1 ? 1 : (want > kStatsMaxBlocks ? kStatsMaxBlocks : want));
}

template <bool VEC, bool STASH, bool BF, bool PEER>
static cudaError_t launch_stats_t(const StatsArgs& a, const SegList& segs, const PeerTable* peers, cudaStream_t s)
{
    return launch_overlapped(zs_stats_kernel<VEC, STASH, BF, PEER>, stats_blocks(VEC, segs), kThreads, 0, s, a,
                             segs, peer_param<PEER>(peers));
}

template <bool BF, bool PEER>
static cudaError_t launch_stats_f(bool vec, const StatsArgs& a, const SegList& segs, const PeerTable* peers,
                                  cudaStream_t s)
{
    const bool stash = a.stash != nullptr;
    if (vec)
        return stash ? launch_stats_t<true, true, BF, PEER>(a, segs, peers, s)
                     : launch_stats_t<true, false, BF, PEER>(a, segs, peers, s);
    return stash ? launch_stats_t<false, true, BF, PEER>(a, segs, peers, s)
                 : launch_stats_t<false, false, BF, PEER>(a, segs, peers, s);
}

cudaError_t launch_stats(bool vec, const StatsArgs& a, const SegList& segs, const PeerTable* peers, cudaStream_t s)
{
    if (peers)
        return a.bf16 ? launch_stats_f<true, true>(vec, a, segs, peers, s)
                      : launch_stats_f<false, true>(vec, a, segs, peers, s);
    return a.bf16 ? launch_stats_f<true, false>(vec, a, segs, peers, s)
                  : launch_stats_f<false, false>(vec, a, segs, peers, s);
}

cudaError_t launch_finalize(WsHeader* ws, const double* partials, int64_t n, float max_norm,
                            zero_opt_state* st, zero_step_result* res, cudaStream_t s)
{
    return launch_overlapped(zs_finalize_kernel, 1, kFinalizeThreads, 0, s, ws, partials, n, max_norm, st, res);
}

cudaError_t launch_vote_local(WsHeader* ws, const double* partials, int64_t n, cudaStream_t s)
{
    return launch_overlapped(zs_vote_local_kernel, 1, kFinalizeThreads, 0, s, ws, partials, n);
}

cudaError_t launch_vote_apply(WsHeader* ws, bool speculative, float max_norm, zero_opt_state* st,
                              zero_step_result* res, cudaStream_t s)
{
    // an ordinary launch: the caller's all-reduce of the vote comes before it
    return launch_plain(zs_vote_apply_kernel, 1, 1, 0, s, ws, speculative ? 1 : 0, max_norm, st, res);
}

template <bool VEC, bool BF, bool PEER>
static cudaError_t launch_commit_t(const UpdateArgs& a, const SegList& segs, bool bookkeeping, zero_opt_state* st,
                                   zero_step_result* res, const PeerTable* peers, cudaStream_t s)
{
    auto kernel = zs_commit_kernel<VEC, BF, PEER>;
    int blocks = 0;
    cudaError_t e = grid_for(kernel, seg_work(segs, VEC), 0, &blocks);
    if (e != cudaSuccess)
        return e;
    return launch_overlapped(kernel, blocks, kThreads, 0, s, a, segs, bookkeeping ? 1 : 0, st, res,
                             peer_param<PEER>(peers));
}

template <bool BF, bool PEER>
static cudaError_t launch_commit_f(bool vec, const UpdateArgs& a, const SegList& segs, bool bookkeeping,
                                   zero_opt_state* st, zero_step_result* res, const PeerTable* peers, cudaStream_t s)
{
    return vec ? launch_commit_t<true, BF, PEER>(a, segs, bookkeeping, st, res, peers, s)
               : launch_commit_t<false, BF, PEER>(a, segs, bookkeeping, st, res, peers, s);
}

cudaError_t launch_commit(bool vec, const UpdateArgs& a, const SegList& segs, bool bookkeeping,
                          zero_opt_state* st, zero_step_result* res, const PeerTable* peers, cudaStream_t s)
{
    if (peers)
        return a.bf16 ? launch_commit_f<true, true>(vec, a, segs, bookkeeping, st, res, peers, s)
                      : launch_commit_f<false, true>(vec, a, segs, bookkeeping, st, res, peers, s);
    return a.bf16 ? launch_commit_f<true, false>(vec, a, segs, bookkeeping, st, res, peers, s)
                  : launch_commit_f<false, false>(vec, a, segs, bookkeeping, st, res, peers, s);
}

template <bool VEC, bool BF, bool PEER>
static cudaError_t launch_reduce_t(const uint16_t* grads, uint16_t* out, int nd, const SegList& segs,
                                   const PeerTable* peers, cudaStream_t s)
{
    auto kernel = zs_reduce_kernel<VEC, BF, PEER>;
    int blocks = 0;
    cudaError_t e = grid_for(kernel, seg_work(segs, VEC), 0, &blocks);
    if (e != cudaSuccess)
        return e;
    return launch_plain(kernel, blocks, kThreads, 0, s, grads, out, nd, segs, peer_param<PEER>(peers));
}

template <bool BF, bool PEER>
static cudaError_t launch_reduce_f(bool vec, const uint16_t* grads, uint16_t* out, int nd, const SegList& segs,
                                   const PeerTable* peers, cudaStream_t s)
{
    return vec ? launch_reduce_t<true, BF, PEER>(grads, out, nd, segs, peers, s)
               : launch_reduce_t<false, BF, PEER>(grads, out, nd, segs, peers, s);
}

cudaError_t launch_reduce(bool vec, bool bf16, const uint16_t* grads, uint16_t* out, int nd, const SegList& segs,
                          const PeerTable* peers, cudaStream_t s)
{
    if (peers)
        return bf16 ? launch_reduce_f<true, true>(vec, grads, out, nd, segs, peers, s)
                    : launch_reduce_f<false, true>(vec, grads, out, nd, segs, peers, s);
    return bf16 ? launch_reduce_f<true, false>(vec, grads, out, nd, segs, peers, s)
                : launch_reduce_f<false, false>(vec, grads, out, nd, segs, peers, s);
}

template <bool VEC, bool BF>
static cudaError_t launch_cast_t(const float* master, uint16_t* params, const SegList& segs, cudaStream_t s)
{
    int blocks = 0;
    cudaError_t e = grid_for(zs_cast_kernel<VEC, BF>, seg_work(segs, VEC), 0, &blocks);
    if (e != cudaSuccess)
        return e;
    return launch_plain(zs_cast_kernel<VEC, BF>, blocks, kThreads, 0, s, master, params, segs);
}

cudaError_t launch_cast(bool vec, bool bf16, const float* master, uint16_t* params, const SegList& segs,
                        cudaStream_t s)
{
    if (bf16)
        return vec ? launch_cast_t<true, true>(master, params, segs, s) : launch_cast_t<false, true>(master, params, segs, s);
    return vec ? launch_cast_t<true, false>(master, params, segs, s) : launch_cast_t<false, false>(master, params, segs, s);
}

} // namespace zs
