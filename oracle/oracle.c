/*
 * oracle.c -- plain, slow CPU restatement of the ZeRO-DP partitioned
 * mixed-precision Adam shard step.
 *
 * TEST INFRASTRUCTURE.  This is the independent checker for the CUDA library
 * in zero_dp_partitioned_shard_b200/.  Only the test suite, the smoke check
 * and the benchmark's CPU-baseline / reference leg load it; the library never
 * does, and the two share no source, header, table or helper.
 *
 * Sources (open-web pages on ZeRO, arXiv:1910.02054), cited below as:
 *   [Note]    "ZeRO" record, anthology-of-the-sota note 103 (dmarx.github.io)
 *   [Dissect] "ZeRO memory optimization: training large models", engineering
 *             dissection (trishampatil.com)
 *   [Gloss]   "ZeRO optimization" glossary (emergent.sh)
 *   [Guide]   "ZeRO: partitioning training state across GPUs" (upskillscore.com)
 *
 * What it computes.  Partitioning does not change the arithmetic of a data-
 * parallel step: ZeRO only changes which process stores and updates which
 * slice ([Dissect] "ZeRO's Core Idea"; [Gloss] "How ZeRO Works").  So the
 * plain definition of the partitioned step is the non-partitioned mixed-
 * precision Adam step on the all-reduced gradient, sliced by owner.  This file
 * computes exactly that, element by element, over the flat parameter vector,
 * and never blocks, fuses or reorders beyond the definition.
 *
 * Precision.  The pages fix the storage types ([Dissect] "The Real Problem",
 * 16-Psi equation; [Note] Concepts, mixed precision): fp16 parameters and
 * gradients, fp32 master copy, momentum and variance.  bfloat16 (the same
 * 2 bytes) is supported as an alternative 16-bit format.  The update is therefore
 * done in fp32 with every operation separately rounded (built with
 * -ffp-contract=off, no fast-math, SSE arithmetic so no excess precision).
 *
 * Readings where the pages are silent (they give neither update equations nor
 * loss scaling, overflow handling or clipping):
 *   - Adam: Kingma & Ba (2015), Algorithm 1, with bias correction and eps
 *     added outside the square root; AdamW decay per Loshchilov & Hutter
 *     (2019): decoupled, lr-scaled, applied to the pre-update parameter.
 *   - Reduce-scatter result = the SUM of the Nd contributions, taken left to
 *     right in rank order 0..Nd-1 in fp32 (optionally divided by Nd).
 *   - Unscaling multiplies by the fp32 reciprocal of the loss scale.
 *   - Overflow: any non-finite reduced, unscaled gradient element skips the
 *     whole step; no state, no parameter and no step counter changes.
 *   - Clipping: global L2 norm over all real elements (pads excluded); the
 *     sum of squares is the exact one to within a few fp64 ulp (Neumaier's
 *     compensated summation, 1974, of the exact fp64 squares of the fp32
 *     gradient); coefficient max/norm only when the norm exceeds max.
 *   - Bias corrections: running products beta^t in fp64, 1 - beta^t rounded
 *     to fp32.
 *   - Padding: equal shards of L = ceil(Psi/(Nd*A))*A elements.
 *   - Stage-2 retention: the gradient an owner keeps after the reduce-scatter
 *     is that fp32 sum rounded once (to nearest even) to the gradients'
 *     16-bit format.
 *
 * Every function here is pinned by a CPU test against values the pages print,
 * closed forms or library routines (tests/test_oracle_*.py).  Nothing is
 * "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* binary16 <-> binary32 (own bit-level code; IEEE 754-2008 formats)         */
/* ------------------------------------------------------------------------ */

/* Exact widening of an IEEE binary16 bit pattern to binary32. */
float oracle_half_to_float(uint16_t h)
{
    uint32_t sign = (uint32_t)(h & 0x8000u) << 16;
    uint32_t exp = (h >> 10) & 0x1Fu;
    uint32_t man = h & 0x3FFu;
    uint32_t bits;
    if (exp == 0x1Fu) {
        /* infinity or NaN: widen the payload */
        bits = sign | 0x7F800000u | (man << 13);
    } else if (exp != 0) {
        /* normal: move the exponent from bias 15 to bias 127 */
        bits = sign | ((exp + 112u) << 23) | (man << 13);
    } else if (man == 0) {
        bits = sign; /* signed zero */
    } else {
        /* subnormal man * 2^-24: shift the leading one up to the hidden bit */
        int e = -14;
        while (!(man & 0x400u)) {
            man <<= 1;
            e -= 1;
        }
        man &= 0x3FFu;
        bits = sign | ((uint32_t)(e + 127) << 23) | (man << 13);
    }
    float f;
    memcpy(&f, &bits, sizeof f);
    return f;
}

/* Round to nearest, ties to even, of q + rem/2^drop (drop >= 1). */
static uint32_t round_nearest_even(uint32_t q, uint32_t rem, int drop)
{
    uint32_t half = 1u << (drop - 1);
    if (rem > half || (rem == half && (q & 1u)))
        q += 1u;
    return q;
}

/* binary32 -> binary16, round to nearest even, subnormals kept, overflow to
 * infinity, NaN kept quiet with its top payload bits. */
uint16_t oracle_float_to_half(float f)
{
    uint32_t x;
    memcpy(&x, &f, sizeof x);
    uint32_t sign = (x >> 16) & 0x8000u;
    uint32_t exp = (x >> 23) & 0xFFu;
    uint32_t man = x & 0x7FFFFFu;
    if (exp == 0xFFu)
        return (uint16_t)(man ? (sign | 0x7E00u | (man >> 13)) : (sign | 0x7C00u));
    int e = (int)exp - 127 + 15; /* exponent in binary16's bias */
    if (e >= 31)
        return (uint16_t)(sign | 0x7C00u);
    if (e >= 1) {
        /* normal result: keep 10 of 23 mantissa bits; a carry out of the
         * mantissa correctly bumps the exponent (and 0x7BFF+1 is infinity) */
        uint32_t q = ((uint32_t)e << 10) | (man >> 13);
        q = round_nearest_even(q, man & 0x1FFFu, 13);
        return (uint16_t)(sign | q);
    }
    /* subnormal (or zero) result: value = full * 2^(e-14-... ) -> units of 2^-24 */
    if (exp == 0)
        return (uint16_t)sign; /* fp32 subnormals are far below 2^-25 */
    int drop = 14 - e;          /* >= 14 */
    if (drop > 24)
        return (uint16_t)sign;  /* below half the smallest subnormal */
    uint32_t full = man | 0x800000u;
    uint32_t q = full >> drop;
    q = round_nearest_even(q, full & ((1u << drop) - 1u), drop);
    return (uint16_t)(sign | q); /* q == 0x400 is the smallest normal */
}

/* bfloat16: the upper 16 bits of a binary32 (same exponent range, 8-bit
 * significand).  Widening is exact. */
float oracle_bf16_to_float(uint16_t h)
{
    uint32_t bits = (uint32_t)h << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return f;
}

/* binary32 -> bfloat16, round to nearest even on the 16 dropped bits
 * (subnormals kept, overflow to infinity, NaN kept quiet). */
uint16_t oracle_float_to_bf16(float f)
{
    uint32_t x;
    memcpy(&x, &f, sizeof x);
    if ((x & 0x7F800000u) == 0x7F800000u && (x & 0x7FFFFFu))
        return (uint16_t)((x >> 16) | 0x0040u);
    return (uint16_t)round_nearest_even(x >> 16, x & 0xFFFFu, 16);
}

void oracle_bf16_to_float_array(const uint16_t* h, float* f, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        f[i] = oracle_bf16_to_float(h[i]);
}

void oracle_float_to_bf16_array(const float* f, uint16_t* h, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        h[i] = oracle_float_to_bf16(f[i]);
}

void oracle_half_to_float_array(const uint16_t* h, float* f, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        f[i] = oracle_half_to_float(h[i]);
}

void oracle_float_to_half_array(const float* f, uint16_t* h, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        h[i] = oracle_float_to_half(f[i]);
}

/* ------------------------------------------------------------------------ */
/* Partition plan                                                            */
/* ------------------------------------------------------------------------ */

/* Each of the Nd processes owns one contiguous 1/Nd slice of the flat model
 * state ([Note] Method, P_os / P_g / P_p; [Dissect] sections ZeRO-1, ZeRO-2,
 * ZeRO-3; [Guide] "How it works").  Psi need not divide by Nd, so every shard
 * is padded to the same length L, a multiple of the alignment A; only the
 * last non-empty shard is short of real elements.  Buckets are fixed ranges of
 * B elements of the flat buffer (the constant-size fused buffers of ZeRO-R,
 * [Note] Method, CB), ignoring owner and tensor boundaries. */
typedef struct {
    int64_t psi;       /* real parameters */
    int64_t psi_pad;   /* Nd * L */
    int64_t shard_len; /* L */
    int64_t align;     /* A */
    int64_t bucket;    /* B (0: one bucket) */
    int64_t n_buckets;
    int32_t nd;
    int32_t pad_;
} oracle_plan_t;

int oracle_plan(int64_t psi, int32_t nd, int64_t align, int64_t bucket, oracle_plan_t* out)
{
    if (!out || psi < 1 || nd < 1 || align < 1 || bucket < 0)
        return -1;
    int64_t unit = (int64_t)nd * align;
    int64_t L = ((psi + unit - 1) / unit) * align;
    out->psi = psi;
    out->nd = nd;
    out->align = align;
    out->shard_len = L;
    out->psi_pad = (int64_t)nd * L;
    out->bucket = bucket;
    out->n_buckets = bucket > 0 ? (psi + bucket - 1) / bucket : 1;
    out->pad_ = 0;
    return 0;
}

/* Owner r's slice: flat [r*L, r*L + real_len), real_len in [0, L]. */
void oracle_shard(const oracle_plan_t* p, int32_t r, int64_t* start, int64_t* real_len)
{
    int64_t s = (int64_t)r * p->shard_len;
    int64_t len = p->psi - s;
    if (len < 0)
        len = 0;
    if (len > p->shard_len)
        len = p->shard_len;
    *start = s;
    *real_len = len;
}

/* Bucket k: flat [k*B, min((k+1)*B, Psi)). */
void oracle_bucket(const oracle_plan_t* p, int64_t k, int64_t* start, int64_t* len)
{
    if (p->bucket <= 0) {
        *start = 0;
        *len = p->psi;
        return;
    }
    int64_t s = k * p->bucket;
    int64_t e = s + p->bucket;
    if (e > p->psi)
        e = p->psi;
    *start = s;
    *len = e > s ? e - s : 0;
}

/* Tensors laid back to back in the flat buffer, split at owner boundaries.
 * Each piece is 5 int64: {tensor, owner, offset_in_tensor, length,
 * offset_in_shard}.  Returns the number of pieces (writing at most cap), or -1
 * when the sizes do not add up to Psi. */
int64_t oracle_tensor_segments(const oracle_plan_t* p, const int64_t* sizes, int32_t n_tensors,
                               int64_t* out, int64_t cap)
{
    int64_t total = 0;
    for (int32_t t = 0; t < n_tensors; ++t) {
        if (sizes[t] < 0)
            return -1;
        total += sizes[t];
    }
    if (total != p->psi)
        return -1;
    int64_t off = 0, k = 0;
    for (int32_t t = 0; t < n_tensors; ++t) {
        int64_t pos = 0;
        while (pos < sizes[t]) {
            int64_t flat = off + pos;
            int64_t owner = flat / p->shard_len;
            int64_t owner_end = (owner + 1) * p->shard_len;
            int64_t len = sizes[t] - pos;
            if (flat + len > owner_end)
                len = owner_end - flat;
            if (k < cap) {
                int64_t* e = out + 5 * k;
                e[0] = t;
                e[1] = owner;
                e[2] = pos;
                e[3] = len;
                e[4] = flat - owner * p->shard_len;
            }
            ++k;
            pos += len;
        }
        off += sizes[t];
    }
    return k;
}

/* ------------------------------------------------------------------------ */
/* Accounting                                                                */
/* ------------------------------------------------------------------------ */

/* Model-state bytes per device and communication volume per step.
 * [Dissect] "The Real Problem": 2 Psi fp16 params + 2 Psi fp16 grads + K Psi
 * Adam states, K = 12 (fp32 copy, momentum, variance), 16 Psi in all.
 * [Dissect] "The Full Progression, in One View" (table): plain DP 16 Psi;
 * P_os 4 Psi + 12 Psi/Nd; P_os+g 2 Psi + 14 Psi/Nd; P_os+g+p 16 Psi/Nd; comm
 * 2 Psi, 2 Psi, 2 Psi, 3 Psi.  [Guide] "How it works": the 3 Psi of stage 3
 * is one gradient reduce-scatter plus two parameter all-gathers (forward and
 * backward), each Psi.  Stage 0 means plain data parallelism.
 * Communication is counted in elements per process per step (the pages write
 * "Psi"); bytes assume fp16 elements.  The ring figure ((Nd-1)/Nd of each
 * collective) is a derived extra, not on the pages. */
typedef struct {
    double params_bytes;    /* closed form, Psi/Nd real-valued */
    double grads_bytes;
    double optim_bytes;
    double total_bytes;
    int64_t params_bytes_padded; /* Psi/Nd replaced by the padded shard L */
    int64_t grads_bytes_padded;
    int64_t optim_bytes_padded;
    int64_t total_bytes_padded;
    double reduction;       /* 16 Psi / total_bytes */
    double comm_elems;      /* per process per step */
    double comm_bytes;      /* 2 bytes per fp16 element */
    double comm_elems_ring; /* derived: (Nd-1)/Nd of each collective */
} oracle_state_report;

int oracle_state_bytes(int64_t psi, int32_t nd, int32_t stage, int64_t align, oracle_state_report* r)
{
    if (!r || psi < 1 || nd < 1 || align < 1 || stage < 0 || stage > 3)
        return -1;
    oracle_plan_t p;
    oracle_plan(psi, nd, align, 0, &p);
    const double P = (double)psi, N = (double)nd;
    const int64_t L = p.shard_len;
    /* per-parameter byte costs: fp16 param 2, fp16 grad 2, Adam states 12 */
    const double Kp = 2.0, Kg = 2.0, Ko = 12.0;
    int part_os = stage >= 1, part_g = stage >= 2, part_p = stage >= 3;
    r->params_bytes = part_p ? Kp * P / N : Kp * P;
    r->grads_bytes = part_g ? Kg * P / N : Kg * P;
    r->optim_bytes = part_os ? Ko * P / N : Ko * P;
    r->total_bytes = r->params_bytes + r->grads_bytes + r->optim_bytes;
    r->params_bytes_padded = part_p ? 2 * L : 2 * psi;
    r->grads_bytes_padded = part_g ? 2 * L : 2 * psi;
    r->optim_bytes_padded = part_os ? 12 * L : 12 * psi;
    r->total_bytes_padded = r->params_bytes_padded + r->grads_bytes_padded + r->optim_bytes_padded;
    r->reduction = 16.0 * P / r->total_bytes;
    /* reduce-scatter Psi + all-gather Psi; stage 3 gathers twice */
    double n_collectives = part_p ? 3.0 : 2.0;
    r->comm_elems = n_collectives * P;
    r->comm_bytes = 2.0 * r->comm_elems;
    r->comm_elems_ring = r->comm_elems * (N - 1.0) / N;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Collectives, written out as their definitions                            */
/* ------------------------------------------------------------------------ */

/* Contribution of rank r at flat index i: rank r's 16-bit buffer starts
 * rank_stride elements after rank r-1's (storage 0: fp16, 1: bf16). */
static float contribution(const uint16_t* G, int64_t rank_stride, int32_t r, int64_t i, int32_t storage)
{
    const uint16_t h = G[(int64_t)r * rank_stride + i];
    return storage ? oracle_bf16_to_float(h) : oracle_half_to_float(h);
}

/* Sum over ranks 0..Nd-1 at index i, left to right in fp32. */
static float rank_sum_of(const uint16_t* G, int64_t rank_stride, int32_t nd, int64_t i, int32_t storage)
{
    float s = contribution(G, rank_stride, 0, i, storage);
    for (int32_t r = 1; r < nd; ++r)
        s = s + contribution(G, rank_stride, r, i, storage);
    return s;
}

static float rank_sum(const uint16_t* G, int64_t rank_stride, int32_t nd, int64_t i)
{
    return rank_sum_of(G, rank_stride, nd, i, 0);
}

/* The cast of an updated master value into the parameter format. */
static uint16_t to_storage(float p, int32_t storage)
{
    return storage ? oracle_float_to_bf16(p) : oracle_float_to_half(p);
}

/* All-reduce: every process ends with the full sum ([Note] Key results: DP's
 * all-reduce).  out[i] for i < n. */
void oracle_all_reduce(const uint16_t* G, int64_t rank_stride, int32_t nd, int64_t n, float* out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = rank_sum(G, rank_stride, nd, i);
}

/* Reduce-scatter: owner o receives the reduced values of its own slice only
 * ([Note] Concepts, Reduce-Scatter; [Dissect] "ZeRO-2").  shards is [Nd][L];
 * pad positions are written 0. */
void oracle_reduce_scatter(const uint16_t* G, int64_t rank_stride, const oracle_plan_t* p, float* shards)
{
    for (int32_t o = 0; o < p->nd; ++o) {
        int64_t start, len;
        oracle_shard(p, o, &start, &len);
        float* dst = shards + (int64_t)o * p->shard_len;
        for (int64_t i = 0; i < p->shard_len; ++i)
            dst[i] = i < len ? rank_sum(G, rank_stride, p->nd, start + i) : 0.0f;
    }
}

/* Reduce-scatter with retention (stage 2, P_os+g): each gradient element is
 * reduced only on the process that owns its partition, which keeps it, and
 * the ranks' full gradients are released ([Guide] "How it works"; [Dissect]
 * "ZeRO-2: Also Partition the Gradients").  What is kept is the reduced
 * gradient in the gradients' own 16-bit format (storage 0: fp16, 1: bf16):
 * the rank-order fp32 sum, rounded once.  shards is [Nd][L]; only the flat
 * range [lo, hi) is written (one bucket, or everything), pads never. */
void oracle_reduce_scatter16(const uint16_t* G, int64_t rank_stride, const oracle_plan_t* p, int32_t storage,
                             int64_t lo, int64_t hi, uint16_t* shards)
{
    for (int32_t o = 0; o < p->nd; ++o) {
        int64_t start, len;
        oracle_shard(p, o, &start, &len);
        uint16_t* dst = shards + (int64_t)o * p->shard_len;
        for (int64_t i = 0; i < len; ++i) {
            const int64_t f = start + i;
            if (f >= lo && f < hi)
                dst[i] = to_storage(rank_sum_of(G, rank_stride, p->nd, f, storage), storage);
        }
    }
}

/* All-gather of fp32 shards [Nd][L] into the flat [Psi] vector
 * ([Note] Method: all-gather rebuilds the full parameters after the update). */
void oracle_all_gather_f32(const float* shards, const oracle_plan_t* p, float* full)
{
    for (int32_t o = 0; o < p->nd; ++o) {
        int64_t start, len;
        oracle_shard(p, o, &start, &len);
        for (int64_t i = 0; i < len; ++i)
            full[start + i] = shards[(int64_t)o * p->shard_len + i];
    }
}

/* Gather-assembly of fp16 parameter shards: full[r*L + i] = shard_r[i] for
 * i < real_len_r, for every r whose pointer is not NULL ([Dissect]
 * "Forward/Backward Under ZeRO-3": a process gathers the parameter shards it
 * does not own).  Positions of NULL shards are left untouched. */
void oracle_gather_params(const uint16_t* const* shards, const oracle_plan_t* p, uint16_t* full)
{
    for (int32_t r = 0; r < p->nd; ++r) {
        if (!shards[r])
            continue;
        int64_t start, len;
        oracle_shard(p, r, &start, &len);
        for (int64_t i = 0; i < len; ++i)
            full[start + i] = shards[r][i];
    }
}

/* On-demand gather of a tensor range (stage 3: a layer's parameters are
 * gathered when the forward or backward pass reaches it, then released --
 * [Dissect] "ZeRO-3" and the figure under "Forward/Backward Under ZeRO-3").
 * Tensors first .. first + count - 1 of the flat layout (sizes as in
 * oracle_tensor_segments) are assembled from the owners' fp16 shards: the
 * element at flat index f comes from shards[f / L][f % L].  compact = 0: into
 * `out` at the flat index (a Psi-element buffer), where a NULL shard means
 * that owner's part is already in place and is left untouched; compact = 1:
 * tensors back to back from out[0], every needed shard required.  Returns
 * the number of elements copied, -1 on bad arguments (sizes not adding up to
 * Psi, range outside the list, or a shard missing in compact mode). */
int64_t oracle_gather_tensors(const oracle_plan_t* p, const int64_t* sizes, int32_t n_tensors,
                              int32_t first, int32_t count, const uint16_t* const* shards,
                              uint16_t* out, int32_t compact)
{
    int64_t total = 0;
    for (int32_t t = 0; t < n_tensors; ++t)
        total += sizes[t];
    if (total != p->psi || first < 0 || count < 0 || first + count > n_tensors)
        return -1;
    int64_t flat = 0, written = 0;
    for (int32_t t = 0; t < first; ++t)
        flat += sizes[t];
    for (int32_t t = first; t < first + count; ++t) {
        for (int64_t j = 0; j < sizes[t]; ++j) {
            const int64_t f = flat + j;
            const int64_t owner = f / p->shard_len;
            if (!shards[owner]) {
                if (compact)
                    return -1;
                continue;
            }
            out[compact ? written : f] = shards[owner][f - owner * p->shard_len];
            ++written;
        }
        flat += sizes[t];
    }
    return written;
}

/* ------------------------------------------------------------------------ */
/* The shard step                                                            */
/* ------------------------------------------------------------------------ */

typedef struct {
    float lr, beta1, beta2, eps, weight_decay;
    float loss_scale;    /* S: contributions carry the loss scaled by S */
    float max_grad_norm; /* <= 0: no clipping */
    int32_t average_over_nd;
    int32_t storage;     /* 16-bit format of gradients and parameters: 0 fp16, 1 bf16 */
} oracle_hparams;

typedef struct {
    int64_t t;        /* steps applied so far */
    double beta1_pow; /* beta1^t, fp64 running product, starts at 1 */
    double beta2_pow;
    /* Dynamic loss scaling (Micikevicius et al. 2018, "Mixed Precision
     * Training", section 3.2; the pages cite that paper only as background):
     * in use when loss_scale > 0, which then replaces the static S of the
     * hyper-parameters.  A skipped step multiplies the scale by
     * backoff_factor; growth_interval consecutive applied steps multiply it by
     * growth_factor.  good_steps counts the applied steps since the last
     * change. */
    float loss_scale;
    int32_t good_steps;
    float growth_factor;
    float backoff_factor;
    int32_t growth_interval;
    int32_t pad_;
} oracle_opt_state;

typedef struct {
    int32_t overflow;  /* 1: step skipped */
    float clip_coef;   /* coefficient the update used */
    double sumsq;      /* sum of squares of the unscaled reduced gradient */
    double grad_norm;  /* sqrt(sumsq) */
    float bc1, bc2;    /* 1 - beta^t of the applied step */
} oracle_step_info;

/* fp32 constants of the update, each rounded once. */
typedef struct {
    float beta1, beta2, one_minus_beta1, one_minus_beta2;
    float lr, lr_wd, eps, bc1, bc2, clip;
} adam_consts;

/* Compensated running sum (Neumaier 1974): s holds the sum, c the lost
 * low-order part; s + c is the total to within about one ulp, whatever the
 * number of terms. */
typedef struct {
    double s, c;
} comp_sum;

static void comp_add(comp_sum* a, double t)
{
    double y = a->s + t;
    if (fabs(a->s) >= fabs(t))
        a->c += (a->s - y) + t;
    else
        a->c += (t - y) + a->s;
    a->s = y;
}

/* Unscale factor: fp32 reciprocal of S (times 1/Nd when averaging). */
static float unscale_factor_of(float loss_scale, int32_t average, int32_t nd)
{
    double d = (double)loss_scale;
    if (average)
        d *= (double)nd;
    return (float)(1.0 / d);
}

static float unscale_factor(const oracle_hparams* hp, int32_t nd)
{
    return unscale_factor_of(hp->loss_scale, hp->average_over_nd, nd);
}

/* The loss scale a step divides by: the dynamic one when in use. */
static float step_loss_scale(const oracle_hparams* hp, const oracle_opt_state* st)
{
    return st->loss_scale > 0.0f ? st->loss_scale : hp->loss_scale;
}

/* Dynamic loss scaling after a step: back off on a skip, grow after
 * growth_interval consecutive applied steps (fp32 products). */
static void advance_loss_scale(oracle_opt_state* st, int32_t skipped)
{
    if (!(st->loss_scale > 0.0f))
        return;
    if (skipped) {
        st->loss_scale = st->loss_scale * st->backoff_factor;
        st->good_steps = 0;
    } else if (++st->good_steps >= st->growth_interval) {
        st->loss_scale = st->loss_scale * st->growth_factor;
        st->good_steps = 0;
    }
}

/* Mixed-precision Adam/AdamW on one element (Kingma & Ba 2015, Alg. 1;
 * decoupled decay per Loshchilov & Hutter 2019).  The fp32 master copy,
 * momentum and variance are the 12 bytes of Adam state per parameter of
 * [Dissect] "The Real Problem"; each owner updates only its own slice
 * ([Guide] "How it works"; [Dissect] "Forward/Backward Under ZeRO-3"). */
static void adam_element(float g, float* p, float* m, float* v, const adam_consts* k)
{
    float m_new = k->beta1 * *m + k->one_minus_beta1 * g;
    float v_new = k->beta2 * *v + k->one_minus_beta2 * (g * g);
    float m_hat = m_new / k->bc1;
    float v_hat = v_new / k->bc2;
    float denom = sqrtf(v_hat) + k->eps;
    float p_old = *p;
    float p_new = (p_old - k->lr_wd * p_old) - k->lr * (m_hat / denom);
    *m = m_new;
    *v = v_new;
    *p = p_new;
}

static void fill_consts(const oracle_hparams* hp, float bc1, float bc2, float clip, adam_consts* k)
{
    k->beta1 = hp->beta1;
    k->beta2 = hp->beta2;
    k->one_minus_beta1 = 1.0f - hp->beta1;
    k->one_minus_beta2 = 1.0f - hp->beta2;
    k->lr = hp->lr;
    k->lr_wd = hp->lr * hp->weight_decay;
    k->eps = hp->eps;
    k->bc1 = bc1;
    k->bc2 = bc2;
    k->clip = clip;
}

/* Bias corrections of step t+1: advance beta^t in fp64, round 1 - beta^t. */
void oracle_bias_corrections(const oracle_hparams* hp, const oracle_opt_state* st,
                             double* b1p_next, double* b2p_next, float* bc1, float* bc2)
{
    double b1 = st->beta1_pow * (double)hp->beta1;
    double b2 = st->beta2_pow * (double)hp->beta2;
    *b1p_next = b1;
    *b2p_next = b2;
    *bc1 = (float)(1.0 - b1);
    *bc2 = (float)(1.0 - b2);
}

/* The update applied to n elements whose global quantities (clip coefficient,
 * bias corrections) are already known: reduce in rank order, unscale, clip,
 * Adam, cast to fp16.  G/rank_stride address the n elements' contributions;
 * master, m, v, params are the same n elements.  Used by oracle_step and, on
 * sampled elements of large problems, directly by the tests. */
void oracle_update_elements(const uint16_t* G, int64_t rank_stride, int32_t nd, int64_t n,
                            float* master, float* exp_avg, float* exp_avg_sq, uint16_t* params,
                            const oracle_hparams* hp, float clip_coef, float bc1, float bc2,
                            int threads)
{
    adam_consts k;
    fill_consts(hp, bc1, bc2, clip_coef, &k);
    const float inv = unscale_factor(hp, nd);
    (void)threads;
#pragma omp parallel for num_threads(threads > 0 ? threads : 1) if (threads > 1) schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        float g = rank_sum_of(G, rank_stride, nd, i, hp->storage) * inv;
        float g_hat = g * k.clip;
        adam_element(g_hat, &master[i], &exp_avg[i], &exp_avg_sq[i], &k);
        params[i] = to_storage(master[i], hp->storage);
    }
}

/* One full step over the flat buffer of Psi real elements (all owners).
 * G: Nd fp16 gradient buffers, rank r at G + r*rank_stride (rank_stride >=
 * psi).  master/exp_avg/exp_avg_sq: fp32 [psi]; params: fp16 [psi], the
 * all-gathered layout.  If use_clip_override, clip_override replaces the
 * computed clip coefficient (tests feed in another implementation's fp32
 * coefficient so a one-ulp difference in the norm cannot cascade).
 * Returns 0, or -1 on bad arguments / allocation failure. */
int oracle_step(const uint16_t* G, int64_t rank_stride, int32_t nd, int64_t psi,
                float* master, float* exp_avg, float* exp_avg_sq, uint16_t* params,
                const oracle_hparams* hp, oracle_opt_state* st,
                int32_t use_clip_override, float clip_override, int threads,
                oracle_step_info* info)
{
    if (!G || !master || !exp_avg || !exp_avg_sq || !params || !hp || !st || !info)
        return -1;
    if (nd < 1 || psi < 1 || (nd > 1 && rank_stride < psi))
        return -1;
    float* g = (float*)malloc((size_t)psi * sizeof(float));
    if (!g)
        return -1;
    const float inv = unscale_factor_of(step_loss_scale(hp, st), hp->average_over_nd, nd);

    /* 1. reduce-scatter sum (every owner's slice) and unscale */
#pragma omp parallel for num_threads(threads > 0 ? threads : 1) if (threads > 1) schedule(static)
    for (int64_t i = 0; i < psi; ++i)
        g[i] = rank_sum_of(G, rank_stride, nd, i, hp->storage) * inv;

    /* 2. overflow: one non-finite element anywhere skips the whole step */
    int32_t overflow = 0;
    for (int64_t i = 0; i < psi; ++i) {
        if (!isfinite(g[i])) {
            overflow = 1;
            break;
        }
    }
    memset(info, 0, sizeof *info);
    info->overflow = overflow;
    if (overflow) {
        info->clip_coef = 1.0f;
        info->grad_norm = NAN;
        info->sumsq = NAN;
        advance_loss_scale(st, 1);
        free(g);
        return 0;
    }

    /* 3. global L2 norm: the exact fp64 squares, summed with compensation;
     * clip coefficient */
    comp_sum acc = {0.0, 0.0};
    for (int64_t i = 0; i < psi; ++i)
        comp_add(&acc, (double)g[i] * (double)g[i]);
    double sumsq = acc.s + acc.c;
    double norm = sqrt(sumsq);
    float clip = 1.0f;
    if (hp->max_grad_norm > 0.0f && norm > (double)hp->max_grad_norm)
        clip = (float)((double)hp->max_grad_norm / norm);
    if (use_clip_override)
        clip = clip_override;

    /* 4. bias corrections of this step; advance the step counter */
    double b1p, b2p;
    float bc1, bc2;
    oracle_bias_corrections(hp, st, &b1p, &b2p, &bc1, &bc2);

    /* 5-6. Adam on every element, then the fp16 cast into the full buffer */
    adam_consts k;
    fill_consts(hp, bc1, bc2, clip, &k);
#pragma omp parallel for num_threads(threads > 0 ? threads : 1) if (threads > 1) schedule(static)
    for (int64_t i = 0; i < psi; ++i) {
        float g_hat = g[i] * k.clip;
        adam_element(g_hat, &master[i], &exp_avg[i], &exp_avg_sq[i], &k);
        params[i] = to_storage(master[i], hp->storage);
    }

    st->t += 1;
    st->beta1_pow = b1p;
    st->beta2_pow = b2p;
    advance_loss_scale(st, 0);
    info->clip_coef = clip;
    info->sumsq = sumsq;
    info->grad_norm = norm;
    info->bc1 = bc1;
    info->bc2 = bc2;
    free(g);
    return 0;
}

/* Sum of squares of the unscaled reduced gradient over n elements (the same
 * compensated fp64 sum as oracle_step), added into the Neumaier accumulator
 * acc = {running sum, compensation}, which is updated in place and may carry
 * over from earlier pieces.  A caller that streams a large problem through in
 * pieces and passes the same acc along gets exactly the single-pass sum (the
 * same additions in the same order); pieces summed with separate accumulators
 * stay exact when their sum and compensation terms are added exactly (for
 * instance with Python's math.fsum).  Returns acc[0] + acc[1].  *nonfinite is
 * set to 1 if any reduced element is non-finite. */
double oracle_grad_sumsq(const uint16_t* G, int64_t rank_stride, int32_t nd, int64_t n,
                         const oracle_hparams* hp, double acc[2], int32_t* nonfinite)
{
    const float inv = unscale_factor(hp, nd);
    comp_sum a = {acc[0], acc[1]};
    for (int64_t i = 0; i < n; ++i) {
        float g = rank_sum_of(G, rank_stride, nd, i, hp->storage) * inv;
        if (!isfinite(g))
            *nonfinite = 1;
        comp_add(&a, (double)g * (double)g);
    }
    acc[0] = a.s;
    acc[1] = a.c;
    return a.s + a.c;
}
