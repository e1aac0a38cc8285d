// gather.cu -- K4: gather-assembly of 16-bit parameter shards (the stage-3
// all-gather as one rank sees it, and the on-demand gathering of tensor
// ranges).  A pure copy: 2 bytes read and 2 written per assembled parameter.
#include "zs_internal.h"
#include "zs_launch.h"

namespace zs {

constexpr int kGatherWaves = 8;               // grid: up to this many times the resident blocks
constexpr int kGatherMinUnitsPerThread = 16;  // ... while every thread keeps at least this many units

// STREAM: evict-first loads and stores.  Measured: they suit the compact
// per-layer gathers, whose two small buffers are rewritten every other layer
// (0.90 of the copy peak against 0.86-0.88 with plain stores); plain
// write-back stores suit the assembly of a full parameter buffer (0.94
// against 0.92).
template <bool STREAM>
__global__ void __launch_bounds__(kThreads)
zs_gather_kernel(uint16_t* dst, const __grid_constant__ GatherList g)
{
    // The pieces' units -- 8-element vectors for aligned pieces, single
    // elements otherwise -- form one grid-stride index space; g.first[k] is
    // the first unit of piece k and g.first[g.count] the total.  A thread
    // finds the piece of its first unit by binary search and then only
    // moves forward, so its set-up does not grow with the piece count.
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t nthr = (int64_t)gridDim.x * blockDim.x;
    const int64_t total = g.first[g.count];
    int64_t u = tid;
    if (u < total) {
        int lo = 0, hi = g.count - 1; // the last piece whose first unit is <= u
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (g.first[mid] <= u)
                lo = mid;
            else
                hi = mid - 1;
        }
        int k = lo;
        for (; u < total; u += nthr) {
            while (u >= g.first[k + 1])
                ++k;
            const GatherEntry& ge = g.e[k];
            const int64_t i = u - g.first[k];
            if (ge.vec) {
                uint4* to = reinterpret_cast<uint4*>(dst + ge.dst_off) + i;
                const uint4* from = reinterpret_cast<const uint4*>(ge.src + (i << 3));
                if (STREAM)
                    __stcs(to, __ldcs(from));
                else
                    *to = *from;
            } else {
                dst[ge.dst_off + i] = ge.src[i];
            }
        }
    }
    if (tid < 8) { // the < 8-element tails of the vector pieces
        for (int j = 0; j < g.count; ++j) {
            const GatherEntry& ge = g.e[j];
            const int64_t e = ((ge.n >> 3) << 3) + tid;
            if (ge.vec && e < ge.n)
                dst[ge.dst_off + e] = ge.src[e];
        }
    }
}

cudaError_t launch_gather(uint16_t* dst, const GatherList& pieces, bool streaming_stores, cudaStream_t s)
{
    GatherList g = pieces;
    int64_t w = 0;
    for (int i = 0; i < g.count; ++i) {
        g.first[i] = w;
        w += g.e[i].vec ? g.e[i].n >> 3 : g.e[i].n;
    }
    g.first[g.count] = w;
    auto kernel = streaming_stores ? zs_gather_kernel<true> : zs_gather_kernel<false>;
    int blocks = 0;
    cudaError_t e = grid_for(kernel, w, 0, &blocks);
    if (e != cudaSuccess)
        return e;
    // A copy of equal read and write streams runs faster with a grid of
    // several times the resident blocks (blocks of later waves start where
    // earlier ones finished): the 63-shard assembly of a 7.5B buffer measured
    // 0.97 of the copy bandwidth at 8 waves against 0.94-0.95 with one.
    // Small gathers (a per-layer gather of a few million units) keep one wave.
    const int64_t by_work = w / ((int64_t)kThreads * kGatherMinUnitsPerThread);
    int64_t grid = by_work < (int64_t)blocks * kGatherWaves ? by_work : (int64_t)blocks * kGatherWaves;
    grid = grid > blocks ? grid : blocks;
    return launch_plain(kernel, (unsigned)(grid < 1 ? 1 : grid), kThreads, 0, s, dst, g);
}

} // namespace zs
