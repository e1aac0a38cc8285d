// zs_launch.h -- launch helpers shared by the kernel files of libzero_shard.so
// (kernels.cu, gather.cu).  Not part of the public ABI.
#pragma once

#include <cstdint>

#include <cuda_runtime.h>

#include "zs_internal.h"

namespace zs {

// SM count of the current device (cached per device).
cudaError_t device_sms(int* sms);
// Resident blocks per SM of `kernel` at kThreads threads and no dynamic shared
// memory on the current device (cached per kernel and device).
cudaError_t blocks_per_sm(const void* kernel, int* occ);

// Persistent grid: SM count x resident blocks, but no more blocks than work
// (and no more than cap when cap > 0).
template <typename K>
cudaError_t grid_for(K kernel, int64_t work_threads, int cap, int* blocks)
{
    int sms = 0, occ = 0;
    cudaError_t e = device_sms(&sms);
    if (e != cudaSuccess || (e = blocks_per_sm(reinterpret_cast<const void*>(kernel), &occ)) != cudaSuccess)
        return e;
    const int64_t want = (work_threads + kThreads - 1) / kThreads;
    int64_t full = (int64_t)sms * occ;
    if (cap > 0 && full > cap)
        full = cap;
    *blocks = (int)(want < 1 ? 1 : (want < full ? want : full));
    return cudaSuccess;
}

// Every kernel launch of the library goes through here.  overlapped: with
// programmatic stream serialization, so the kernel may begin while its
// predecessor in the stream drains (it orders itself with
// griddepcontrol.wait); used for the kernels after the first of a step.
// While a prepare call is running (zs::preparing()) the kernel is only
// loaded -- the caller has already resolved its geometry -- and nothing is
// enqueued or counted.
template <typename... Params, typename... Args>
cudaError_t launch_k(bool overlapped, void (*kernel)(Params...), unsigned grid, unsigned block, size_t smem,
                     cudaStream_t s, Args... args)
{
    if (preparing()) {
        cudaFuncAttributes fa;
        return cudaFuncGetAttributes(&fa, reinterpret_cast<const void*>(kernel));
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = overlapped ? 1 : 0;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<Params>(args)...);
    if (e == cudaSuccess) {
        count_launches(1);
        record_launch(reinterpret_cast<const void*>(kernel));
    }
    return e;
}

template <typename... Params, typename... Args>
cudaError_t launch_overlapped(void (*kernel)(Params...), unsigned grid, unsigned block, size_t smem,
                              cudaStream_t s, Args... args)
{
    return launch_k(true, kernel, grid, block, smem, s, args...);
}

template <typename... Params, typename... Args>
cudaError_t launch_plain(void (*kernel)(Params...), unsigned grid, unsigned block, size_t smem, cudaStream_t s,
                         Args... args)
{
    return launch_k(false, kernel, grid, block, smem, s, args...);
}

} // namespace zs
