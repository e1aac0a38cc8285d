// static_scratch.cu -- zero_shard_step_static_scratch: the shard step with its
// scratch memory in a fixed device array owned by the library, for callers
// that cannot allocate device memory themselves.
//
// The array below is created with the library's device code on every GPU
// that loads it and lives until the process exits.  Host code cannot use the
// symbol's name as a device address, so the address is resolved once per
// device, with that device current, through cudaGetSymbolAddress, cached,
// and handed to the kernels like a caller-provided workspace.
#include <map>
#include <mutex>

#include "zs_internal.h"

namespace {

__device__ __align__(256) unsigned char zs_static_scratch[ZERO_STATIC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
std::map<int, void*> g_scratch_addr; // device ordinal -> address of zs_static_scratch

zero_status static_scratch_address(void** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return zs::fail(ZERO_ERR_CUDA, "zero_shard_step_static_scratch: cudaGetDevice: %s",
                        cudaGetErrorString(e));
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    auto it = g_scratch_addr.find(dev);
    if (it != g_scratch_addr.end()) {
        *out = it->second;
        return ZERO_OK;
    }
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, zs_static_scratch);
    if (e != cudaSuccess || p == nullptr)
        return zs::fail(ZERO_ERR_CUDA,
                        "zero_shard_step_static_scratch: cudaGetSymbolAddress of the static "
                        "scratch failed on device %d: %s", dev, cudaGetErrorString(e));
    g_scratch_addr[dev] = p;
    *out = p;
    return ZERO_OK;
}

} // namespace

extern "C" zero_status zero_shard_step_static_scratch(const zero_plan_t* plan,
                                                      const zero_hparams* hp,
                                                      const zero_step_args* args, void* stream)
{
    zs::clear_error();
    if (!args)
        return zs::fail(ZERO_ERR_INVALID_ARG, "zero_shard_step_static_scratch: null args");
    zero_step_args a = *args;
    a.workspace = nullptr;
    a.workspace_bytes = 0;
    size_t need = 0;
    zero_status s = zero_workspace_bytes(plan, hp, &a, &need); // validates; touches no device
    if (s != ZERO_OK)
        return s;
    if (need > (size_t)ZERO_STATIC_SCRATCH_BYTES)
        return zs::fail(ZERO_ERR_WORKSPACE,
                        "zero_shard_step_static_scratch: this call needs %zu bytes of scratch but "
                        "the library's static scratch holds %d; pass a workspace to "
                        "zero_shard_step instead", need, (int)ZERO_STATIC_SCRATCH_BYTES);
    void* p = nullptr;
    if ((s = static_scratch_address(&p)) != ZERO_OK)
        return s;
    a.workspace = p;
    a.workspace_bytes = (size_t)ZERO_STATIC_SCRATCH_BYTES;
    return zero_shard_step(plan, hp, &a, stream);
}
