// static_scratch.cu -- zero_shard_step_static_scratch: the shard step with its
// scratch memory in a fixed device array owned by the library, for callers
// that cannot allocate device memory themselves.
//
// The array below is created with the library's device code on every GPU
// that loads it and lives until the process exits (or until the context
// holding it is destroyed).  Host code cannot use the symbol's name as a
// device address, so the address is resolved with the device current,
// through cudaGetSymbolAddress, and handed to the kernels like a
// caller-provided workspace.  The resolved address is cached per device and
// per context: a context created after a reset of the device (which reloads
// the module, so the array may move) has a new unique id and resolves the
// address again instead of reusing a stale one.
#include <cuda.h> // driver types only: the two driver calls are looked up at run time

#include <map>
#include <mutex>
#include <utility>

#include "zs_internal.h"

namespace {

__device__ __align__(256) unsigned char zs_static_scratch[ZERO_STATIC_SCRATCH_BYTES];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

std::mutex g_scratch_mu;
std::map<std::pair<int, unsigned long long>, void*> g_scratch_addr; // (device, context id) -> address
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;

// Unique id of the context current on this thread, 0 when none is current.
// Ids are never reused within a process.  Caller holds g_scratch_mu.
zero_status current_context_id(unsigned long long* id)
{
    *id = 0;
    if (!g_ctx_get_current || !g_ctx_get_id) {
        cudaDriverEntryPointQueryResult q1 = cudaDriverEntryPointSymbolNotFound, q2 = q1;
        void* f1 = nullptr;
        void* f2 = nullptr;
        const cudaError_t e1 = cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f1, 12000, cudaEnableDefault, &q1);
        const cudaError_t e2 = cudaGetDriverEntryPointByVersion("cuCtxGetId", &f2, 12000, cudaEnableDefault, &q2);
        if (e1 != cudaSuccess || e2 != cudaSuccess || q1 != cudaDriverEntryPointSuccess ||
            q2 != cudaDriverEntryPointSuccess || !f1 || !f2)
            return zs::fail(ZERO_ERR_CUDA, "zero_shard_step_static_scratch: the driver's context queries are "
                            "not available (%s)", cudaGetErrorString(e1 != cudaSuccess ? e1 : e2));
        g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
        g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(f2);
    }
    CUcontext ctx = nullptr;
    if (g_ctx_get_current(&ctx) != CUDA_SUCCESS)
        return zs::fail(ZERO_ERR_CUDA, "zero_shard_step_static_scratch: cuCtxGetCurrent failed");
    if (ctx && g_ctx_get_id(ctx, id) != CUDA_SUCCESS)
        return zs::fail(ZERO_ERR_CUDA, "zero_shard_step_static_scratch: cuCtxGetId failed");
    return ZERO_OK;
}

zero_status static_scratch_address(void** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return zs::fail(ZERO_ERR_CUDA, "zero_shard_step_static_scratch: cudaGetDevice: %s",
                        cudaGetErrorString(e));
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    unsigned long long ctx = 0;
    zero_status s = current_context_id(&ctx);
    if (s != ZERO_OK)
        return s;
    if (ctx != 0) {
        auto it = g_scratch_addr.find({dev, ctx});
        if (it != g_scratch_addr.end()) {
            *out = it->second;
            return ZERO_OK;
        }
    }
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, zs_static_scratch); // makes the device's primary context current if none is
    if (e != cudaSuccess || p == nullptr)
        return zs::fail(ZERO_ERR_CUDA,
                        "zero_shard_step_static_scratch: cudaGetSymbolAddress of the static "
                        "scratch failed on device %d: %s", dev, cudaGetErrorString(e));
    if (ctx == 0 && (s = current_context_id(&ctx)) != ZERO_OK)
        return s;
    if (ctx != 0)
        g_scratch_addr[{dev, ctx}] = p;
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
