// peer.cpp -- mapping other processes' device buffers into this one (CUDA IPC)
// so that a step's kernels can load the ranks' gradients and store the
// parameters of every rank directly (the peer tables of zero_step_args).
// Nothing here allocates device memory: an export names an existing
// allocation, an open maps one that another process owns.
#include <cstring>
#include <map>
#include <mutex>
#include <string>

#include "zs_internal.h"

using zs::fail;

namespace {

static_assert(sizeof(cudaIpcMemHandle_t) == sizeof(((zero_ipc_handle*)nullptr)->handle),
              "zero_ipc_handle must hold a cudaIpcMemHandle_t");

// cuMemGetAddressRange through the runtime's driver entry point (no link
// against the driver library): the allocation that holds a pointer.
using AddressRangeFn = int (*)(unsigned long long* base, size_t* size, unsigned long long ptr);

zero_status allocation_base(const void* ptr, const char** base)
{
    static std::once_flag once;
    static AddressRangeFn fn = nullptr;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<AddressRangeFn>(f);
    });
    if (!fn)
        return fail(ZERO_ERR_CUDA, "zero_ipc_export: cuMemGetAddressRange is not available");
    unsigned long long b = 0;
    size_t size = 0;
    const int rc = fn(&b, &size, reinterpret_cast<unsigned long long>(ptr));
    if (rc != 0)
        return fail(ZERO_ERR_INVALID_ARG, "zero_ipc_export: %p is not inside a device allocation (driver error %d)",
                    ptr, rc);
    *base = reinterpret_cast<const char*>(b);
    return ZERO_OK;
}

// Open mappings, reference counted per exported allocation: a process may
// map several buffers of one peer allocation, which CUDA opens only once.
struct Mapping {
    char* base = nullptr;
    int refs = 0;
};

std::mutex g_mu;
std::map<std::string, Mapping> g_by_handle;      // handle bytes -> mapping
struct Address {
    std::string key; // handle bytes of the mapping
    int opens = 0;   // zero_ipc_open calls that returned this address
};
std::map<const void*, Address> g_by_address;

} // namespace

extern "C" {

zero_status zero_ipc_export(const void* dev_ptr, zero_ipc_handle* out)
{
    zs::clear_error();
    if (!dev_ptr || !out)
        return fail(ZERO_ERR_INVALID_ARG, "zero_ipc_export: null argument");
    cudaPointerAttributes attr;
    cudaError_t e = cudaPointerGetAttributes(&attr, dev_ptr);
    if (e != cudaSuccess || attr.type != cudaMemoryTypeDevice) {
        cudaGetLastError();
        return fail(ZERO_ERR_INVALID_ARG, "zero_ipc_export: %p is not device memory", dev_ptr);
    }
    const char* base = nullptr;
    zero_status s = allocation_base(dev_ptr, &base);
    if (s != ZERO_OK)
        return s;
    cudaIpcMemHandle_t h;
    if ((e = cudaIpcGetMemHandle(&h, const_cast<char*>(base))) != cudaSuccess)
        return fail(ZERO_ERR_CUDA, "zero_ipc_export: cudaIpcGetMemHandle: %s", cudaGetErrorString(e));
    std::memset(out, 0, sizeof *out);
    std::memcpy(out->handle, &h, sizeof h);
    out->offset = static_cast<const char*>(dev_ptr) - base;
    out->device = attr.device;
    return ZERO_OK;
}

zero_status zero_ipc_open(const zero_ipc_handle* h, void** dev_ptr)
{
    zs::clear_error();
    if (!h || !dev_ptr)
        return fail(ZERO_ERR_INVALID_ARG, "zero_ipc_open: null argument");
    if (h->offset < 0)
        return fail(ZERO_ERR_INVALID_ARG, "zero_ipc_open: negative offset");
    const std::string key(reinterpret_cast<const char*>(h->handle), sizeof h->handle);
    std::lock_guard<std::mutex> lk(g_mu);
    Mapping& m = g_by_handle[key];
    if (m.refs == 0) {
        cudaIpcMemHandle_t ih;
        std::memcpy(&ih, h->handle, sizeof ih);
        void* base = nullptr;
        const cudaError_t e = cudaIpcOpenMemHandle(&base, ih, cudaIpcMemLazyEnablePeerAccess);
        if (e != cudaSuccess) {
            cudaGetLastError();
            g_by_handle.erase(key);
            return fail(ZERO_ERR_CUDA, "zero_ipc_open: cudaIpcOpenMemHandle: %s", cudaGetErrorString(e));
        }
        m.base = static_cast<char*>(base);
    }
    m.refs += 1;
    char* p = m.base + h->offset;
    Address& ad = g_by_address[p];
    ad.key = key;
    ad.opens += 1;
    *dev_ptr = p;
    return ZERO_OK;
}

zero_status zero_ipc_close(void* dev_ptr)
{
    zs::clear_error();
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_by_address.find(dev_ptr);
    if (it == g_by_address.end())
        return fail(ZERO_ERR_INVALID_ARG, "zero_ipc_close: %p was not returned by zero_ipc_open", dev_ptr);
    auto mt = g_by_handle.find(it->second.key);
    if (--it->second.opens == 0)
        g_by_address.erase(it);
    if (mt == g_by_handle.end() || --mt->second.refs > 0)
        return ZERO_OK;
    char* base = mt->second.base;
    g_by_handle.erase(mt);
    const cudaError_t e = cudaIpcCloseMemHandle(base);
    if (e != cudaSuccess)
        return fail(ZERO_ERR_CUDA, "zero_ipc_close: cudaIpcCloseMemHandle: %s", cudaGetErrorString(e));
    return ZERO_OK;
}

} // extern "C"
