// Block-sparse attention without a caller workspace, for callers that cannot hand the library
// any extra device memory.
//
// sa_block_sparse_attn_fwd needs a few bytes of device scratch (the counter from which CTAs
// claim query blocks), and it asks the caller for them.  Some callers cannot do that: their
// device memory belongs to another runtime's allocator and they have no spare buffer to lend,
// or they must not call cudaMalloc on the path that invokes attention (it can synchronise the
// device and is not available inside every host framework).  This variant keeps the scratch in
// a fixed-size array in the library's own device image instead, so nothing is allocated.
//
// The scratch below is a file-scope __device__ array: every GPU that loads the library holds
// one copy until the process exits.  Host code must not use its name as an address (on the host
// it is only a stand-in symbol); the device address is obtained with cudaGetSymbolAddress, with
// the device current, once per device context, and passed to the kernel.  A context that is
// destroyed and created again (cudaDeviceReset, or the primary context released and retained)
// loads the module again and may place the array elsewhere, so the cached address is keyed on
// the current context's unique id and resolved again when that id changes.
#include <cudaTypedefs.h>

#include <mutex>

#include "bsa_internal.h"
#include "sparse_attn.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 256;  // maximum scratch this variant provides
static __device__ __align__(256) unsigned char g_bsa_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
struct ScratchAddr {
    unsigned long long ctx_id;  // unique id of the context the address belongs to
    void *ptr;
};
ScratchAddr g_noalloc[kMaxDevices] = {};
std::mutex g_noalloc_mutex;

// Unique id of the current context (cuCtxGetId through the runtime's driver entry point), or
// false when it cannot be read; the caller then resolves the address on every call.
bool current_ctx_id(unsigned long long *id) {
    static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static bool looked = false;
    if (!looked) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
        p = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
        looked = true;
    }
    if (!get_cur || !get_id) return false;
    CUcontext ctx = nullptr;
    if (get_cur(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch array on device `dev` (which must be current).  The first call
// in a device context resolves it; later calls in the same context reuse the cached address.
sa_status noalloc_scratch(int dev, void **out) {
    if (dev < 0 || dev >= kMaxDevices) return SA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    // the caller's output buffer was found to be memory of this device, so its context is
    // current here
    unsigned long long id = 0;
    const bool have_id = current_ctx_id(&id);
    if (!have_id || !g_noalloc[dev].ptr || g_noalloc[dev].ctx_id != id) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_bsa_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            g_noalloc[dev].ptr = nullptr;
            return SA_ERR_CUDA;
        }
        g_noalloc[dev].ptr = p;
        g_noalloc[dev].ctx_id = have_id ? id : 0;
    }
    *out = g_noalloc[dev].ptr;
    return SA_OK;
}

}  // namespace

extern "C" sa_status sa_block_sparse_attn_fwd_noalloc(const void *q, const void *k, const void *v,
                                                      const int32_t *kv_idx,
                                                      const int32_t *kv_cnt, void *o, int B,
                                                      int H, int N, int d, int bs, float scale,
                                                      void *stream) {
    // the same host-side checks as the workspace entry point, before any device work
    const sa_status a = check_sparse_attn_args(q, k, v, kv_idx, kv_cnt, o, B, H, N, d, bs, scale);
    if (a != SA_OK) return a;
    // the scratch this call needs must fit in the fixed array
    if (sa_attn_workspace_bytes() > kNoAllocScratchBytes) return SA_ERR_UNSUPPORTED;
    int dev;
    if (!select_device(o, &dev)) return SA_ERR_INVALID_ARG;
    void *scratch = nullptr;
    const sa_status st = noalloc_scratch(dev, &scratch);
    if (st != SA_OK) return st;
    // the counter is zeroed on `stream` before the kernel, as in the workspace entry point
    return sa_block_sparse_attn_fwd(q, k, v, kv_idx, kv_cnt, o, B, H, N, d, bs, scale, scratch,
                                    kNoAllocScratchBytes, stream);
}
