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
// it is only a stand-in symbol); the device address is obtained with cudaGetSymbolAddress once
// per device, with that device current, and passed to the kernel.
#include <mutex>

#include "bsa_internal.h"
#include "sparse_attn.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 256;  // maximum scratch this variant provides
static __device__ __align__(256) unsigned char g_bsa_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void *g_noalloc_ptr[kMaxDevices] = {nullptr};
std::mutex g_noalloc_mutex;

// Device address of the scratch array on device `dev` (which must be current).  The first call
// on a device resolves it; later calls reuse the cached address.
sa_status noalloc_scratch(int dev, void **out) {
    if (dev < 0 || dev >= kMaxDevices) return SA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_bsa_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return SA_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return SA_OK;
}

}  // namespace

extern "C" sa_status sa_block_sparse_attn_fwd_noalloc(const void *q, const void *k, const void *v,
                                                      const int32_t *kv_idx,
                                                      const int32_t *kv_cnt, void *o, int B,
                                                      int H, int N, int d, int bs, float scale,
                                                      void *stream) {
    // the scratch this call needs must fit in the fixed array
    if (sa_attn_workspace_bytes() > kNoAllocScratchBytes) return SA_ERR_UNSUPPORTED;
    if (!o) return SA_ERR_INVALID_ARG;
    int dev;
    if (!select_device(o, &dev)) return SA_ERR_INVALID_ARG;
    void *scratch = nullptr;
    const sa_status st = noalloc_scratch(dev, &scratch);
    if (st != SA_OK) return st;
    // the counter is zeroed on `stream` before the kernel, as in the workspace entry point
    return sa_block_sparse_attn_fwd(q, k, v, kv_idx, kv_cnt, o, B, H, N, d, bs, scale, scratch,
                                    kNoAllocScratchBytes, stream);
}
