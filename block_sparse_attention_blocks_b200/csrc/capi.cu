// C ABI of libbsa: argument validation, device selection, tensor-map encoding and launches.
// Every check happens on the host before anything is launched; see include/sparse_attn.h for
// the contract of each entry point.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <cudaTypedefs.h>

#include "bsa_internal.h"
#include "sparse_attn.h"

namespace {

constexpr unsigned long long kDefaultWaitNs = 2000000000ull;
unsigned long long g_wait_ns = kDefaultWaitNs;
unsigned int *g_progress = nullptr;  // host-mapped stage words of the attention kernel, or null

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// int32 / fp32 buffers read and written element by element
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

bool shape_ok(int B, int H, int N) {
    if (B < 1 || H < 1 || N < 1) return false;
    const long long BH = (long long)B * H;
    return BH <= 65535;
}

bool dims_supported(int d, int bs) { return (d == 64 || d == 128) && (bs == 64 || bs == 128); }

float resolve_scale(float scale, int d) { return scale > 0.f ? scale : 1.0f / sqrtf((float)d); }

// Run on the device that owns `p` (a device pointer).  Returns false if p is not device memory.
bool select_device(const void *p, int *dev_out) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) return false;
    int cur = -1;
    cudaGetDevice(&cur);
    if (cur != a.device && cudaSetDevice(a.device) != cudaSuccess) return false;
    *dev_out = a.device;
    return true;
}

int num_sms(int dev) {
    static int cache[64] = {0};
    if (dev >= 0 && dev < 64 && cache[dev]) return cache[dev];
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (dev >= 0 && dev < 64) cache[dev] = n;
    return n;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// [BH, N, d] bf16 viewed as a 3-D tensor (d innermost); boxes of 64 columns x box_rows rows,
// 128-byte swizzle (the layout the tcgen05 descriptors expect), zero fill out of bounds.
bool make_tmap(CUtensorMap *m, const void *base, long long BH, int N, int d, int box_rows) {
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)N * d * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                     box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

sa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? SA_OK : SA_ERR_CUDA; }

constexpr size_t kAttnWorkspaceBytes = 256;

// Host-side argument checks of the block-sparse attention entry points (no device work).
sa_status check_sparse_attn_args(const void *q, const void *k, const void *v,
                                 const int32_t *kv_idx, const int32_t *kv_cnt, const void *o,
                                 int B, int H, int N, int d, int bs, float scale) {
    if (!q || !k || !v || !kv_idx || !kv_cnt || !o || !shape_ok(B, H, N)) return SA_ERR_INVALID_ARG;
    if (!dims_supported(d, bs)) return SA_ERR_UNSUPPORTED;
    if (sa_num_blocks(N, bs) > 1024) return SA_ERR_UNSUPPORTED;
    if (isnan(scale)) return SA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return SA_ERR_INVALID_ARG;
    return SA_OK;
}

sa_status run_attention(const void *q, const void *k, const void *v, const int32_t *kv_idx,
                        const int32_t *kv_cnt, void *o, int B, int H, int N, int d, int bs,
                        float scale, void *workspace, void *stream) {
    int dev;
    if (!select_device(o, &dev)) return SA_ERR_INVALID_ARG;
    const long long BH = (long long)B * H;
    CUtensorMap tq, tk, tv;
    if (!make_tmap(&tq, q, BH, N, d, 128) || !make_tmap(&tk, k, BH, N, d, bs) ||
        !make_tmap(&tv, v, BH, N, d, bs))
        return SA_ERR_CUDA;
    return from_cuda(bsa::attn_fwd(tq, tk, tv, kv_idx, kv_cnt, o, BH, N, d, bs,
                                   resolve_scale(scale, d), g_wait_ns, num_sms(dev), g_progress,
                                   reinterpret_cast<unsigned int *>(workspace),
                                   (cudaStream_t)stream));
}

}  // namespace

extern "C" {

const char *sa_get_error_string(sa_status s) {
    switch (s) {
        case SA_OK: return "SA_OK";
        case SA_ERR_INVALID_ARG: return "SA_ERR_INVALID_ARG: invalid argument";
        case SA_ERR_UNSUPPORTED: return "SA_ERR_UNSUPPORTED: unsupported head size, block size or block count";
        case SA_ERR_CUDA: return "SA_ERR_CUDA: CUDA call failed";
        case SA_ERR_TIMEOUT: return "SA_ERR_TIMEOUT: a device-side wait ran out";
    }
    return "unknown sa_status";
}

int sa_num_blocks(int N, int bs) { return (N > 0 && bs > 0) ? (N + bs - 1) / bs : 0; }

size_t sa_attn_workspace_bytes(void) { return kAttnWorkspaceBytes; }

sa_status sa_set_wait_limit_ns(uint64_t ns) {
    g_wait_ns = ns ? (unsigned long long)ns : kDefaultWaitNs;
    return SA_OK;
}

sa_status sa_pool_blocks(const void *q, const void *k, float *qp, float *kp, int B, int H, int N,
                         int d, int bs, void *stream) {
    if (!q || !k || !qp || !kp || !shape_ok(B, H, N)) return SA_ERR_INVALID_ARG;
    if (!dims_supported(d, bs)) return SA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(qp) || !aligned16(kp)) return SA_ERR_INVALID_ARG;
    int dev;
    if (!select_device(qp, &dev)) return SA_ERR_INVALID_ARG;
    return from_cuda(bsa::pool_blocks(q, k, qp, kp, (long long)B * H, N, d, bs, (cudaStream_t)stream));
}

sa_status sa_select_from_logits(const float *logits, int B, int H, int nb, int topk, float topp,
                                uint8_t *mask, int32_t *kv_idx, int32_t *kv_cnt, void *stream) {
    if (!logits || !mask || !kv_idx || !kv_cnt || !shape_ok(B, H, nb)) return SA_ERR_INVALID_ARG;
    if (topk < 0 || !(topp >= 0.f && topp <= 1.f)) return SA_ERR_INVALID_ARG;
    if (nb > 1024) return SA_ERR_UNSUPPORTED;
    if (!aligned4(logits) || !aligned4(kv_idx)) return SA_ERR_INVALID_ARG;
    int dev;
    if (!select_device(kv_idx, &dev)) return SA_ERR_INVALID_ARG;
    return from_cuda(bsa::select_rows(logits, (long long)B * H * nb, nb, topk, topp, mask, kv_idx,
                                      kv_cnt, (cudaStream_t)stream));
}

sa_status sa_block_scores(const float *qp, const float *kp, int B, int H, int nb, int d, float scale,
                          float *logits, void *stream) {
    if (!qp || !kp || !logits || !shape_ok(B, H, nb)) return SA_ERR_INVALID_ARG;
    if (isnan(scale)) return SA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return SA_ERR_UNSUPPORTED;
    if (!aligned16(qp) || !aligned16(kp) || !aligned4(logits)) return SA_ERR_INVALID_ARG;
    int dev;
    if (!select_device(logits, &dev)) return SA_ERR_INVALID_ARG;
    return from_cuda(bsa::block_scores_tc(qp, kp, logits, (long long)B * H, nb, d,
                                          resolve_scale(scale, d), g_wait_ns, (cudaStream_t)stream));
}

sa_status sa_static_mask(const int32_t *patterns, int B, int H, int nb, uint8_t *mask,
                         int32_t *kv_idx, int32_t *kv_cnt, void *stream) {
    if (!patterns || !mask || !kv_idx || !kv_cnt || !shape_ok(B, H, nb)) return SA_ERR_INVALID_ARG;
    if (!aligned4(kv_idx)) return SA_ERR_INVALID_ARG;
    int dev;
    if (!select_device(kv_idx, &dev)) return SA_ERR_INVALID_ARG;
    return from_cuda(bsa::static_mask(patterns, (long long)B * H, H, nb, mask, kv_idx, kv_cnt,
                                      (cudaStream_t)stream));
}

sa_status sa_select_mask_topk_topp(const float *qp, const float *kp, int B, int H, int nb, int d,
                                   int topk, float topp, float scale, uint8_t *mask,
                                   int32_t *kv_idx, int32_t *kv_cnt, void *stream) {
    if (!qp || !kp || !mask || !kv_idx || !kv_cnt || !shape_ok(B, H, nb)) return SA_ERR_INVALID_ARG;
    if (topk < 0 || !(topp >= 0.f && topp <= 1.f) || isnan(scale)) return SA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return SA_ERR_UNSUPPORTED;
    if (nb > 1024) return SA_ERR_UNSUPPORTED;
    if (!aligned16(qp) || !aligned16(kp) || !aligned4(kv_idx)) return SA_ERR_INVALID_ARG;
    int dev;
    if (!select_device(kv_idx, &dev)) return SA_ERR_INVALID_ARG;
    const long long BH = (long long)B * H;
    float *logits = reinterpret_cast<float *>(kv_idx);  // staging: same size, row-owned
    cudaError_t e = bsa::block_scores_tc(qp, kp, logits, BH, nb, d, resolve_scale(scale, d),
                                         g_wait_ns, (cudaStream_t)stream);
    if (e != cudaSuccess) return SA_ERR_CUDA;
    return from_cuda(bsa::select_rows(logits, BH * nb, nb, topk, topp, mask, kv_idx, kv_cnt,
                                      (cudaStream_t)stream));
}

sa_status sa_block_sparse_attn_fwd(const void *q, const void *k, const void *v,
                                   const int32_t *kv_idx, const int32_t *kv_cnt, void *o, int B,
                                   int H, int N, int d, int bs, float scale, void *workspace,
                                   size_t workspace_bytes, void *stream) {
    const sa_status a = check_sparse_attn_args(q, k, v, kv_idx, kv_cnt, o, B, H, N, d, bs, scale);
    if (a != SA_OK) return a;
    if (!workspace || workspace_bytes < kAttnWorkspaceBytes || !aligned16(workspace))
        return SA_ERR_INVALID_ARG;
    return run_attention(q, k, v, kv_idx, kv_cnt, o, B, H, N, d, bs, scale, workspace, stream);
}

sa_status sa_dense_attn_fwd(const void *q, const void *k, const void *v, void *o, int B, int H,
                            int N, int d, float scale, void *workspace, size_t workspace_bytes,
                            void *stream) {
    if (!q || !k || !v || !o || !shape_ok(B, H, N)) return SA_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < kAttnWorkspaceBytes || !aligned16(workspace))
        return SA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return SA_ERR_UNSUPPORTED;
    if (isnan(scale)) return SA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return SA_ERR_INVALID_ARG;
    return run_attention(q, k, v, nullptr, nullptr, o, B, H, N, d, 128, scale, workspace, stream);
}

sa_status sa_get_device_error(void *stream) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return SA_ERR_CUDA;
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_bsa_device_error, sizeof v) != cudaSuccess) return SA_ERR_CUDA;
    if (v && cudaMemcpyToSymbol(g_bsa_device_error, &zero, sizeof zero) != cudaSuccess)
        return SA_ERR_CUDA;
    if (v & BSA_DEVERR_TIMEOUT) return SA_ERR_TIMEOUT;
    if (v & BSA_DEVERR_BOUNDS) return SA_ERR_INVALID_ARG;
    return SA_OK;
}

sa_status sa_set_progress_buffer(void *words) {
    g_progress = reinterpret_cast<unsigned int *>(words);
    return SA_OK;
}

sa_status sa_get_wait_diagnostics(uint64_t *record) {
    if (!record) return SA_ERR_INVALID_ARG;
    unsigned long long v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_bsa_wait_diag, sizeof v) != cudaSuccess) return SA_ERR_CUDA;
    if (v && cudaMemcpyToSymbol(g_bsa_wait_diag, &zero, sizeof zero) != cudaSuccess) return SA_ERR_CUDA;
    *record = v;
    return SA_OK;
}

sa_status sa_test_exp2_poly(const float *x, float *y, int n, void *stream) {
    if (!x || !y || n < 0) return SA_ERR_INVALID_ARG;
    int dev;
    if (!select_device(y, &dev)) return SA_ERR_INVALID_ARG;
    return from_cuda(bsa::exp2_poly_eval(x, y, n, (cudaStream_t)stream));
}

sa_status sa_probe_bounded_wait(void *stream) {
    return from_cuda(bsa::bounded_wait_probe(g_wait_ns, (cudaStream_t)stream));
}

}  // extern "C"
