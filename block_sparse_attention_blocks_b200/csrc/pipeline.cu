// Pooling and block selection of one attention call in one entry point: the pooling kernel, the
// block-score kernel and the per-row selection kernel, in that order on the caller's stream.
// The results are the ones sa_pool_blocks followed by sa_select_mask_topk_topp give.
#include "bsa_internal.h"
#include "sparse_attn.h"

extern "C" sa_status sa_pool_select_topk_topp(const void *q, const void *k, float *qp, float *kp,
                                              int B, int H, int N, int d, int bs, int topk,
                                              float topp, float scale, uint8_t *mask,
                                              int32_t *kv_idx, int32_t *kv_cnt, void *stream) {
    if (!q || !k || !qp || !kp || !mask || !kv_idx || !kv_cnt || !shape_ok(B, H, N))
        return SA_ERR_INVALID_ARG;
    if (topk < 0 || !(topp >= 0.f && topp <= 1.f) || isnan(scale)) return SA_ERR_INVALID_ARG;
    if (!dims_supported(d, bs)) return SA_ERR_UNSUPPORTED;
    const int nb = sa_num_blocks(N, bs);
    if (nb > 1024) return SA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(qp) || !aligned16(kp) || !aligned4(kv_idx))
        return SA_ERR_INVALID_ARG;
    int dev;
    if (!select_device(kv_idx, &dev)) return SA_ERR_INVALID_ARG;
    const cudaStream_t st = (cudaStream_t)stream;
    const long long BH = (long long)B * H;
    cudaError_t e = bsa::pool_blocks(q, k, qp, kp, BH, N, d, bs, st);
    float *logits = reinterpret_cast<float *>(kv_idx);  // staging: same size, row-owned
    if (e == cudaSuccess)
        e = bsa::block_scores_tc(qp, kp, logits, BH, nb, d, resolve_scale(scale, d), g_wait_ns, st);
    if (e == cudaSuccess) e = bsa::select_rows(logits, BH * nb, nb, topk, topp, mask, kv_idx, kv_cnt, st);
    return from_cuda(e);
}
