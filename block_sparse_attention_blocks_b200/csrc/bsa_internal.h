// Declarations shared by the CUDA translation units of libbsa (not part of the public C ABI).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ptx.cuh"

namespace bsa {

cudaError_t pool_blocks(const void *q, const void *k, float *qp, float *kp, long long BH, int N,
                        int d, int bs, cudaStream_t st);

cudaError_t block_scores_tc(const float *qp, const float *kp, float *logits, long long BH, int nb,
                            int d, float scale, unsigned long long wait_ns, cudaStream_t st);

cudaError_t static_mask(const int32_t *patterns, long long BH, int H, int nb, uint8_t *mask,
                        int32_t *kv_idx, int32_t *kv_cnt, cudaStream_t st);

cudaError_t permute_tokens(const void *src, void *dst, long long G, long long A, long long R,
                           int d, int num_sms, cudaStream_t st);

cudaError_t select_rows(const float *logits, long long rows, int nb, int topk, float topp,
                        uint8_t *mask, int32_t *kv_idx, int32_t *kv_cnt, cudaStream_t st);

cudaError_t attn_fwd(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                     const int32_t *kv_idx, const int32_t *kv_cnt, void *o, long long BH, int N,
                     int d, int bs, float scale, unsigned long long wait_ns, int num_sms,
                     unsigned int *progress, unsigned int *workspace, cudaStream_t st);

cudaError_t bounded_wait_probe(unsigned long long wait_ns, cudaStream_t st);

cudaError_t exp2_poly_eval(const float *x, float *y, int n, cudaStream_t st);

}  // namespace bsa
