// Declarations shared by the CUDA translation units of libbsa (not part of the public C ABI).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ptx.cuh"

namespace bsa {

// Launch `kern` on `st` with programmatic stream serialization, so that it may begin while the
// previous kernel on the stream drains; the kernel calls grid_dependency_wait() before it reads
// what that kernel wrote.
template <typename... KArgs, typename... Args>
static cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                    cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

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

// attention within short sequences of W tokens stored back to back (Ntot rows), packed 128 / W
// to a tile with a block-diagonal mask (attn.cu, GroupWalk); W <= 128
cudaError_t attn_group_fwd(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                           void *o, long long Ntot, int W, int d, float scale,
                           unsigned long long wait_ns, int num_sms, unsigned int *workspace,
                           cudaStream_t st);

// attention over variable-length tiles (attn.cu, TileWalk); part_o / part_lse select the split form
cudaError_t attn_varlen_fwd(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                            const int2 *units, int units_per_head, const int32_t *tiles,
                            const int32_t *tcnt, int tstride, const int32_t *perm_q, void *o,
                            long long BH, int N, int Nq, int Cq, int d, float scale,
                            unsigned long long wait_ns, int num_sms, unsigned int *workspace,
                            cudaStream_t st, float *part_o = nullptr, float *part_lse = nullptr);

// parts [BH, 3, C, d] bf16, norms [BH, C] fp32 and, when C > 128, partial
// [ceil(C / 128), BH, N] uint64 are scratch for the tensor-core assignment, hist the cluster
// sort's chunk counts (cluster_sort_scratch_bytes); tx / tp are tensor maps of x ({d, N, BH})
// and parts ({d, C, 3 BH}), 128-row boxes.
cudaError_t kmeans_lloyd(const void *x, float *cent, int32_t *assign, int32_t *perm,
                         int32_t *cstart, int32_t *csize, long long BH, int N, int d, int C,
                         int iters, void *parts, float *norms, uint64_t *partial, int32_t *hist,
                         const CUtensorMap *tx, const CUtensorMap *tp, unsigned long long wait_ns,
                         cudaStream_t st);

cudaError_t cluster_sort(const int32_t *assign, long long BH, int N, int C, int32_t *perm,
                         int32_t *cstart, int32_t *csize, int32_t *hist, cudaStream_t st);
size_t cluster_sort_scratch_bytes(long long BH, int N, int C);

cudaError_t centroid_logits(const float *cq, const float *ck, const int32_t *size_k,
                            float *logits, long long BH, int Cq, int Ck, int d, float scale,
                            cudaStream_t st);

cudaError_t prune_empty(uint8_t *sel, const int32_t *size_k, long long BH, int Cq, int Ck,
                        int num_sms, cudaStream_t st);

cudaError_t build_cluster_tables(const uint8_t *sel, const int32_t *qstart, const int32_t *qsize,
                                 const int32_t *kstart, const int32_t *ksize, long long BH,
                                 int Cq, int Ck, int U, int tstride, int2 *units, int32_t *tiles,
                                 int32_t *tcnt, cudaStream_t st);

cudaError_t gather_rows(const void *src, const int32_t *perm, void *dst, long long BH, int N,
                        int d, int num_sms, cudaStream_t st);

cudaError_t bounded_wait_probe(unsigned long long wait_ns, cudaStream_t st);

cudaError_t exp2_poly_eval(const float *x, float *y, int n, cudaStream_t st);

}  // namespace bsa
