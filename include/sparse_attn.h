/*
 * sparse_attn.h: C ABI of libbsa, block-sparse self-attention for video diffusion transformers
 * with hybrid top-k + top-p block masks, for NVIDIA B200 (sm_100a).
 *
 * The path, one attention call (all steps asynchronous on one CUDA stream):
 *
 *   Q, K, V [B, H, N, d] bf16
 *     sa_pool_blocks            -> Qp, Kp [B, H, nb, d] fp32    mean of each block of bs tokens
 *     sa_select_mask_topk_topp  -> mask [B, H, nb, nb] uint8, kv_idx, kv_cnt
 *                                  softmax(Qp Kp^T * scale) per query-block row; keep the union of
 *                                  the top-k blocks and the shortest top-p prefix
 *     sa_block_sparse_attn_fwd  -> O [B, H, N, d] bf16          softmax attention over the kept
 *                                                               key blocks only
 *   sa_dense_attn_fwd is the 0 %-sparsity control (every key block).
 *
 * Sources (page title, section):
 *   SpargeAttention2 ("SpargeAttention2とは？Top-k+Top-pハイブリッドマスキングでビデオ生成を16.2倍高速化"):
 *     section "Top-kとTop-pの限界を解剖する" defines top-k (keep the k largest probabilities) and
 *     top-p (take from the top until the cumulative probability passes p); section
 *     "ハイブリッドマスキングと蒸留微調整" makes the mask the union of the two.
 *   Sparse VideoGen2 ("Sparse VideoGen2: Accelerate Video Generation with Sparse Attention via
 *     Semantic-Aware Permutation"): section 1 (block representatives by mean pooling), section
 *     2.B (scores between representatives, sorted, taken until the cumulative score reaches p),
 *     section 2.C (sparse loads of the kept key/value blocks, dense compute on query tiles).
 *   The block size, mean pooling, the score scale 1/sqrt(d) and the tensor layouts are fixed by
 *   the problem statement this library implements; the pages leave them open.
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers owned by the caller.  The library allocates and frees
 *     nothing; it never synchronises the stream except in sa_get_device_error.  The attention
 *     entry points take a small caller-owned device workspace (sa_attn_workspace_bytes()) that
 *     holds their work counter; calls that may overlap on the GPU need separate workspaces.
 *   - Tensors are dense and row-major with the last dimension contiguous.  bf16 tensors are
 *     passed as void*; their base addresses, and those of the pooled fp32 tensors and of
 *     workspaces, must be 16-byte aligned.  int32 lists and counts, uint8 masks and fp32 block
 *     scores are accessed element by element and need only their natural alignment.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).  The call
 *     runs on the device that owns the output pointer.
 *   - Supported shapes: d in {64, 128}, bs in {64, 128}, N >= 1 (any N; a tail block shorter
 *     than bs is handled inside), B*H in [1, 65535], nb = ceil(N / bs) <= 1024.
 *   - Argument errors are detected on the host and returned before anything is launched.
 *     A failed launch returns SA_ERR_CUDA.  Device-side conditions (a bounded wait that ran
 *     out, an out-of-range block id in kv_idx) are recorded in a device error word that
 *     sa_get_device_error reads and clears.
 */
#ifndef SPARSE_ATTN_H
#define SPARSE_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SA_OK = 0,
    SA_ERR_INVALID_ARG = 1, /* null or misaligned pointer, bad size or parameter */
    SA_ERR_UNSUPPORTED = 2, /* d, bs or nb outside the supported set */
    SA_ERR_CUDA = 3,        /* a CUDA runtime or driver call failed */
    SA_ERR_TIMEOUT = 4      /* a device-side bounded wait ran out (reported by sa_get_device_error) */
} sa_status;

/*
 * Block representatives (Sparse VideoGen2, section 1: mean pooling of contiguous blocks).
 *   qp[b,h,i,:] = mean over t in [i*bs, min((i+1)*bs, N)) of q[b,h,t,:], likewise kp from k.
 * q, k   : [B, H, N, d] bf16, read only.
 * qp, kp : [B, H, nb, d] fp32, written; nb = ceil(N / bs).  Accumulation is fp32.
 */
sa_status sa_pool_blocks(const void *q, const void *k, float *qp, float *kp, int B, int H, int N,
                         int d, int bs, void *stream);

/*
 * Hybrid block selection (SpargeAttention2, "Top-kとTop-pの限界を解剖する" and
 * "ハイブリッドマスキングと蒸留微調整"; Sparse VideoGen2 section 2.B).
 *   P[i,:]  = softmax_j(qp_i . kp_j * scale) over the nb key blocks of row i (fp32)
 *   order   = key blocks by P descending, the lower block id first on equal P
 *   S_k     = first min(topk, nb) blocks of the order
 *   S_p     = first m blocks, m the least count whose cumulative P is >= topp
 *             (topp <= 0: m = 0; topp >= 1: m = nb)
 *   keep(i) = S_k union S_p      (both are prefixes of one order, so |keep| = max(min(k,nb), m))
 * qp, kp  : [B, H, nb, d] fp32 (as written by sa_pool_blocks).
 * topk    : >= 0 (values above nb act as nb).  topp : in [0, 1].
 * scale   : score scale; <= 0 selects 1/sqrt(d).
 * mask    : [B, H, nb, nb] uint8, written with 0/1.
 * kv_idx  : [B, H, nb, nb] int32.  Row (b,h,i) receives the kept key-block ids in ascending
 *           order in its first kv_cnt[b,h,i] entries; the remaining entries are scratch and
 *           undefined on return (the buffer also stages the fp32 block scores).
 * kv_cnt  : [B, H, nb] int32, written.
 */
sa_status sa_select_mask_topk_topp(const float *qp, const float *kp, int B, int H, int nb, int d,
                                   int topk, float topp, float scale, uint8_t *mask,
                                   int32_t *kv_idx, int32_t *kv_cnt, void *stream);

/*
 * Pooling and selection in one call: sa_pool_blocks followed by sa_select_mask_topk_topp (same
 * arguments, same outputs, bit for bit), all on `stream`.  Needs nb <= 1024.
 */
sa_status sa_pool_select_topk_topp(const void *q, const void *k, float *qp, float *kp, int B,
                                   int H, int N, int d, int bs, int topk, float topp, float scale,
                                   uint8_t *mask, int32_t *kv_idx, int32_t *kv_cnt, void *stream);

/*
 * The pooled block scores alone (the first half of sa_select_mask_topk_topp):
 *   logits[b,h,i,j] = scale * qp[b,h,i,:] . kp[b,h,j,:]
 * computed on the tensor cores at fp32 accuracy (each fp32 operand split exactly into three
 * bf16 parts; the six part products of weight >= 2^-16 accumulate in fp32).
 * qp, kp : [B, H, nb, d] fp32.  logits : [B, H, nb, nb] fp32, written.  d in {64, 128}.
 * scale  : <= 0 selects 1/sqrt(d).
 */
sa_status sa_block_scores(const float *qp, const float *kp, int B, int H, int nb, int d, float scale,
                          float *logits, void *stream);

/*
 * Static block patterns (Sparse-vDiT, section 3: diagonal, multi-diagonal and vertical-stripe
 * heads, and skipped heads) as a mask and kept-block lists for sa_block_sparse_attn_fwd.
 * patterns : [H, 4] int32 on the device, one {flags, w, p, s} per head, shared by the batch; key
 *            block j is kept for query block i when any enabled part holds:
 *              flags & 1: |i - j| <= w                                  (diagonal band)
 *              flags & 2: i - j within w of a multiple of p, p > 0      (diagonals every p)
 *              flags & 4: j < s                                         (first s key blocks)
 *            flags == 0 keeps nothing (skipped head; the attention then writes zeros).
 * mask, kv_idx, kv_cnt : as for sa_select_mask_topk_topp ([B, H, nb, nb] u8, [B, H, nb, nb] i32
 *            with the ascending kept ids first, [B, H, nb] i32).
 */
sa_status sa_static_mask(const int32_t *patterns, int B, int H, int nb, uint8_t *mask,
                         int32_t *kv_idx, int32_t *kv_cnt, void *stream);

/*
 * SQuad attention (SQuad: Sub-Quadratic Attention Distillation, method section 1): a local pass
 * of softmax attention within fixed windows of w tokens, then a global pass of softmax attention
 * among the tokens at the same position of every window, whose values are the local outputs.
 * With N = W w and token t = a w + r (window a, position r):
 *   Y[a w + r] = sum_{r'} softmax_{r'}(scale q[a w + r] . k[a w + r']) v[a w + r']
 *   O[a w + r] = sum_{a'} softmax_{a'}(scale q[a w + r] . k[a' w + r]) Y[a' w + r]
 * Runs as two dense attention calls with token regrouping between them (Y is held in bf16).
 * q, k, v, o : [B, H, N, d] bf16, d in {64, 128}; N must be a multiple of w, and w and N / w
 *              at most 131072.  scale <= 0 selects 1/sqrt(d) (both passes).
 * workspace  : at least sa_squad_workspace_bytes(B, H, N, d) bytes of device memory, 16-byte
 *              aligned, owned by the caller (four regrouped tensors and the work counter).
 */
size_t sa_squad_workspace_bytes(int B, int H, int N, int d);
sa_status sa_squad_attn_fwd(const void *q, const void *k, const void *v, void *o, int B, int H,
                            int N, int d, int w, float scale, void *workspace,
                            size_t workspace_bytes, void *stream);

/*
 * Semantic-aware permutation with centroid top-p (Sparse VideoGen2, method sections A-C).
 * Cluster counts C, Cq, Ck are in [1, 1024]; d in {64, 128}; N < 2^24 for the attention calls.
 *
 * sa_kmeans: Lloyd's algorithm on the token rows of every head of x [B, H, N, d] bf16, from the
 *   centroids in cent [B, H, C, d] fp32 (16-byte aligned; a centroid cache, overwritten with the
 *   result).  `iters` update steps, each the mean of the rows assigned to a cluster (a cluster
 *   with no rows keeps its centroid), then a final assignment to the updated centroids: nearest
 *   centroid by squared Euclidean distance in fp32, the lower index on a tie.  Outputs (int32):
 *   assign [B, H, N] the final cluster of each token; perm [B, H, N] the tokens in order of
 *   cluster, ascending within a cluster; cstart, csize [B, H, C] where each cluster's tokens sit
 *   in perm.  Cluster sums run in token order, so results repeat bit for bit.  The nearest
 *   centroid runs on the tensor cores (rows exact in bf16, each fp32 centroid split exactly
 *   into three bf16 parts, fp32 accumulation); workspace: sa_kmeans_workspace_bytes() bytes,
 *   16-byte aligned, owned by the caller (the centroid parts and norms, and for C > 128 each
 *   128-centroid tile's nearest candidate per token).
 */
size_t sa_kmeans_workspace_bytes(int B, int H, int N, int C, int d);
sa_status sa_kmeans(const void *x, float *cent, int32_t *assign, int32_t *perm, int32_t *cstart,
                    int32_t *csize, int B, int H, int N, int d, int C, int iters, void *workspace,
                    size_t workspace_bytes, void *stream);

/*
 * The stable order of the tokens by cluster id (the permutation of section A) alone:
 * assign [B, H, N] int32 ids in [0, C) (others are clamped and flagged in the device error word)
 * -> perm, cstart, csize as for sa_kmeans.  workspace: sa_cluster_sort_workspace_bytes() bytes,
 * 16-byte aligned, owned by the caller (per-chunk cluster counts).
 */
size_t sa_cluster_sort_workspace_bytes(int B, int H, int N, int C);
sa_status sa_cluster_sort(const int32_t *assign, int B, int H, int N, int C, int32_t *perm,
                          int32_t *cstart, int32_t *csize, void *workspace,
                          size_t workspace_bytes, void *stream);

/*
 * Centroid top-p (section B).  For query cluster a of head (b, h), key cluster j is estimated to
 * receive the share  w[a, j] = size_k[j] exp(scale cq[a] . ck[j]) / sum_j' (same)  of the
 * attention (each key represented by its centroid).  Key clusters are ranked by w descending
 * (the lower id first on a tie) and taken until the cumulative share reaches topp; topp <= 0
 * takes none, topp >= 1 every cluster with keys; a cluster with size_k = 0 is never taken.
 * The decision runs in fp32 (the top-p kernel of the block path), so clusters whose share lies
 * within ~1e-5 of the cut may differ from an exact evaluation.
 * cq [B, H, Cq, d], ck [B, H, Ck, d] fp32; size_k [B, H, Ck] int32; sel [B, H, Cq, Ck] uint8
 * 0/1, written.  workspace: sa_centroid_topp_workspace_bytes() bytes, 16-byte aligned.
 */
size_t sa_centroid_topp_workspace_bytes(int B, int H, int Cq, int Ck);
sa_status sa_centroid_topp(const float *cq, const float *ck, const int32_t *size_k, int B, int H,
                           int Cq, int Ck, int d, float topp, float scale, uint8_t *sel,
                           void *workspace, size_t workspace_bytes, void *stream);

/*
 * Attention over selected clusters (section C):
 *   O[b,h,t,:] = sum over keys s with sel[b,h,assign_q[t],assign_k[s]] != 0 of
 *                softmax_s(scale Q[t] . K[s]) V[s];   zero when the selection is empty.
 * Q is permuted by query cluster and K, V by key cluster (each cluster contiguous); every query
 * tile of up to 128 rows of one cluster runs over key tiles of up to 128 consecutive permuted
 * keys covering exactly the selected clusters (adjacent clusters share tiles), on the tensor
 * cores; outputs go straight back to the original token positions.
 * q, k, v, o : [B, H, N, d] bf16.  assign_q, assign_k : [B, H, N] int32 in [0, Cq) / [0, Ck).
 * sel : [B, H, Cq, Ck] uint8, nonzero = selected.  scale <= 0 selects 1/sqrt(d).
 * workspace : sa_cluster_attn_workspace_bytes() bytes, 16-byte aligned (the permuted tensors,
 *             the permutations and the tile tables).
 */
size_t sa_cluster_attn_workspace_bytes(int B, int H, int N, int d, int Cq, int Ck);
sa_status sa_cluster_attn_fwd(const void *q, const void *k, const void *v, void *o,
                              const int32_t *assign_q, const int32_t *assign_k,
                              const uint8_t *sel, int B, int H, int N, int d, int Cq, int Ck,
                              float scale, void *workspace, size_t workspace_bytes, void *stream);

/*
 * The whole SVG2 path: sa_kmeans of Q (into cent_q [B, H, Cq, d]) and of K (into cent_k
 * [B, H, Ck, d]) with `iters` update steps from the caller's centroid cache, sa_centroid_topp on
 * the resulting centroids and key cluster sizes (sel [B, H, Cq, Ck] uint8, written), then the
 * attention of sa_cluster_attn_fwd.  workspace: sa_svg2_workspace_bytes() bytes, 16-byte aligned.
 */
size_t sa_svg2_workspace_bytes(int B, int H, int N, int d, int Cq, int Ck);
sa_status sa_svg2_attn_fwd(const void *q, const void *k, const void *v, void *o, float *cent_q,
                           float *cent_k, int B, int H, int N, int d, int Cq, int Ck, int iters,
                           float topp, float scale, uint8_t *sel, void *workspace,
                           size_t workspace_bytes, void *stream);

/*
 * Selection from caller-provided block scores (the second half of sa_select_mask_topk_topp,
 * exposed for tests that feed hand-made rows).  logits: [B, H, nb, nb] fp32 scores already
 * scaled; the row softmax, ranking, top-k union top-p and outputs are as above.  logits may be
 * the same buffer as kv_idx.
 */
sa_status sa_select_from_logits(const float *logits, int B, int H, int nb, int topk, float topp,
                                uint8_t *mask, int32_t *kv_idx, int32_t *kv_cnt, void *stream);

/*
 * Block-sparse attention forward (online softmax over the kept key blocks only): the attention
 * that the hybrid mask of the SpargeAttention2 page (section "ハイブリッドマスキングと蒸留微調整")
 * restricts to the kept blocks, computed as the Sparse VideoGen2 page's kernel description
 * (section 2.C) puts it: sparse loads of the kept key/value blocks, dense compute on a
 * contiguous query tile.
 *   O[b,h,t,:] = sum over kept blocks j of query block i = t / bs, keys s in block j with s < N,
 *                of softmax_s(scale * Q[t] . K[s]) V[s]; zero when the block keeps nothing.
 * q, k, v : [B, H, N, d] bf16.       o : [B, H, N, d] bf16, written.
 * kv_idx  : [B, H, nb, nb] int32, ascending ids < nb in the first kv_cnt entries of each row
 *           (as written by sa_select_mask_topk_topp).  kv_cnt : [B, H, nb] int32 in [0, nb].
 *           Ids outside [0, nb) are clamped and flagged in the device error word.
 * bs      : block size of both query and key blocks.  scale : <= 0 selects 1/sqrt(d).
 * workspace: device memory of at least sa_attn_workspace_bytes() bytes, 16-byte aligned, owned
 *           by the caller; the call zeroes its counter on `stream` before the kernel starts.
 * Arithmetic: bf16 operands, fp32 accumulation on the tensor cores, P rounded to bf16.
 */
sa_status sa_block_sparse_attn_fwd(const void *q, const void *k, const void *v,
                                   const int32_t *kv_idx, const int32_t *kv_cnt, void *o, int B,
                                   int H, int N, int d, int bs, float scale, void *workspace,
                                   size_t workspace_bytes, void *stream);

/*
 * Dense attention forward, the 0 %-sparsity control: O = softmax(scale Q K^T) V over all N keys
 * (the full attention that the SpargeAttention2 page's speed-ups and quality comparisons are
 * measured against, section "実験結果：速度と品質の両立").
 * Same layouts, workspace and arithmetic as sa_block_sparse_attn_fwd (internally bs = 128).
 */
sa_status sa_dense_attn_fwd(const void *q, const void *k, const void *v, void *o, int B, int H,
                            int N, int d, float scale, void *workspace, size_t workspace_bytes,
                            void *stream);

/* Bytes of device workspace the attention entry points need (a small constant). */
size_t sa_attn_workspace_bytes(void);

/*
 * Block-sparse attention forward for callers that cannot provide device memory beyond their
 * inputs and outputs (the pages have no counterpart: this is a deployment variant of
 * sa_block_sparse_attn_fwd).  Some callers cannot lend the library a workspace: their device
 * memory belongs to another runtime's allocator and they have no spare buffer, or they may not
 * call cudaMalloc where attention runs because it can synchronise the device.  This entry point
 * allocates nothing: its scratch (the work counter) lives in a fixed 256-byte array in the
 * library's device image, which every GPU that loads the library holds until the process exits.
 * Arguments, layouts and results are those of sa_block_sparse_attn_fwd without the workspace.
 * - The first call on a device resolves the array's device address (cudaGetSymbolAddress, with
 *   that device current) and caches it; make that first call before any stream capture.  The
 *   cache is keyed on the device context's unique id: after cudaDeviceReset (or any other end
 *   of the context) the next call resolves the address again in the new context, and that
 *   call, too, should come before any stream capture.
 * - Every call shares the one array, which keeps the last call's contents; each call zeroes
 *   the counter on `stream` before its kernel.  Calls that overlap on the GPU (different
 *   streams, or several host threads) race on the array and must be serialised by the caller.
 * - Returns SA_ERR_UNSUPPORTED if the scratch the call needs exceeds the 256-byte array, and the
 *   errors of sa_block_sparse_attn_fwd otherwise.
 */
sa_status sa_block_sparse_attn_fwd_noalloc(const void *q, const void *k, const void *v,
                                           const int32_t *kv_idx, const int32_t *kv_cnt, void *o,
                                           int B, int H, int N, int d, int bs, float scale,
                                           void *stream);

/*
 * SparsePR: block-sparse attention followed by the probe-fitted residual correction (page
 * "Partition the Support, Reconstruct the Residual: Training-Free Sparse Attention for Video
 * Generation and World Models", abstract and summary section 3: a few probe queries are computed
 * exactly, and their residuals against the sparse output are fitted by an affine map of the
 * sparse output, restricted to the span of those residuals, which then corrects every row).
 *   O_s = sa_block_sparse_attn_fwd(q, k, v, kv_idx, kv_cnt);  per head, with P = probes[b, h, :]
 *   X = [O_s[P], 1], R = exact(P) - O_s[P], W = X^+ R (minimum norm), O = O_s + [O_s, 1] W.
 * probes  : [B, H, m] int32 token ids in [0, N) chosen by the caller (ids outside are clamped);
 *           1 <= m <= min(N, 8192).  Repeated ids are allowed.
 * q, k, v, kv_idx, kv_cnt, o, bs, scale: as sa_block_sparse_attn_fwd.
 * workspace: device memory of sa_sparsepr_workspace_bytes(B, H, N, d, m) bytes, 16-byte
 *           aligned, owned by the caller (probe rows, their exact outputs, the fp64 fit).
 * Arithmetic: the sparse output in bf16 and the probes' exact outputs in fp32 (fp32
 * accumulation on the tensor cores; the exact outputs combined from runs of keys in fp64), the
 * fit in fp64 (normal equations of the smaller side, Cholesky with a ridge of 1e-12 times the
 * mean diagonal), the correction [O_s, 1] W on the tensor cores in fp32 with W's first d rows
 * split into two bf16 parts (relative error 2^-17), rounded to bf16 once, in place in o.
 */
sa_status sa_sparsepr_attn_fwd(const void *q, const void *k, const void *v,
                               const int32_t *kv_idx, const int32_t *kv_cnt,
                               const int32_t *probes, int m, void *o, int B, int H, int N, int d,
                               int bs, float scale, void *workspace, size_t workspace_bytes,
                               void *stream);

/* Bytes of device workspace sa_sparsepr_attn_fwd needs (0 for unsupported arguments). */
size_t sa_sparsepr_workspace_bytes(int B, int H, int N, int d, int m);

/* Human-readable name of a status code (static storage). */
const char *sa_get_error_string(sa_status status);

/*
 * Synchronise `stream`, then read and clear the device error word of the current device.
 * Returns SA_ERR_TIMEOUT if a bounded wait ran out since the last call, SA_ERR_INVALID_ARG if
 * a kernel met an out-of-range key-block id, SA_ERR_CUDA if the synchronisation failed.
 */
sa_status sa_get_device_error(void *stream);

/*
 * Upper bound, in nanoseconds of device time, on every device-side wait of later launches
 * (default 2e9).  After it a kernel records SA_ERR_TIMEOUT, unwinds and exits.  0 restores the
 * default.
 */
sa_status sa_set_wait_limit_ns(uint64_t ns);

/*
 * Failure-detection check: launches one CTA that waits on a barrier nothing ever arrives at,
 * bounded by the current wait limit.  A subsequent sa_get_device_error returns SA_ERR_TIMEOUT.
 */
sa_status sa_probe_bounded_wait(void *stream);

/*
 * Where the first device-side wait that ran out since the last call gave up, then cleared:
 * bits 56..63 identify the wait site (role and barrier), bits 32..55 the CTA, bits 0..31 the
 * position (query-block unit and step).  0 when no wait has run out.
 */
sa_status sa_get_wait_diagnostics(uint64_t *record);

/*
 * Diagnosis aid: when `words` is non-null (host-mapped pinned memory, 8 x 32-bit words per CTA
 * of the attention grid, i.e. at least 8 * 2 * SM-count words), later attention launches write
 * each role's current stage there, readable by the host while the kernel runs.  NULL turns it
 * off (the default).  The caller keeps the memory alive while launches that use it run.
 */
sa_status sa_set_progress_buffer(void *words);

/*
 * Test hook: y[i] = the FMA-pipe 2^x the attention softmax uses for a quarter of its
 * probabilities (range reduction to [-1/2, 1/2] and a degree-3 minimax polynomial, relative
 * error below 1e-4 where the result is a normal float; inputs below -126 give values below 2e-38).
 * x, y: n fp32 device values.
 */
sa_status sa_test_exp2_poly(const float *x, float *y, int n, void *stream);

/* Number of key-block ids per row of kv_idx for a given N and bs, i.e. nb = ceil(N / bs). */
int sa_num_blocks(int N, int bs);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_ATTN_H */
