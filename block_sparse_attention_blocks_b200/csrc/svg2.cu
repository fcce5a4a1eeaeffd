// Semantic-aware permutation with centroid top-p (page "Sparse VideoGen2: Accelerate Video
// Generation with Sparse Attention via Semantic-Aware Permutation", method sections A, B and C).
//
//   A. k-means (Lloyd) of the Q rows and, separately, of the K rows of every head into Cq and Ck
//      clusters, started from the caller's centroids (the centroid cache of section C); tokens
//      are then reordered so that every cluster is a contiguous range.
//   B. The score of key cluster j for query cluster a is estimated from the centroids, every key
//      represented by its centroid: |j| exp(scale mu_q[a] . mu_k[j]), normalised over j.
//      Key clusters are taken in descending order of it until the cumulative score reaches p.
//   C. Attention of each query token over the keys of the clusters its cluster selected, on the
//      permuted tensors (dense query tiles, key tiles of variable length), written back in the
//      original token order.
//
// Kernels here: the assignment step (nearest centroid, squared Euclidean distance, the lower
// index on a tie), a stable counting sort of the assignment (the permutation and each cluster's
// range), the update step (the mean of each cluster's rows, summed in token order), the
// centroid scores, the tables of query tiles and key tiles, and the row gather.  Selection runs
// on the top-p kernel of the block path (top-k = 0) over the scores log|j| + scale mu_q . mu_k,
// whose softmax is the estimate above; the attention is attn.cu's kernel with variable-length
// tiles (TileWalk).
#include "bsa_internal.h"
#include "sparse_attn.h"

namespace bsa {

constexpr int kMaxClusters = 1024;   // Cq, Ck: one selection row per warp, sort counters in smem
constexpr int kMaxVarlenN = 1 << 24; // key tile entries pack (first row << 7) into 31 bits

// ------------------------------------------------------------------------------------------
// Stable counting sort of each head's assignment, in three launches over chunks of
// kSortChunk tokens: per-chunk cluster counts; per head, the cluster ranges and each chunk's
// first position in every cluster (counts scanned in (cluster, chunk) order); then each chunk
// places its tokens in token order (one CTA per chunk, 8 warps each owning a contiguous eighth,
// their counts scanned in warp order; lanes of a 32-token step that share a cluster are ranked
// with match.any).  Cluster c occupies perm[cstart[c] .. cstart[c] + csize[c]) with its tokens
// ascending.
// ------------------------------------------------------------------------------------------
constexpr int kSortChunk = 4096;

// hist[bh, chunk, c] = the chunk's tokens assigned to c (out-of-range clusters are clamped and
// flagged)
__global__ void __launch_bounds__(256) cluster_hist_kernel(const int32_t *__restrict__ assign,
                                                           int N, int C, int nchunk,
                                                           int32_t *__restrict__ hist) {
    extern __shared__ int32_t sm_hist[];
    const long long bh = blockIdx.y;
    const int ch = blockIdx.x;
    for (int c = threadIdx.x; c < C; c += 256) sm_hist[c] = 0;
    __syncthreads();
    const int lo = ch * kSortChunk, hi = min(N, lo + kSortChunk);
    bool bad = false;
    for (int n = lo + threadIdx.x; n < hi; n += 256) {
        int a = assign[bh * N + n];
        if (a < 0 || a >= C) {
            bad = true;
            a = a < 0 ? 0 : C - 1;
        }
        atomicAdd(&sm_hist[a], 1);
    }
    if (bad) atomicOr(&g_bsa_device_error, BSA_DEVERR_BOUNDS);
    __syncthreads();
    for (int c = threadIdx.x; c < C; c += 256) hist[(bh * nchunk + ch) * C + c] = sm_hist[c];
}

// Per head: cstart / csize, and hist rewritten in place to each chunk's first position in
// every cluster.  One CTA per head, thread per cluster (C <= 1024).
__global__ void __launch_bounds__(1024) cluster_scan_kernel(int32_t *__restrict__ hist, int nchunk,
                                                            int C, int32_t *__restrict__ cstart,
                                                            int32_t *__restrict__ csize) {
    __shared__ int32_t s_warp[32];
    const long long bh = blockIdx.x;
    const int c = threadIdx.x, warp = c >> 5, lane = c & 31;
    int32_t *h = hist + bh * nchunk * C;
    int total = 0;
    if (c < C)
        for (int ch = 0; ch < nchunk; ++ch) total += h[ch * C + c];
    // exclusive scan of the totals over c (warp scans, then the warp sums)
    int incl = total;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int v = lane < (int)(blockDim.x >> 5) ? s_warp[lane] : 0;
        int wi = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += y;
        }
        s_warp[lane] = wi - v;
    }
    __syncthreads();
    if (c < C) {
        int run = s_warp[warp] + incl - total;
        cstart[bh * C + c] = run;
        csize[bh * C + c] = total;
        for (int ch = 0; ch < nchunk; ++ch) {
            const int t = h[ch * C + c];
            h[ch * C + c] = run;
            run += t;
        }
    }
}

// One CTA per (chunk, head): the chunk's tokens into perm at their stable positions.
__global__ void __launch_bounds__(256) cluster_place_kernel(const int32_t *__restrict__ assign,
                                                            const int32_t *__restrict__ base,
                                                            int N, int C, int nchunk,
                                                            int32_t *__restrict__ perm) {
    extern __shared__ int32_t sm_place[];  // [8][C]: count, then the warp's next free position
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long bh = blockIdx.y;
    const int ch = blockIdx.x;
    const int32_t *as = assign + bh * N;
    for (int i = threadIdx.x; i < 8 * C; i += 256) sm_place[i] = 0;
    __syncthreads();
    const int c0 = ch * kSortChunk, c1 = min(N, c0 + kSortChunk);
    const int per = (c1 - c0 + 7) / 8;
    const int lo = min(c1, c0 + warp * per), hi = min(c1, lo + per);
    for (int s = lo; s < hi; s += 32) {
        const int n = s + lane;
        if (n < hi) atomicAdd(&sm_place[warp * C + min(max(as[n], 0), C - 1)], 1);
    }
    __syncthreads();
    const int32_t *bs = base + (bh * nchunk + ch) * C;
    for (int c = threadIdx.x; c < C; c += 256) {
        int run = bs[c];
        for (int w = 0; w < 8; ++w) {
            const int t = sm_place[w * C + c];
            sm_place[w * C + c] = run;
            run += t;
        }
    }
    __syncthreads();
    const uint32_t lt = (1u << lane) - 1u;
    for (int s = lo; s < hi; s += 32) {  // warp-uniform bounds
        const int n = s + lane;
        const bool v = n < hi;
        int a = -1;
        if (v) a = min(max(as[n], 0), C - 1);
        const uint32_t peers = __match_any_sync(0xffffffffu, a);
        const int rank = __popc(peers & lt);
        if (v) perm[bh * N + sm_place[warp * C + a] + rank] = n;
        __syncwarp();
        if (v && rank == 0) sm_place[warp * C + a] += __popc(peers);
        __syncwarp();
    }
}

// ------------------------------------------------------------------------------------------
// k-means update: one CTA per (cluster, head).  Thread = (16-byte column group, token lane);
// each lane sums its tokens in permuted (= token) order with several rows in flight, the lanes
// are added in lane order, so the result does not depend on scheduling.  A cluster without
// tokens keeps its centroid.
// ------------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(512) kmeans_update_kernel(const __nv_bfloat16 *__restrict__ x,
                                                            const int32_t *__restrict__ perm,
                                                            const int32_t *__restrict__ cstart,
                                                            const int32_t *__restrict__ csize,
                                                            float *__restrict__ cent, int N, int C) {
    constexpr int V = D / 8;     // 16-byte groups (8 channels) per row
    constexpr int G = 512 / V;   // token lanes
    constexpr int U = 4;         // rows in flight per lane
    __shared__ float part[G][D + 1];
    const int c = blockIdx.x;
    const long long bh = blockIdx.y;
    const int vg = threadIdx.x % V, g = threadIdx.x / V;
    const int sz = csize[bh * C + c];
    if (sz <= 0) return;  // the whole CTA leaves together
    const int32_t *pm = perm + bh * N + cstart[bh * C + c];
    const uint4 *xb = reinterpret_cast<const uint4 *>(x) + (size_t)bh * N * V;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int s0 = g; s0 < sz; s0 += G * U) {
        int n[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int s = s0 + u * G;
            n[u] = s < sz ? min(max(pm[s], 0), N - 1) : -1;
        }
        uint4 w[U];
#pragma unroll
        for (int u = 0; u < U; ++u) w[u] = n[u] >= 0 ? xb[(size_t)n[u] * V + vg] : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < U; ++u) {  // in token order within the lane
            if (n[u] < 0) break;
            const uint32_t ws[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                acc[2 * h] += __uint_as_float(ws[h] << 16);
                acc[2 * h + 1] += __uint_as_float(ws[h] & 0xFFFF0000u);
            }
        }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) part[g][vg * 8 + e] = acc[e];
    __syncthreads();
    for (int j = threadIdx.x; j < D; j += 512) {
        float t = 0.f;
        for (int i = 0; i < G; ++i) t += part[i][j];
        cent[(bh * C + c) * D + j] = t / (float)sz;
    }
}

// ------------------------------------------------------------------------------------------
// Centroid scores: logits[a, j] = log|j| + scale mu_q[a] . mu_k[j], -inf for an empty key
// cluster, so that softmax_j(logits[a, :]) is the estimated score of section B.  One warp per
// query centroid, one lane per key centroid of a 32-wide chunk staged in shared memory.
// ------------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) centroid_logits_kernel(const float *__restrict__ cq,
                                                              const float *__restrict__ ck,
                                                              const int32_t *__restrict__ size_k,
                                                              float *__restrict__ logits, int Cq,
                                                              int Ck, float scale) {
    __shared__ float qs[8][D];
    __shared__ float ks[32][D + 1];  // +1: lane j reads row j, conflict-free
    __shared__ float lns[32];
    __shared__ int nonempty[32];
    const long long bh = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int a = blockIdx.x * 8 + warp;
    for (int i = threadIdx.x; i < 8 * D; i += 256) {
        const int w = i / D, e = i % D;
        const int aa = blockIdx.x * 8 + w;
        qs[w][e] = aa < Cq ? cq[(bh * Cq + aa) * D + e] : 0.f;
    }
    for (int j0 = 0; j0 < Ck; j0 += 32) {
        __syncthreads();
        for (int i = threadIdx.x; i < 32 * D; i += 256) {
            const int jj = i / D, e = i % D;
            ks[jj][e] = j0 + jj < Ck ? ck[(bh * Ck + j0 + jj) * D + e] : 0.f;
        }
        if (threadIdx.x < 32) {
            const int j = j0 + threadIdx.x;
            const int sz = j < Ck ? size_k[bh * Ck + j] : 0;
            nonempty[threadIdx.x] = sz > 0;
            lns[threadIdx.x] = sz > 0 ? logf((float)sz) : 0.f;
        }
        __syncthreads();
        const int j = j0 + lane;
        if (a < Cq && j < Ck) {
            float s = 0.f;
#pragma unroll 8
            for (int e = 0; e < D; ++e) s = fmaf(qs[warp][e], ks[lane][e], s);
            logits[(bh * Cq + a) * Ck + j] = nonempty[lane] ? fmaf(s, scale, lns[lane]) : -INFINITY;
        }
    }
}

// A selected key cluster without keys is dropped from the selection.
__global__ void __launch_bounds__(256) prune_empty_kernel(uint8_t *__restrict__ sel,
                                                          const int32_t *__restrict__ size_k,
                                                          long long rows, int Cq, int Ck) {
    const long long total = rows * Ck;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const long long row = i / Ck;
        const int j = (int)(i - row * Ck);
        if (size_k[(row / Cq) * Ck + j] <= 0) sel[i] = 0;
    }
}

// ------------------------------------------------------------------------------------------
// Query tiles of a head (one warp per head): cluster a's rows [qstart, qstart + qsize) are cut
// into tiles of up to 128 rows, in cluster order; unused slots up to U get q_rows = 0.
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) build_units_kernel(const int32_t *__restrict__ qstart,
                                                          const int32_t *__restrict__ qsize,
                                                          long long BH, int Cq, int U,
                                                          int2 *__restrict__ units) {
    const int lane = threadIdx.x & 31;
    const long long bh = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (bh >= BH) return;
    int2 *ub = units + bh * U;
    int base = 0;
    bool bad = false;
    for (int a0 = 0; a0 < Cq; a0 += 32) {
        const int a = a0 + lane;
        const int sz = a < Cq ? max(qsize[bh * Cq + a], 0) : 0;
        const int st = a < Cq ? qstart[bh * Cq + a] : 0;
        const int nt = (sz + 127) >> 7;
        int incl = nt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const int off = base + incl - nt;
        for (int t = 0; t < nt; ++t) {
            const int u = off + t;
            if (u < U)
                ub[u] = make_int2(st + 128 * t, (min(128, sz - 128 * t) << 16) | a);
            else
                bad = true;
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
    }
    for (int u = base + lane; u < U; u += 32) ub[u] = make_int2(0, 0);
    if (bad) atomicOr(&g_bsa_device_error, BSA_DEVERR_BOUNDS);
}

// ------------------------------------------------------------------------------------------
// Key tiles of each (head, query cluster) row (one warp per row): the selected non-empty key
// clusters in id order; clusters that are adjacent in the permuted order (nothing but empty
// clusters between them) merge into one run, and each run is cut into tiles of up to 128 keys,
// so only the last tile of a run is partial.  Entry = (first row << 7) | (valid keys - 1).
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) build_key_tiles_kernel(
    const uint8_t *__restrict__ sel, const int32_t *__restrict__ kstart,
    const int32_t *__restrict__ ksize, long long rows, int Cq, int Ck, int tstride,
    int32_t *__restrict__ tiles, int32_t *__restrict__ tcnt) {
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= rows) return;
    const long long bh = row / Cq;
    const uint8_t *sr = sel + row * Ck;
    int32_t *out = tiles + row * tstride;
    int pos = 0, rs = 0, re = 0;  // the open run of keys [rs, re)
    bool overflow = false;
    auto flush = [&]() {
        if (re > rs) {
            const int nt = (re - rs + 127) >> 7;
            for (int t = lane; t < nt; t += 32) {
                const int r0 = rs + 128 * t;
                if (pos + t < tstride) out[pos + t] = (r0 << 7) | (min(128, re - r0) - 1);
            }
            if (pos + nt > tstride) overflow = true;
            pos = min(pos + nt, tstride);
        }
    };
    for (int j0 = 0; j0 < Ck; j0 += 32) {
        const int j = j0 + lane;
        int st = 0, sz = 0;
        if (j < Ck && sr[j]) {
            st = kstart[bh * Ck + j];
            sz = ksize[bh * Ck + j];
        }
        uint32_t b = __ballot_sync(0xffffffffu, sz > 0);
        while (b) {  // warp-uniform
            const int src = __ffs(b) - 1;
            b &= b - 1;
            const int s = __shfl_sync(0xffffffffu, st, src);
            const int len = __shfl_sync(0xffffffffu, sz, src);
            if (re > rs && s == re) {
                re += len;
            } else {
                flush();
                rs = s;
                re = s + len;
            }
        }
    }
    flush();
    if (lane == 0) {
        tcnt[row] = pos;
        if (overflow) atomicOr(&g_bsa_device_error, BSA_DEVERR_BOUNDS);
    }
}

// dst[bh, s, :] = src[bh, perm[bh, s], :], token rows moved as 16-byte vectors.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4 *__restrict__ src,
                                                          uint4 *__restrict__ dst,
                                                          const int32_t *__restrict__ perm,
                                                          long long rows, int N, int vec) {
    const long long total = rows * vec;
    for (long long x = (long long)blockIdx.x * blockDim.x + threadIdx.x; x < total;
         x += (long long)gridDim.x * blockDim.x) {
        const long long row = x / vec;
        const int c = (int)(x - row * vec);
        const long long bh = row / N;
        const int n = min(max(perm[row], 0), N - 1);
        dst[x] = src[(bh * N + n) * vec + c];
    }
}

}  // namespace bsa

namespace bsa {

// ------------------------------------------------------------------------------------------
// nearest centroid on the tensor cores
// ------------------------------------------------------------------------------------------
// For a 128-token tile of one head, the nearest centroid is argmin_c |c|^2 - 2 x.c (|x|^2 is
// common to every c).  The dot products x.c are a 128 x C x d contraction: x is bf16 already
// (exact), each fp32 centroid is split exactly into three bf16 parts c = h + m + l
// (centroid_split_kernel), and the three products x.h + x.m + x.l accumulate in one fp32
// tensor-memory tile, so the result is an fp32 dot product up to accumulation rounding.
//
// Work items are (head, 128-centroid tile, 128-token tile), ordered by (head, centroid tile)
// and then token tile; persistent CTAs (one per SM) own contiguous runs of that order, so a
// CTA keeps one centroid tile's three parts resident in shared memory while the token tiles
// stream past it:
//   warp 0 lane 0  TMA producer: the parts on every change of (head, centroid tile), token
//                  tiles into a 3-stage ring
//   warp 1 lane 0  MMA issuer: 3 x d/16 MMAs per item into one of two accumulators
//   warp 2         tensor-memory allocator (2 x 128 columns)
//   warps 4..7     epilogue: thread = token; the first minimum of |c|^2 - 2 x.c over the
//                  tile's centroids (the lower index on a tie, as Lloyd's step is read).  With
//                  one centroid tile this is the assignment; with several, each tile's
//                  (distance, index) goes out packed as an order-preserving 64-bit key and
//                  kmeans_merge_kernel keeps the least, which is again the first minimum.
template <int D>
struct KmTcCfg {
    static constexpr int CHUNKS = D / 64;
    static constexpr int TILE = CHUNKS * 16384;  // 128 rows x D bf16, 128-byte swizzled chunks
    static constexpr int NX = 3;                 // token-tile stages
    static constexpr int OFF_P = 0;              // part p of the resident centroid tile
    static constexpr int OFF_X = 3 * TILE;       // stage s of the token-tile ring
    static constexpr int OFF_BAR = OFF_X + NX * TILE;
    static constexpr int SMEM = OFF_BAR + 128 + 1024;  // + alignment slack
};

enum { KB_PF, KB_PE, KB_XF0, KB_XE0 = KB_XF0 + 3, KB_AF0 = KB_XE0 + 3, KB_AE0 = KB_AF0 + 2,
       KB_FIN = KB_AE0 + 2, KB_COUNT };

struct KmParams {
    const float *norms;     // [BH, C] |c|^2
    int32_t *assign;        // [BH, N], written when T == 1
    uint64_t *partial;      // [T, BH, N] packed (distance key, index), written when T > 1
    long long BH, total;    // heads; items = BH * T * NT
    int N, C, T, NT;        // tokens, centroids, centroid tiles, token tiles
    unsigned long long wait_ns;
};

// order-preserving key of a float (-0 taken as +0), in the high half; the index in the low half
__device__ __forceinline__ uint64_t pack_dist(float dist, int idx) {
    const uint32_t u = __float_as_uint(dist + 0.0f);
    const uint32_t key = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((uint64_t)key << 32) | (uint32_t)idx;
}

template <int D>
__global__ void __launch_bounds__(256, 1)
    kmeans_assign_tc_kernel(const __grid_constant__ CUtensorMap tmX,
                            const __grid_constant__ CUtensorMap tmP, const KmParams prm) {
    using Cf = KmTcCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cf::OFF_BAR);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + Cf::OFF_BAR + 8 * KB_COUNT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Cf::OFF_BAR + 8 * KB_COUNT + 4);
    static_assert(8 * KB_COUNT + 8 <= 128, "barrier area");

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long lo = prm.total * blockIdx.x / gridDim.x;
    const long long hi = prm.total * (blockIdx.x + 1) / gridDim.x;
    const unsigned long long wns = prm.wait_ns;
    auto bar = [&](int b) { return smem_u32(&bars[b]); };
    const uint32_t sP = smem_u32(smem + Cf::OFF_P), sX = smem_u32(smem + Cf::OFF_X);

    if (threadIdx.x == 0) {
        mbar_init(bar(KB_PF), 1);
        mbar_init(bar(KB_PE), 1);
        for (int s = 0; s < Cf::NX; ++s) {
            mbar_init(bar(KB_XF0 + s), 1);
            mbar_init(bar(KB_XE0 + s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(bar(KB_AF0 + a), 1);
            mbar_init(bar(KB_AE0 + a), 4);
        }
        mbar_init(bar(KB_FIN), 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmX);
        prefetch_tmap(&tmP);
    }
    if (warp == 2) {
        tmem_alloc(smem_u32(tmem_holder), 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_holder;

    if (warp == 0) {
        // ------------------------------------------------------------------ producer
        bool ok = true;
        uint32_t np = 0, nx = 0;
        long long cur = -1;
        for (long long t = lo; t < hi && ok; ++t) {
            const long long g = t / prm.NT;  // (head, centroid tile)
            const int tt = (int)(t - g * prm.NT);
            const int bh = (int)(g / prm.T), ct = (int)(g - (long long)bh * prm.T);
            if (g != cur) {
                if (np > 0 && !(ok = warp_wait(bar(KB_PE), (np - 1) & 1, wns, abort_flag, 0x91, (uint32_t)t)))
                    break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar(KB_PF), 3 * Cf::TILE);
                    for (int p = 0; p < 3; ++p)
                        for (int c = 0; c < Cf::CHUNKS; ++c)
                            tma_load_3d(sP + p * Cf::TILE + c * 16384, &tmP, bar(KB_PF), c * 64, ct * 128,
                                        bh * 3 + p);
                }
                ++np;
                cur = g;
            }
            const int s = nx % Cf::NX;
            if (nx >= Cf::NX &&
                !(ok = warp_wait(bar(KB_XE0 + s), ((nx / Cf::NX) - 1) & 1, wns, abort_flag, 0x92, (uint32_t)t)))
                break;
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(KB_XF0 + s), Cf::TILE);
                for (int c = 0; c < Cf::CHUNKS; ++c)
                    tma_load_3d(sX + s * Cf::TILE + c * 16384, &tmX, bar(KB_XF0 + s), c * 64, tt * 128, bh);
            }
            ++nx;
        }
        if (!ok && lane == 0) {  // every started copy lands before the CTA leaves
            if (np) drain_wait(bar(KB_PF), (np - 1) & 1, wns, 0x98);
            for (uint32_t i = nx > Cf::NX ? nx - Cf::NX : 0; i < nx; ++i)
                drain_wait(bar(KB_XF0 + i % Cf::NX), (i / Cf::NX) & 1, wns, 0x99);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        constexpr uint32_t IDESC = idesc_bf16_f32(128, 128, 0, 0);
        const uint64_t dP = smem_desc_sw128(sP, 16, 1024);
        const uint64_t dX = smem_desc_sw128(sX, 16, 1024);
        bool ok = true;
        uint32_t np = 0, nx = 0;
        long long cur = -1;
        for (long long t = lo; t < hi && ok; ++t) {
            const long long g = t / prm.NT;
            if (g != cur) {
                if (!(ok = warp_wait(bar(KB_PF), np & 1, wns, abort_flag, 0xA1, (uint32_t)t))) break;
                ++np;
                cur = g;
            }
            const int s = nx % Cf::NX, a = nx & 1;  // token stage, accumulator
            if (!(ok = warp_wait(bar(KB_XF0 + s), (nx / Cf::NX) & 1, wns, abort_flag, 0xA2, (uint32_t)t))) break;
            if (nx >= 2 && !(ok = warp_wait(bar(KB_AE0 + a), ((nx >> 1) - 1) & 1, wns, abort_flag, 0xA3, (uint32_t)t)))
                break;
            tc_fence_after();
            const bool last_of_group = t + 1 >= hi || (t + 1) / prm.NT != g;
            if (lane == 0) {
                const uint32_t acc = tbase + (uint32_t)(a * 128);
                const uint64_t xs = (uint64_t)((s * Cf::TILE) >> 4);
#pragma unroll
                for (int p = 0; p < 3; ++p) {
                    const uint64_t ps = (uint64_t)((p * Cf::TILE) >> 4);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t off = (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
                        mma_ss(acc, dX + xs + off, dP + ps + off, IDESC, (p > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                mma_commit(bar(KB_AF0 + a));
                mma_commit(bar(KB_XE0 + s));
                if (last_of_group) mma_commit(bar(KB_PE));
            }
            __syncwarp();
            ++nx;
        }
        if (lane == 0) {  // every MMA complete before tensor memory is released
            mma_commit(bar(KB_FIN));
            drain_wait(bar(KB_FIN), 0, wns, 0xA4);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------------ epilogue
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;  // token row of the tile == TMEM lane
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        bool ok = true;
        uint32_t nx = 0;
        long long cur = -1;
        float nv[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
        for (long long t = lo; t < hi && ok; ++t) {
            const long long g = t / prm.NT;
            const int tt = (int)(t - g * prm.NT);
            const int bh = (int)(g / prm.T), ct = (int)(g - (long long)bh * prm.T);
            if (g != cur) {
                // lane e holds the norm of column q * 32 + e (padding centroids are never nearest)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int c = ct * 128 + q * 32 + lane;
                    nv[q] = c < prm.C ? prm.norms[(size_t)bh * prm.C + c] : INFINITY;
                }
                cur = g;
            }
            const int a = nx & 1;  // accumulator
            if (!(ok = warp_wait(bar(KB_AF0 + a), (nx >> 1) & 1, wns, abort_flag, 0xB1, (uint32_t)t))) break;
            tc_fence_after();
            // four independent first-minimum chains (one per 32 columns), merged in column order
            float bq[4];
            int aq[4];
            uint32_t v[128];
            tmem_ld_cols<128>(tbase + lane_off + (uint32_t)(a * 128), v);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                bq[q] = INFINITY;
                aq[q] = ct * 128 + q * 32;
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const float cn = __shfl_sync(0xffffffffu, nv[q], e);
                    const float dist = fmaf(-2.f, __uint_as_float(v[q * 32 + e]), cn);
                    if (dist < bq[q]) {
                        bq[q] = dist;
                        aq[q] = ct * 128 + q * 32 + e;
                    }
                }
            }
            float best = bq[0];
            int arg = aq[0];
#pragma unroll
            for (int q = 1; q < 4; ++q) {
                if (bq[q] < best) {
                    best = bq[q];
                    arg = aq[q];
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(KB_AE0 + a));
            const int n = tt * 128 + r;
            if (n < prm.N) {
                if (prm.T == 1)
                    prm.assign[(size_t)bh * prm.N + n] = arg;
                else
                    prm.partial[((size_t)ct * prm.BH + bh) * prm.N + n] = pack_dist(best, arg);
            }
            ++nx;
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 2) tmem_dealloc(tbase, 256);
}

// assign[x] = the index of the least packed (distance, index) over the T centroid tiles
__global__ void __launch_bounds__(256) kmeans_merge_kernel(const uint64_t *__restrict__ partial,
                                                           int32_t *__restrict__ assign,
                                                           long long total, int T) {
    for (long long x = (long long)blockIdx.x * blockDim.x + threadIdx.x; x < total;
         x += (long long)gridDim.x * blockDim.x) {
        uint64_t b = partial[x];
        for (int t = 1; t < T; ++t) {
            const uint64_t v = partial[(size_t)t * total + x];
            b = v < b ? v : b;
        }
        assign[x] = (int32_t)(uint32_t)(b & 0xFFFFFFFFull);
    }
}

// parts[bh, p, c, :] (p = 0, 1, 2: h, m, l of cent[bh, c, :]) and norms[bh, c] = |cent[bh, c]|^2
template <int D>
__global__ void __launch_bounds__(256) centroid_split_kernel(const float *__restrict__ cent,
                                                             __nv_bfloat16 *__restrict__ parts,
                                                             float *__restrict__ norms, int C) {
    const int bh = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x * 8 + warp;
    if (c >= C) return;
    const float *src = cent + ((size_t)bh * C + c) * D;
    uint16_t *dst = reinterpret_cast<uint16_t *>(parts);
    float s = 0.f;
    for (int e = lane; e < D; e += 32) {
        const float x = src[e];
        s = fmaf(x, x, s);
        const uint32_t h = __float_as_uint(x) & 0xFFFF0000u;
        const float rm = x - __uint_as_float(h);
        const uint32_t m = __float_as_uint(rm) & 0xFFFF0000u;
        const uint32_t l = __float_as_uint(rm - __uint_as_float(m));
        const size_t base = (((size_t)bh * 3) * C + c) * D + e;
        dst[base] = (uint16_t)(h >> 16);
        dst[base + (size_t)C * D] = (uint16_t)(m >> 16);
        dst[base + 2 * (size_t)C * D] = (uint16_t)(l >> 16);
    }
    s = warp_sum(s);
    if (lane == 0) norms[(size_t)bh * C + c] = s;
}

}  // namespace bsa

namespace bsa {

template <int D>
static cudaError_t launch_assign_tc(const CUtensorMap &tx, const CUtensorMap &tp, const KmParams &p,
                                    cudaStream_t st) {
    using Cf = KmTcCfg<D>;
    cudaError_t e = cudaFuncSetAttribute(kmeans_assign_tc_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::SMEM);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long long grid = p.total < sms ? p.total : sms;
    if (grid <= 0) return cudaSuccess;
    kmeans_assign_tc_kernel<D><<<(unsigned)grid, 256, Cf::SMEM, st>>>(tx, tp, p);
    e = cudaGetLastError();
    if (e != cudaSuccess || p.T == 1) return e;
    const long long n = p.BH * p.N;
    const long long blocks = (n + 255) / 256 < 16LL * sms ? (n + 255) / 256 : 16LL * sms;
    kmeans_merge_kernel<<<(unsigned)blocks, 256, 0, st>>>(p.partial, p.assign, n, p.T);
    return cudaGetLastError();
}

// partial: [ceil(C / 128), BH, N] uint64 scratch, used when C > 128
cudaError_t kmeans_assign_tc(const CUtensorMap &tx, const CUtensorMap &tp, const float *norms,
                             int32_t *assign, uint64_t *partial, long long BH, int N, int d, int C,
                             unsigned long long wait_ns, cudaStream_t st) {
    KmParams p;
    p.norms = norms;
    p.assign = assign;
    p.partial = partial;
    p.BH = BH;
    p.N = N;
    p.C = C;
    p.T = (C + 127) / 128;
    p.NT = (N + 127) / 128;
    p.total = BH * p.T * p.NT;
    p.wait_ns = wait_ns;
    if (d == 128) return launch_assign_tc<128>(tx, tp, p, st);
    if (d == 64) return launch_assign_tc<64>(tx, tp, p, st);
    return cudaErrorInvalidValue;
}

cudaError_t centroid_split(const float *cent, void *parts, float *norms, long long BH, int C,
                           int d, cudaStream_t st) {
    const dim3 g((unsigned)((C + 7) / 8), (unsigned)BH);
    auto *p = reinterpret_cast<__nv_bfloat16 *>(parts);
    if (d == 128)
        centroid_split_kernel<128><<<g, 256, 0, st>>>(cent, p, norms, C);
    else
        centroid_split_kernel<64><<<g, 256, 0, st>>>(cent, p, norms, C);
    return cudaGetLastError();
}

}  // namespace bsa

namespace bsa {

// ------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------
static unsigned grid_for(long long work, int per_block, int num_sms) {
    long long g = (work + per_block - 1) / per_block;
    const long long cap = (long long)num_sms * 16;
    if (g > cap) g = cap;
    return (unsigned)(g > 0 ? g : 1);
}

// parts: [BH, 3, C, d] bf16, norms [BH, C] fp32 and (C > 128) partial [ceil(C / 128), BH, N]
// uint64 scratch for the tensor-core assignment; tx / tp: tensor maps of x ({d, N, BH},
// 128-row boxes) and of parts ({d, C, 3 BH}, 128-row boxes).
cudaError_t kmeans_lloyd(const void *x, float *cent, int32_t *assign, int32_t *perm,
                         int32_t *cstart, int32_t *csize, long long BH, int N, int d, int C,
                         int iters, void *parts, float *norms, uint64_t *partial, int32_t *hist,
                         const CUtensorMap *tx, const CUtensorMap *tp, unsigned long long wait_ns,
                         cudaStream_t st) {
    const dim3 gu((unsigned)C, (unsigned)BH);
    const auto *xb = reinterpret_cast<const __nv_bfloat16 *>(x);
    for (int it = 0;; ++it) {
        cudaError_t e = centroid_split(cent, parts, norms, BH, C, d, st);
        if (e == cudaSuccess)
            e = kmeans_assign_tc(*tx, *tp, norms, assign, partial, BH, N, d, C, wait_ns, st);
        if (e != cudaSuccess) return e;
        e = cluster_sort(assign, BH, N, C, perm, cstart, csize, hist, st);
        if (e != cudaSuccess) return e;
        if (it == iters) break;
        if (d == 128)
            kmeans_update_kernel<128><<<gu, 512, 0, st>>>(xb, perm, cstart, csize, cent, N, C);
        else
            kmeans_update_kernel<64><<<gu, 512, 0, st>>>(xb, perm, cstart, csize, cent, N, C);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

// hist: [BH, ceil(N / kSortChunk), C] int32 scratch
cudaError_t cluster_sort(const int32_t *assign, long long BH, int N, int C, int32_t *perm,
                         int32_t *cstart, int32_t *csize, int32_t *hist, cudaStream_t st) {
    const int nchunk = (N + kSortChunk - 1) / kSortChunk;
    const dim3 g((unsigned)nchunk, (unsigned)BH);
    cluster_hist_kernel<<<g, 256, (size_t)C * sizeof(int32_t), st>>>(assign, N, C, nchunk, hist);
    cluster_scan_kernel<<<(unsigned)BH, 1024, 0, st>>>(hist, nchunk, C, cstart, csize);
    cluster_place_kernel<<<g, 256, (size_t)8 * C * sizeof(int32_t), st>>>(assign, hist, N, C, nchunk,
                                                                          perm);
    return cudaGetLastError();
}

size_t cluster_sort_scratch_bytes(long long BH, int N, int C) {
    return (size_t)BH * ((N + kSortChunk - 1) / kSortChunk) * C * sizeof(int32_t);
}

cudaError_t centroid_logits(const float *cq, const float *ck, const int32_t *size_k,
                            float *logits, long long BH, int Cq, int Ck, int d, float scale,
                            cudaStream_t st) {
    const dim3 g((unsigned)((Cq + 7) / 8), (unsigned)BH);
    if (d == 128)
        centroid_logits_kernel<128><<<g, 256, 0, st>>>(cq, ck, size_k, logits, Cq, Ck, scale);
    else
        centroid_logits_kernel<64><<<g, 256, 0, st>>>(cq, ck, size_k, logits, Cq, Ck, scale);
    return cudaGetLastError();
}

cudaError_t prune_empty(uint8_t *sel, const int32_t *size_k, long long BH, int Cq, int Ck,
                        int num_sms, cudaStream_t st) {
    const long long rows = BH * Cq;
    prune_empty_kernel<<<grid_for(rows * Ck, 256, num_sms), 256, 0, st>>>(sel, size_k, rows, Cq, Ck);
    return cudaGetLastError();
}

cudaError_t build_cluster_tables(const uint8_t *sel, const int32_t *qstart, const int32_t *qsize,
                                 const int32_t *kstart, const int32_t *ksize, long long BH,
                                 int Cq, int Ck, int U, int tstride, int2 *units, int32_t *tiles,
                                 int32_t *tcnt, cudaStream_t st) {
    build_units_kernel<<<(unsigned)((BH + 7) / 8), 256, 0, st>>>(qstart, qsize, BH, Cq, U, units);
    const long long rows = BH * Cq;
    build_key_tiles_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(sel, kstart, ksize, rows, Cq,
                                                                       Ck, tstride, tiles, tcnt);
    return cudaGetLastError();
}

cudaError_t gather_rows(const void *src, const int32_t *perm, void *dst, long long BH, int N,
                        int d, int num_sms, cudaStream_t st) {
    const int vec = d / 8;
    const long long rows = BH * N;
    gather_rows_kernel<<<grid_for(rows * vec, 256, num_sms), 256, 0, st>>>(
        reinterpret_cast<const uint4 *>(src), reinterpret_cast<uint4 *>(dst), perm, rows, N, vec);
    return cudaGetLastError();
}

}  // namespace bsa

// ------------------------------------------------------------------------------------------
// C ABI
// ------------------------------------------------------------------------------------------
namespace {

size_t round256(size_t b) { return (b + 255) & ~(size_t)255; }

// Carves the caller's workspace.  Every region starts on a 256-byte boundary.
struct ClusterWorkspace {
    unsigned int *counter;
    int32_t *perm_q, *perm_k, *qstart, *qsize, *kstart, *ksize, *tiles, *tcnt;
    int2 *units;
    void *qp, *kp, *vp;
    // the full path only: assignments, centroid scores (then the selection's id lists) and counts
    int32_t *assign_q, *assign_k, *sel_cnt;
    float *logits;
    void *parts;   // centroid parts for the tensor-core assignment, sized for max(Cq, Ck)
    float *norms;
    uint64_t *partial;  // per-centroid-tile nearest candidates, when max(Cq, Ck) > 128
    int32_t *hist;      // cluster-sort chunk counts
    int U, tstride;
};

size_t cluster_workspace(int B, int H, int N, int d, int Cq, int Ck, bool full, void *base,
                         ClusterWorkspace *w) {
    const size_t BH = (size_t)B * H;
    const int nbt = (N + 127) / 128;
    const int U = nbt + Cq, tstride = nbt + Ck;
    size_t off = 0;
    uint8_t *p = reinterpret_cast<uint8_t *>(base);
    auto take = [&](size_t bytes) -> void * {
        void *r = p ? p + off : nullptr;
        off += round256(bytes);
        return r;
    };
    ClusterWorkspace t;
    t.counter = (unsigned int *)take(kAttnWorkspaceBytes);
    t.perm_q = (int32_t *)take(BH * N * 4);
    t.perm_k = (int32_t *)take(BH * N * 4);
    t.qstart = (int32_t *)take(BH * Cq * 4);
    t.qsize = (int32_t *)take(BH * Cq * 4);
    t.kstart = (int32_t *)take(BH * Ck * 4);
    t.ksize = (int32_t *)take(BH * Ck * 4);
    t.tiles = (int32_t *)take(BH * Cq * (size_t)tstride * 4);
    t.tcnt = (int32_t *)take(BH * Cq * 4);
    t.units = (int2 *)take(BH * (size_t)U * 8);
    t.qp = take(BH * N * (size_t)d * 2);
    t.kp = take(BH * N * (size_t)d * 2);
    t.vp = take(BH * N * (size_t)d * 2);
    t.assign_q = t.assign_k = t.sel_cnt = nullptr;
    t.logits = nullptr;
    t.parts = nullptr;
    t.norms = nullptr;
    t.partial = nullptr;
    t.hist = (int32_t *)take(bsa::cluster_sort_scratch_bytes((long long)BH, N, Cq > Ck ? Cq : Ck));
    if (full) {
        t.assign_q = (int32_t *)take(BH * N * 4);
        t.assign_k = (int32_t *)take(BH * N * 4);
        t.logits = (float *)take(BH * Cq * (size_t)Ck * 4);
        t.sel_cnt = (int32_t *)take(BH * Cq * 4);
        const size_t Cm = (size_t)(Cq > Ck ? Cq : Ck);
        t.parts = take(BH * 3 * Cm * d * 2);
        t.norms = (float *)take(BH * Cm * 4);
        t.partial = Cm > 128 ? (uint64_t *)take(((Cm + 127) / 128) * BH * N * 8) : nullptr;
    }
    t.U = U;
    t.tstride = tstride;
    if (w) *w = t;
    return off;
}

bool clusters_ok(int C) { return C >= 1 && C <= bsa::kMaxClusters; }

// Shape checks shared by the cluster entry points.
sa_status cluster_shape(int B, int H, int N, int d, int Cq, int Ck) {
    if (!shape_ok(B, H, N) || !clusters_ok(Cq) || !clusters_ok(Ck)) return SA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return SA_ERR_UNSUPPORTED;
    if (N >= bsa::kMaxVarlenN) return SA_ERR_UNSUPPORTED;
    const long long units = (long long)B * H * ((N + 127) / 128 + Cq);
    if (units > 0x7FFFFFFFLL) return SA_ERR_UNSUPPORTED;
    return SA_OK;
}

// Tables, permuted tensors and the attention, from the two permutations and the selection.
sa_status cluster_attention_tail(const void *q, const void *k, const void *v, void *o,
                                 const uint8_t *sel, const ClusterWorkspace &w, int B, int H,
                                 int N, int d, int Cq, int Ck, float scale, int dev,
                                 cudaStream_t st) {
    const long long BH = (long long)B * H;
    const int sms = num_sms(dev);
    cudaError_t e = bsa::build_cluster_tables(sel, w.qstart, w.qsize, w.kstart, w.ksize, BH, Cq, Ck,
                                              w.U, w.tstride, w.units, w.tiles, w.tcnt, st);
    if (e == cudaSuccess) e = bsa::gather_rows(q, w.perm_q, w.qp, BH, N, d, sms, st);
    if (e == cudaSuccess) e = bsa::gather_rows(k, w.perm_k, w.kp, BH, N, d, sms, st);
    if (e == cudaSuccess) e = bsa::gather_rows(v, w.perm_k, w.vp, BH, N, d, sms, st);
    if (e != cudaSuccess) return SA_ERR_CUDA;
    CUtensorMap tq, tk, tv;
    if (!make_tmap(&tq, w.qp, BH, N, d, 128) || !make_tmap(&tk, w.kp, BH, N, d, 128) ||
        !make_tmap(&tv, w.vp, BH, N, d, 128))
        return SA_ERR_CUDA;
    return from_cuda(bsa::attn_varlen_fwd(tq, tk, tv, w.units, w.U, w.tiles, w.tcnt, w.tstride,
                                          w.perm_q, o, BH, N, N, Cq, d, resolve_scale(scale, d),
                                          g_wait_ns, sms, w.counter, st));
}

// Centroid scores, top-p and the removal of empty clusters; logits doubles as the id list.
cudaError_t centroid_select(const float *cq, const float *ck, const int32_t *size_k, long long BH,
                            int Cq, int Ck, int d, float topp, float scale, uint8_t *sel,
                            float *logits, int32_t *sel_cnt, int sms, cudaStream_t st) {
    cudaError_t e = bsa::centroid_logits(cq, ck, size_k, logits, BH, Cq, Ck, d, scale, st);
    if (e == cudaSuccess)
        e = bsa::select_rows(logits, BH * Cq, Ck, 0, topp, sel,
                             reinterpret_cast<int32_t *>(logits), sel_cnt, st);
    if (e == cudaSuccess) e = bsa::prune_empty(sel, size_k, BH, Cq, Ck, sms, st);
    return e;
}

}  // namespace

extern "C" size_t sa_kmeans_workspace_bytes(int B, int H, int N, int C, int d) {
    if (B <= 0 || H <= 0 || N <= 0 || C <= 0 || d <= 0) return 0;
    const size_t BH = (size_t)B * H;
    const size_t T = ((size_t)C + 127) / 128;
    return round256(BH * 3 * (size_t)C * d * 2) + round256(BH * (size_t)C * 4) +
           (T > 1 ? round256(T * BH * (size_t)N * 8) : 0) +
           round256(bsa::cluster_sort_scratch_bytes((long long)BH, N, C));
}

extern "C" sa_status sa_kmeans(const void *x, float *cent, int32_t *assign, int32_t *perm,
                               int32_t *cstart, int32_t *csize, int B, int H, int N, int d, int C,
                               int iters, void *workspace, size_t workspace_bytes, void *stream) {
    if (!x || !cent || !assign || !perm || !cstart || !csize || !workspace) return SA_ERR_INVALID_ARG;
    if (!shape_ok(B, H, N) || !clusters_ok(C) || iters < 0) return SA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return SA_ERR_UNSUPPORTED;
    if (workspace_bytes < sa_kmeans_workspace_bytes(B, H, N, C, d) || !aligned16(workspace))
        return SA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(cent) || !aligned4(assign) || !aligned4(perm) ||
        !aligned4(cstart) || !aligned4(csize))
        return SA_ERR_INVALID_ARG;
    int dev;
    if (!select_device(assign, &dev)) return SA_ERR_INVALID_ARG;
    const long long BH = (long long)B * H;
    void *parts = workspace;
    float *norms = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(workspace) +
                                             round256((size_t)BH * 3 * C * d * 2));
    uint8_t *after_norms = reinterpret_cast<uint8_t *>(norms) + round256((size_t)BH * C * 4);
    uint64_t *partial = C > 128 ? reinterpret_cast<uint64_t *>(after_norms) : nullptr;
    const size_t T = ((size_t)C + 127) / 128;
    int32_t *hist = reinterpret_cast<int32_t *>(after_norms +
                                                (T > 1 ? round256(T * BH * (size_t)N * 8) : 0));
    CUtensorMap tx, tp;
    if (!make_tmap(&tx, x, BH, N, d, 128) || !make_tmap(&tp, parts, BH * 3, C, d, 128))
        return SA_ERR_CUDA;
    return from_cuda(bsa::kmeans_lloyd(x, cent, assign, perm, cstart, csize, BH, N, d, C, iters,
                                       parts, norms, partial, hist, &tx, &tp, g_wait_ns,
                                       (cudaStream_t)stream));
}

extern "C" size_t sa_cluster_sort_workspace_bytes(int B, int H, int N, int C) {
    if (B <= 0 || H <= 0 || N <= 0 || C <= 0) return 0;
    return round256(bsa::cluster_sort_scratch_bytes((long long)B * H, N, C));
}

extern "C" sa_status sa_cluster_sort(const int32_t *assign, int B, int H, int N, int C,
                                     int32_t *perm, int32_t *cstart, int32_t *csize,
                                     void *workspace, size_t workspace_bytes, void *stream) {
    if (!assign || !perm || !cstart || !csize || !workspace) return SA_ERR_INVALID_ARG;
    if (!shape_ok(B, H, N) || !clusters_ok(C)) return SA_ERR_INVALID_ARG;
    if (!aligned4(assign) || !aligned4(perm) || !aligned4(cstart) || !aligned4(csize))
        return SA_ERR_INVALID_ARG;
    if (workspace_bytes < sa_cluster_sort_workspace_bytes(B, H, N, C) || !aligned16(workspace))
        return SA_ERR_INVALID_ARG;
    int dev;
    if (!select_device(perm, &dev)) return SA_ERR_INVALID_ARG;
    return from_cuda(bsa::cluster_sort(assign, (long long)B * H, N, C, perm, cstart, csize,
                                       reinterpret_cast<int32_t *>(workspace),
                                       (cudaStream_t)stream));
}

extern "C" size_t sa_centroid_topp_workspace_bytes(int B, int H, int Cq, int Ck) {
    if (B <= 0 || H <= 0 || Cq <= 0 || Ck <= 0) return 0;
    const size_t BH = (size_t)B * H;
    return round256(BH * Cq * (size_t)Ck * 4) + round256(BH * Cq * 4);
}

extern "C" sa_status sa_centroid_topp(const float *cq, const float *ck, const int32_t *size_k,
                                      int B, int H, int Cq, int Ck, int d, float topp, float scale,
                                      uint8_t *sel, void *workspace, size_t workspace_bytes,
                                      void *stream) {
    if (!cq || !ck || !size_k || !sel || !workspace) return SA_ERR_INVALID_ARG;
    if (!shape_ok(B, H, 1) || !clusters_ok(Cq) || !clusters_ok(Ck)) return SA_ERR_INVALID_ARG;
    if (!(topp >= 0.f && topp <= 1.f) || isnan(scale)) return SA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return SA_ERR_UNSUPPORTED;
    if (workspace_bytes < sa_centroid_topp_workspace_bytes(B, H, Cq, Ck) || !aligned16(workspace))
        return SA_ERR_INVALID_ARG;
    if (!aligned4(cq) || !aligned4(ck) || !aligned4(size_k)) return SA_ERR_INVALID_ARG;
    int dev;
    if (!select_device(sel, &dev)) return SA_ERR_INVALID_ARG;
    const long long BH = (long long)B * H;
    float *logits = reinterpret_cast<float *>(workspace);
    int32_t *cnt = reinterpret_cast<int32_t *>(reinterpret_cast<uint8_t *>(workspace) +
                                               round256((size_t)BH * Cq * Ck * 4));
    return from_cuda(centroid_select(cq, ck, size_k, BH, Cq, Ck, d, topp, resolve_scale(scale, d),
                                     sel, logits, cnt, num_sms(dev), (cudaStream_t)stream));
}

extern "C" size_t sa_cluster_attn_workspace_bytes(int B, int H, int N, int d, int Cq, int Ck) {
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0 || Cq <= 0 || Ck <= 0) return 0;
    return cluster_workspace(B, H, N, d, Cq, Ck, false, nullptr, nullptr);
}

extern "C" sa_status sa_cluster_attn_fwd(const void *q, const void *k, const void *v, void *o,
                                         const int32_t *assign_q, const int32_t *assign_k,
                                         const uint8_t *sel, int B, int H, int N, int d, int Cq,
                                         int Ck, float scale, void *workspace,
                                         size_t workspace_bytes, void *stream) {
    if (!q || !k || !v || !o || !assign_q || !assign_k || !sel || !workspace)
        return SA_ERR_INVALID_ARG;
    const sa_status s = cluster_shape(B, H, N, d, Cq, Ck);
    if (s != SA_OK) return s;
    if (isnan(scale)) return SA_ERR_INVALID_ARG;
    if (workspace_bytes < sa_cluster_attn_workspace_bytes(B, H, N, d, Cq, Ck) ||
        !aligned16(workspace))
        return SA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(assign_q) ||
        !aligned4(assign_k))
        return SA_ERR_INVALID_ARG;
    int dev;
    if (!select_device(o, &dev)) return SA_ERR_INVALID_ARG;
    const cudaStream_t st = (cudaStream_t)stream;
    ClusterWorkspace w;
    cluster_workspace(B, H, N, d, Cq, Ck, false, workspace, &w);
    const long long BH = (long long)B * H;
    cudaError_t e = bsa::cluster_sort(assign_q, BH, N, Cq, w.perm_q, w.qstart, w.qsize, w.hist, st);
    if (e == cudaSuccess)
        e = bsa::cluster_sort(assign_k, BH, N, Ck, w.perm_k, w.kstart, w.ksize, w.hist, st);
    if (e != cudaSuccess) return SA_ERR_CUDA;
    return cluster_attention_tail(q, k, v, o, sel, w, B, H, N, d, Cq, Ck, scale, dev, st);
}

extern "C" size_t sa_svg2_workspace_bytes(int B, int H, int N, int d, int Cq, int Ck) {
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0 || Cq <= 0 || Ck <= 0) return 0;
    return cluster_workspace(B, H, N, d, Cq, Ck, true, nullptr, nullptr);
}

extern "C" sa_status sa_svg2_attn_fwd(const void *q, const void *k, const void *v, void *o,
                                      float *cent_q, float *cent_k, int B, int H, int N, int d,
                                      int Cq, int Ck, int iters, float topp, float scale,
                                      uint8_t *sel, void *workspace, size_t workspace_bytes,
                                      void *stream) {
    if (!q || !k || !v || !o || !cent_q || !cent_k || !sel || !workspace) return SA_ERR_INVALID_ARG;
    const sa_status s = cluster_shape(B, H, N, d, Cq, Ck);
    if (s != SA_OK) return s;
    if (iters < 0 || !(topp >= 0.f && topp <= 1.f) || isnan(scale)) return SA_ERR_INVALID_ARG;
    if (workspace_bytes < sa_svg2_workspace_bytes(B, H, N, d, Cq, Ck) || !aligned16(workspace))
        return SA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(cent_q) ||
        !aligned16(cent_k))
        return SA_ERR_INVALID_ARG;
    int dev;
    if (!select_device(o, &dev)) return SA_ERR_INVALID_ARG;
    const cudaStream_t st = (cudaStream_t)stream;
    ClusterWorkspace w;
    cluster_workspace(B, H, N, d, Cq, Ck, true, workspace, &w);
    const long long BH = (long long)B * H;
    CUtensorMap txq, txk, tpq, tpk;
    if (!make_tmap(&txq, q, BH, N, d, 128) || !make_tmap(&txk, k, BH, N, d, 128) ||
        !make_tmap(&tpq, w.parts, BH * 3, Cq, d, 128) || !make_tmap(&tpk, w.parts, BH * 3, Ck, d, 128))
        return SA_ERR_CUDA;
    cudaError_t e = bsa::kmeans_lloyd(q, cent_q, w.assign_q, w.perm_q, w.qstart, w.qsize, BH, N, d,
                                      Cq, iters, w.parts, w.norms, w.partial, w.hist, &txq, &tpq,
                                      g_wait_ns, st);
    if (e == cudaSuccess)
        e = bsa::kmeans_lloyd(k, cent_k, w.assign_k, w.perm_k, w.kstart, w.ksize, BH, N, d, Ck,
                              iters, w.parts, w.norms, w.partial, w.hist, &txk, &tpk, g_wait_ns,
                              st);
    if (e == cudaSuccess)
        e = centroid_select(cent_q, cent_k, w.ksize, BH, Cq, Ck, d, topp, resolve_scale(scale, d),
                            sel, w.logits, w.sel_cnt, num_sms(dev), st);
    if (e != cudaSuccess) return SA_ERR_CUDA;
    return cluster_attention_tail(q, k, v, o, sel, w, B, H, N, d, Cq, Ck, scale, dev, st);
}
