// Hybrid top-k + top-p block selection.
//
// SpargeAttention2 ("Top-kとTop-pの限界を解剖する", "ハイブリッドマスキングと蒸留微調整"): each query
// block keeps the union of its k most probable key blocks and the top-p prefix of key blocks.
// Sparse VideoGen2 (section 2.B): the estimated block scores are sorted and blocks are taken in
// order until the cumulative score reaches p.  The problem statement fixes the estimate as
// softmax(Qp Kp^T * scale) over pooled blocks.
//
// Two launches:
//   1. block_scores_kernel: fp32 SIMT GEMM L = scale * Qp Kp^T per (b, h), written into the
//      kv_idx buffer (same size: nb x nb 32-bit words per head), which doubles as staging.
//   2. select_rows_kernel: one warp per query-block row.  Softmax in fp32, bitonic sort of
//      (score, block id) keys in registers (ranking by score is ranking by probability), warp
//      prefix sum of the sorted probabilities for the top-p cut, union with top-k, then the 0/1
//      mask row, the ascending kv_idx list and kv_cnt.  The row's logits are read into
//      registers before any of the row's kv_idx entries is written.
//
// Because top-k and top-p both take prefixes of the same ranked order (probability descending,
// lower block id first), their union is the longer of the two prefixes: |keep| = max(min(k,nb), m).
#include "bsa_internal.h"

namespace bsa {

// ------------------------------------------------------------------------------------------
// 1. block scores
// ------------------------------------------------------------------------------------------
constexpr int SC_TILE = 64;
constexpr int SC_KC = 16;

__global__ void __launch_bounds__(256) block_scores_kernel(const float *__restrict__ qp,
                                                           const float *__restrict__ kp,
                                                           float *__restrict__ logits, int nb,
                                                           int d, float scale) {
    __shared__ __align__(16) float As[SC_KC][SC_TILE + 4];
    __shared__ __align__(16) float Bs[SC_KC][SC_TILE + 4];
    const int bh = blockIdx.z;
    const int i0 = blockIdx.y * SC_TILE;
    const int j0 = blockIdx.x * SC_TILE;
    const float *A = qp + (size_t)bh * nb * d;
    const float *Bm = kp + (size_t)bh * nb * d;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    const int lr = threadIdx.x / 4, lk = (threadIdx.x % 4) * 4;

    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;

    for (int c0 = 0; c0 < d; c0 += SC_KC) {
        float4 va = make_float4(0.f, 0.f, 0.f, 0.f), vb = va;
        if (i0 + lr < nb) va = *reinterpret_cast<const float4 *>(A + (size_t)(i0 + lr) * d + c0 + lk);
        if (j0 + lr < nb) vb = *reinterpret_cast<const float4 *>(Bm + (size_t)(j0 + lr) * d + c0 + lk);
        __syncthreads();
        As[lk + 0][lr] = va.x; As[lk + 1][lr] = va.y; As[lk + 2][lr] = va.z; As[lk + 3][lr] = va.w;
        Bs[lk + 0][lr] = vb.x; Bs[lk + 1][lr] = vb.y; Bs[lk + 2][lr] = vb.z; Bs[lk + 3][lr] = vb.w;
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < SC_KC; ++kk) {
            const float4 a = *reinterpret_cast<const float4 *>(&As[kk][ty * 4]);
            const float4 b = *reinterpret_cast<const float4 *>(&Bs[kk][tx * 4]);
            const float av[4] = {a.x, a.y, a.z, a.w};
            const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(av[x], bv[y], acc[x][y]);
        }
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) {
        const int i = i0 + ty * 4 + x;
        if (i >= nb) continue;
        float *row = logits + ((size_t)bh * nb + i) * nb;
#pragma unroll
        for (int y = 0; y < 4; ++y) {
            const int j = j0 + tx * 4 + y;
            if (j < nb) row[j] = acc[x][y] * scale;
        }
    }
}

// ------------------------------------------------------------------------------------------
// 2. per-row selection
// ------------------------------------------------------------------------------------------
constexpr int SEL_WARPS = 4;

// Order-preserving map of a finite float to uint32 (and back); -0 maps like +0.
__device__ __forceinline__ uint32_t ord_bits(float x) {
    uint32_t u = __float_as_uint(x);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float from_ord(uint32_t o) {
    return __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
}

template <int E>
__global__ void __launch_bounds__(SEL_WARPS * 32) select_rows_kernel(
    const float *logits, long long rows, int nb, int topk, float topp, uint8_t *__restrict__ mask,
    int32_t *kv_idx, int32_t *__restrict__ kv_cnt) {
    __shared__ __align__(16) uint8_t mrow_all[SEL_WARPS][32 * E];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const long long row = (long long)blockIdx.x * SEL_WARPS + warp;
    if (row >= rows) return;
    uint8_t *mrow = mrow_all[warp];
    const float *lg = logits + (size_t)row * nb;

    // element e = lane * E + r
    float x[E];
#pragma unroll
    for (int r = 0; r < E; ++r) {
        const int e = lane * E + r;
        x[r] = e < nb ? lg[e] : -INFINITY;
    }
    float mx = -INFINITY;
#pragma unroll
    for (int r = 0; r < E; ++r) mx = fmaxf(mx, x[r]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < E; ++r) s += (lane * E + r) < nb ? expf(x[r] - mx) : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);

    // Keys: the logit mapped to an order-preserving unsigned pattern, then ~id.  Ranking by the
    // logit is ranking by P (softmax is strictly increasing) but keeps the order of blocks whose
    // fp32 probability underflows to 0.  -0 is folded into +0 so that equal scores tie.
    unsigned long long key[E];
#pragma unroll
    for (int r = 0; r < E; ++r) {
        const int e = lane * E + r;
        key[r] = e < nb ? ((unsigned long long)ord_bits(x[r]) << 32) |
                              (0xFFFFFFFFu - (uint32_t)e)
                        : 0ull;
    }
    __syncwarp();

    // bitonic sort, descending, over 32*E elements
#pragma unroll
    for (int k = 2; k <= 32 * E; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            if (j < E) {
#pragma unroll
                for (int r = 0; r < E; ++r) {
                    const int l = r ^ j;
                    if (l > r) {
                        const bool up = ((lane * E + r) & k) == 0;
                        const unsigned long long a = key[r], b = key[l];
                        const bool swap = up ? (a < b) : (a > b);
                        key[r] = swap ? b : a;
                        key[l] = swap ? a : b;
                    }
                }
            } else {
                const int lx = j / E;
                const bool lower = (lane & lx) == 0;
                const bool up = ((lane * E) & k) == 0;
                const bool keep_max = (lower == up);
#pragma unroll
                for (int r = 0; r < E; ++r) {
                    const unsigned long long o = __shfl_xor_sync(0xffffffffu, key[r], lx);
                    key[r] = keep_max ? (key[r] > o ? key[r] : o) : (key[r] < o ? key[r] : o);
                }
            }
        }
    }

    // prefix sum of the sorted probabilities P = exp(L - max) / sum: lane-local, then across lanes
    float cum[E];
    float run = 0.f;
#pragma unroll
    for (int r = 0; r < E; ++r) {
        if (lane * E + r < nb) run += expf(from_ord((uint32_t)(key[r] >> 32)) - mx) / s;
        cum[r] = run;
    }
    float incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    float excl = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) excl = 0.f;
    int nlt = 0;
#pragma unroll
    for (int r = 0; r < E; ++r) nlt += ((lane * E + r) < nb && excl + cum[r] < topp) ? 1 : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) nlt += __shfl_xor_sync(0xffffffffu, nlt, o);
    int m;
    if (!(topp > 0.f))
        m = 0;
    else if (topp >= 1.f)
        m = nb;
    else
        m = nlt < nb ? nlt + 1 : nb;
    const int keep = max(min(topk, nb), m);

    // mask row in shared memory, by block id
#pragma unroll
    for (int r = 0; r < E; ++r) mrow[lane * E + r] = 0;
    __syncwarp();
#pragma unroll
    for (int r = 0; r < E; ++r) {
        const int e = lane * E + r;
        const uint32_t id = 0xFFFFFFFFu - (uint32_t)key[r];
        if (e < keep && id < (uint32_t)nb) mrow[id] = 1;
    }
    __syncwarp();
    uint8_t *mout = mask + (size_t)row * nb;
    for (int j = lane; j < nb; j += 32) mout[j] = mrow[j];

    // ascending compaction of kept ids
    int c = 0;
#pragma unroll
    for (int r = 0; r < E; ++r) c += mrow[lane * E + r];
    int ic = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, ic, o);
        if (lane >= o) ic += y;
    }
    int off = ic - c;
    int32_t *idx = kv_idx + (size_t)row * nb;
#pragma unroll
    for (int r = 0; r < E; ++r) {
        const int j = lane * E + r;
        if (mrow[j]) idx[off++] = j;
    }
    if (lane == 31) kv_cnt[row] = ic;
}

template <int E>
static cudaError_t launch_select_rows(const float *logits, long long rows, int nb, int topk,
                                      float topp, uint8_t *mask, int32_t *kv_idx, int32_t *kv_cnt,
                                      cudaStream_t st) {
    const long long grid = (rows + SEL_WARPS - 1) / SEL_WARPS;
    select_rows_kernel<E><<<(unsigned)grid, SEL_WARPS * 32, 0, st>>>(logits, rows, nb, topk, topp,
                                                                     mask, kv_idx, kv_cnt);
    return cudaGetLastError();
}

cudaError_t select_rows(const float *logits, long long rows, int nb, int topk, float topp,
                        uint8_t *mask, int32_t *kv_idx, int32_t *kv_cnt, cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    if (nb <= 32) return launch_select_rows<1>(logits, rows, nb, topk, topp, mask, kv_idx, kv_cnt, st);
    if (nb <= 64) return launch_select_rows<2>(logits, rows, nb, topk, topp, mask, kv_idx, kv_cnt, st);
    if (nb <= 128) return launch_select_rows<4>(logits, rows, nb, topk, topp, mask, kv_idx, kv_cnt, st);
    if (nb <= 256) return launch_select_rows<8>(logits, rows, nb, topk, topp, mask, kv_idx, kv_cnt, st);
    if (nb <= 512) return launch_select_rows<16>(logits, rows, nb, topk, topp, mask, kv_idx, kv_cnt, st);
    if (nb <= 1024) return launch_select_rows<32>(logits, rows, nb, topk, topp, mask, kv_idx, kv_cnt, st);
    return cudaErrorInvalidValue;
}

cudaError_t block_scores(const float *qp, const float *kp, float *logits, long long BH, int nb,
                         int d, float scale, cudaStream_t st) {
    if (BH == 0 || nb == 0) return cudaSuccess;
    dim3 grid((nb + SC_TILE - 1) / SC_TILE, (nb + SC_TILE - 1) / SC_TILE, (unsigned)BH);
    block_scores_kernel<<<grid, 256, 0, st>>>(qp, kp, logits, nb, d, scale);
    return cudaGetLastError();
}

}  // namespace bsa
