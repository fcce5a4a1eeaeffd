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
//   2. select_rows_kernel: one warp per query-block row.  Softmax in fp32, then the two
//      prefixes of the ranked order (score descending, id ascending; ranking by score is ranking
//      by probability) found by exact threshold searches over order-preserving score keys
//      instead of a full sort, the union, the 0/1 mask row, the ascending kv_idx list and
//      kv_cnt.  The row's logits are read into registers before any kv_idx entry is written.
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

// Order-preserving map of a finite float to uint32 (-0 maps like +0); 0 is below every score.
__device__ __forceinline__ uint32_t ord_bits(float x) {
    uint32_t u = __float_as_uint(x);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ int warp_isum(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// One warp per query-block row; element e = r*32 + lane (coalesced, index order is r-major).
//
// The ranked order is (score descending, block id ascending); key[e] is the score mapped to an
// order-preserving uint32, so "rank < R" is "key > T, or key == T and among the first few
// tied ids" for the right threshold T.  Both sets the pages define are prefixes of this order:
//   top-p: T_p = the largest key value whose mass  sum{P_e : key_e >= T_p} >= p  (bitwise
//          search, 32 steps, fp32 sums in a fixed order so they are monotone in T); then the
//          tied blocks at T_p are taken in id order until the mass reaches p;  m = their count
//          plus the blocks above T_p.
//   top-k: same search with the count  #{e : key_e >= T} >= k.
// Their union is the longer prefix, |keep| = max(min(k, nb), m).
template <int E>
__global__ void __launch_bounds__(SEL_WARPS * 32) select_rows_kernel(
    const float *logits, long long rows, int nb, int topk, float topp, uint8_t *__restrict__ mask,
    int32_t *kv_idx, int32_t *__restrict__ kv_cnt) {
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * SEL_WARPS + (threadIdx.x >> 5);
    if (row >= rows) return;
    const float *lg = logits + (size_t)row * nb;
    const uint32_t lt_mask = (1u << lane) - 1u;

    float x[E];
#pragma unroll
    for (int r = 0; r < E; ++r) {
        const int e = r * 32 + lane;
        x[r] = e < nb ? lg[e] : -INFINITY;
    }
    __syncwarp();  // every lane has read the row before any lane writes kv_idx (same buffer)
    float mx = -INFINITY;
#pragma unroll
    for (int r = 0; r < E; ++r) mx = fmaxf(mx, x[r]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float z = 0.f;
#pragma unroll
    for (int r = 0; r < E; ++r) z += (r * 32 + lane) < nb ? expf(x[r] - mx) : 0.f;
    z = warp_sum(z);
    float p[E];
    uint32_t key[E];
#pragma unroll
    for (int r = 0; r < E; ++r) {
        const bool ok = (r * 32 + lane) < nb;
        p[r] = ok ? expf(x[r] - mx) / z : 0.f;
        key[r] = ok ? ord_bits(x[r]) : 0u;
    }

    // ---- top-p cut m
    int m;
    uint32_t T = 0u;  // final threshold and the number of tied blocks taken at it
    int take = 0;
    bool decided = false;
    if (!(topp > 0.f)) {
        m = 0;
    } else if (topp >= 1.f) {
        m = nb;
    } else {
        float tot = 0.f;
#pragma unroll
        for (int r = 0; r < E; ++r) tot += p[r];
        if (!(warp_sum(tot) >= topp)) {
            m = nb;
        } else {
            uint32_t tp = 0u;
#pragma unroll 1
            for (int bit = 31; bit >= 0; --bit) {
                const uint32_t cand = tp | (1u << bit);
                float ms = 0.f;
#pragma unroll
                for (int r = 0; r < E; ++r) ms += key[r] >= cand ? p[r] : 0.f;
                if (warp_sum(ms) >= topp) tp = cand;
            }
            int above = 0;
            float base = 0.f;
#pragma unroll
            for (int r = 0; r < E; ++r) {
                above += key[r] > tp ? 1 : 0;
                base += key[r] > tp ? p[r] : 0.f;
            }
            above = warp_isum(above);
            base = warp_sum(base);
            // blocks tied at tp, in id order, until the mass reaches p (at least one)
            int ntie = 0, need = 0;
            float run = base;
#pragma unroll
            for (int r = 0; r < E; ++r) {
                const bool tied = key[r] == tp;
                const uint32_t bal = __ballot_sync(0xffffffffu, tied);
                float v = tied ? p[r] : 0.f;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, v, o);
                    if (lane >= o) v += y;
                }
                need += __popc(__ballot_sync(0xffffffffu, tied && run + v < topp));
                run += __shfl_sync(0xffffffffu, v, 31);
                ntie += __popc(bal);
            }
            const int ntake = min(need + 1, ntie);
            m = above + ntake;
            T = tp;
            take = ntake;
            decided = true;  // valid if the union is the top-p set
        }
    }
    const int kk = min(topk, nb);
    const int keep = max(kk, m);

    if (!(decided && keep == m)) {
        if (keep >= nb) {
            T = 0u;  // every valid block (valid keys are > 0, padding is 0)
            take = 0;
        } else if (keep <= 0) {
            T = 0xFFFFFFFFu;
            take = 0;
        } else {
            // the keep-th largest key by count
            uint32_t tk = 0u;
#pragma unroll 1
            for (int bit = 31; bit >= 0; --bit) {
                const uint32_t cand = tk | (1u << bit);
                int c = 0;
#pragma unroll
                for (int r = 0; r < E; ++r) c += key[r] >= cand ? 1 : 0;
                if (warp_isum(c) >= keep) tk = cand;
            }
            int above = 0;
#pragma unroll
            for (int r = 0; r < E; ++r) above += key[r] > tk ? 1 : 0;
            T = tk;
            take = keep - warp_isum(above);
        }
    }

    // ---- mark, write the mask row and the ascending id list
    uint8_t *mrow = mask + (size_t)row * nb;
    int32_t *idx = kv_idx + (size_t)row * nb;
    int tied_before = 0, pos = 0;
#pragma unroll
    for (int r = 0; r < E; ++r) {
        const int e = r * 32 + lane;
        const bool tied = key[r] == T;
        const uint32_t tb = __ballot_sync(0xffffffffu, tied);
        const bool kept = e < nb && (key[r] > T || (tied && tied_before + __popc(tb & lt_mask) < take));
        tied_before += __popc(tb);
        const uint32_t kb = __ballot_sync(0xffffffffu, kept);
        if (e < nb) mrow[e] = kept ? 1 : 0;
        if (kept) idx[pos + __popc(kb & lt_mask)] = e;
        pos += __popc(kb);
    }
    if (lane == 0) kv_cnt[row] = pos;
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
    if (nb <= 384) return launch_select_rows<12>(logits, rows, nb, topk, topp, mask, kv_idx, kv_cnt, st);
    if (nb <= 512) return launch_select_rows<16>(logits, rows, nb, topk, topp, mask, kv_idx, kv_cnt, st);
    if (nb <= 640) return launch_select_rows<20>(logits, rows, nb, topk, topp, mask, kv_idx, kv_cnt, st);
    if (nb <= 768) return launch_select_rows<24>(logits, rows, nb, topk, topp, mask, kv_idx, kv_cnt, st);
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
