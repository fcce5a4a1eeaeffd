// Static block patterns: the mask and kept-block lists of Sparse-vDiT's head patterns (page
// "Sparse-vDiT：動画拡散トランスフォーマの高速化を可能にするスパースアテンションの解放",
// section 3: diagonal, multi-diagonal and vertical-stripe attention maps, fixed per layer and
// head, and skipped heads), at block granularity, in the layout the block-sparse attention kernel
// reads.  Per head h, patterns[h] = {flags, w, p, s}; key block j is kept for query block i when
// any enabled part holds:
//   flags & 1  |i - j| <= w                                      diagonal band
//   flags & 2  i - j within w of a multiple of p (p > 0)          diagonals every p blocks
//   flags & 4  j < s                                              vertical stripe, first s blocks
// flags == 0 keeps nothing (a skipped head: the attention writes zeros for it).
#include "bsa_internal.h"

namespace bsa {

constexpr int ST_WARPS = 4;

// One warp per (b, h, i) row: 32 key blocks per step, ballots compact the kept ids in order.
__global__ void __launch_bounds__(ST_WARPS * 32) static_mask_kernel(const int32_t *__restrict__ patterns,
                                                                   long long rows, int H, int nb,
                                                                   uint8_t *__restrict__ mask,
                                                                   int32_t *__restrict__ kv_idx,
                                                                   int32_t *__restrict__ kv_cnt) {
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * ST_WARPS + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int i = (int)(row % nb);
    const int h = (int)((row / nb) % H);
    const int flags = patterns[4 * h], w = patterns[4 * h + 1], p = patterns[4 * h + 2],
              s = patterns[4 * h + 3];
    const uint32_t lt_mask = (1u << lane) - 1u;
    uint8_t *mrow = mask + (size_t)row * nb;
    int32_t *idx = kv_idx + (size_t)row * nb;
    int pos = 0;
    for (int jb = 0; jb < nb; jb += 32) {
        const int j = jb + lane;
        const int diff = i - j;
        bool keep = false;
        if (flags & 1) keep = keep || (diff <= w && -diff <= w);
        if ((flags & 2) && p > 0) {
            const int r = ((diff % p) + p) % p;  // distance to the multiple of p below
            keep = keep || r <= w || p - r <= w;
        }
        if (flags & 4) keep = keep || j < s;
        keep = keep && j < nb;
        const uint32_t kb = __ballot_sync(0xffffffffu, keep);
        if (j < nb) mrow[j] = keep ? 1 : 0;
        if (keep) idx[pos + __popc(kb & lt_mask)] = j;
        pos += __popc(kb);
    }
    if (lane == 0) kv_cnt[row] = pos;
}

cudaError_t static_mask(const int32_t *patterns, long long BH, int H, int nb, uint8_t *mask,
                        int32_t *kv_idx, int32_t *kv_cnt, cudaStream_t st) {
    const long long rows = BH * nb;
    if (rows == 0) return cudaSuccess;
    const long long grid = (rows + ST_WARPS - 1) / ST_WARPS;
    static_mask_kernel<<<(unsigned)grid, ST_WARPS * 32, 0, st>>>(patterns, rows, H, nb, mask,
                                                                  kv_idx, kv_cnt);
    return cudaGetLastError();
}

}  // namespace bsa
