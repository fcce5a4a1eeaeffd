// Hybrid top-k + top-p block selection.
//
// SpargeAttention2 ("Top-kとTop-pの限界を解剖する", "ハイブリッドマスキングと蒸留微調整"): each query
// block keeps the union of its k most probable key blocks and the top-p prefix of key blocks.
// Sparse VideoGen2 (section 2.B): the estimated block scores are sorted and blocks are taken in
// order until the cumulative score reaches p.  The problem statement fixes the estimate as
// softmax(Qp Kp^T * scale) over pooled blocks.
//
// Two launches:
//   1. block_scores_tc_kernel: L = scale * Qp Kp^T per (b, h) on the tensor cores at fp32
//      accuracy, written into the kv_idx buffer (same size: nb x nb 32-bit words per head),
//      which doubles as staging.
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
// L = scale * Qp Kp^T on the tensor cores.  Each fp32 operand x is split exactly into three bf16
// parts, x = h + m + l: h keeps the sign, exponent and top 7 fraction bits of x (the low 16 bits
// cleared), m the same of x - h, and l = x - h - m, which has at most 8 significant bits left
// (each difference is exact in fp32).  The dot product is the sum of the six part products whose
// weight is at least 2^-16 relative (l.h, m.m, h.l, m.h, h.m, h.h, smallest first), each a
// tcgen05.mma.kind::f16 accumulating in one fp32 tensor-memory tile.  The products of bf16 parts
// are exact in fp32, so the result differs from an fp32 FFMA dot product by accumulation
// rounding of the same order (fp32, not bf16 or TF32: the mask decision needs the scores to
// ~1e-6).  One CTA computes one 128 x 128 tile (128 query blocks x 128 key
// blocks of one head) in 64-channel chunks: 256 threads load a chunk of both fp32 row tiles
// (coalesced), split it into the six bf16 tiles in shared memory (the 128-byte swizzled K-major
// layout the MMA descriptor reads), and thread 0 issues the 6 x 4 MMAs of the chunk; the finished tile goes
// through shared memory to coalesced row stores.  96 KB of shared memory, two CTAs per SM, so one
// CTA's loads and stores overlap the other's MMAs.
constexpr int TC_ROWS = 128;

struct ScoresTcCfg {
    static constexpr int PART = TC_ROWS * 128;        // one bf16 tile: 128 rows x 64 channels
    static constexpr int OFF_Q = 0;                   // 3 parts of the query-block chunk
    static constexpr int OFF_K = 3 * PART;            // 3 parts of the key-block chunk
    static constexpr int OFF_BAR = 6 * PART;          // mbarrier, TMEM address
    static constexpr int OUT_LD = TC_ROWS + 4;        // padded fp32 row of the output staging
    static_assert(TC_ROWS * OUT_LD * 4 <= 6 * PART, "output staging must fit in the operands");
    static constexpr int SMEM = OFF_BAR + 16 + 1024;  // + alignment slack
};

// 8-byte shared-memory store through a shared-window address
__device__ __forceinline__ void st_shared_v2(uint32_t addr, uint32_t a, uint32_t b) {
    asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}

// byte offset of element (row, col) of a 128-row x 64-column bf16 tile in the 128-byte swizzled
// layout: the 16-byte unit u = col / 8 of a row is stored at unit u ^ (row % 8)
__device__ __forceinline__ uint32_t sw128_offset(int row, int col) {
    return (uint32_t)(row * 128 + ((((col >> 3) ^ row) & 7) << 4));
}

template <int D>
__global__ void __launch_bounds__(256, 2) block_scores_tc_kernel(const float *__restrict__ qp,
                                                                 const float *__restrict__ kp,
                                                                 float *__restrict__ logits,
                                                                 int nb, float scale,
                                                                 unsigned long long wait_ns) {
    using C = ScoresTcCfg;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::OFF_BAR + 8);
    const int bh = blockIdx.z, i0 = blockIdx.y * TC_ROWS, j0 = blockIdx.x * TC_ROWS;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    grid_dependency_wait();  // the pooled tiles of a programmatically dependent launch are complete

    if (tid == 0) {
        mbar_init(smem_u32(bar), 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_holder), 128);
        tmem_relinquish();
    }
    int never = 0;
    bool done = true;
    uint32_t tmem = 0;
    constexpr uint32_t IDESC = idesc_bf16_f32(128, 128, 0, 0);

#pragma unroll 1
    for (int dc = 0; dc < D / 64; ++dc) {
        // 128 rows x 64 channels of each operand: float4 f = v * 256 + tid is row f / 16,
        // channels 4 (f % 16) .. + 3, so 16 lanes read one row's 256 contiguous bytes; every
        // load of the chunk is issued before any store
        float4 xq[8], xk[8];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            const int f = v * 256 + tid, row = f >> 4, ch = dc * 64 + (f & 15) * 4;
            const int gi = i0 + row, gj = j0 + row;
            xq[v] = gi < nb ? *reinterpret_cast<const float4 *>(qp + ((size_t)bh * nb + gi) * D + ch)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
            xk[v] = gj < nb ? *reinterpret_cast<const float4 *>(kp + ((size_t)bh * nb + gj) * D + ch)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (dc > 0) {
            // the previous chunk's MMAs must have read the parts before they are overwritten
            done = done && mbar_wait(smem_u32(bar), (dc - 1) & 1, wait_ns, (volatile int *)&never, 0x51, 0);
        }
        // 4 channels -> 8 bytes of each bf16 part, half of a swizzled 16-byte unit
        auto stash = [&](const float4 (&x)[8], uint32_t base) {
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const int f = v * 256 + tid, row = f >> 4, col = (f & 15) * 4;
                const float xv[4] = {x[v].x, x[v].y, x[v].z, x[v].w};
                uint32_t hb[4], mb[4], lb[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    hb[q] = __float_as_uint(xv[q]) & 0xFFFF0000u;
                    const float rm = xv[q] - __uint_as_float(hb[q]);  // exact
                    mb[q] = __float_as_uint(rm) & 0xFFFF0000u;
                    lb[q] = __float_as_uint(rm - __uint_as_float(mb[q]));  // exact, low half zero
                }
                // the high halves of two words are the bf16 parts, the lower channel in the low half
                const uint32_t off = smem_u32(smem) + base + sw128_offset(row, col) + (col & 4) * 2;
                st_shared_v2(off, __byte_perm(hb[0], hb[1], 0x7632), __byte_perm(hb[2], hb[3], 0x7632));
                st_shared_v2(off + C::PART, __byte_perm(mb[0], mb[1], 0x7632), __byte_perm(mb[2], mb[3], 0x7632));
                st_shared_v2(off + 2 * C::PART, __byte_perm(lb[0], lb[1], 0x7632), __byte_perm(lb[2], lb[3], 0x7632));
            }
        };
        stash(xq, C::OFF_Q);
        stash(xk, C::OFF_K);
        // the tensor core reads shared memory through the async proxy
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        tmem = *tmem_holder;
        if (tid == 0) {
            const uint64_t dq = smem_desc_sw128(smem_u32(smem + C::OFF_Q), 16, 1024);
            const uint64_t dk = smem_desc_sw128(smem_u32(smem + C::OFF_K), 16, 1024);
            // (query part, key part): l.h, m.m, h.l, m.h, h.m, h.h (0 = h, 1 = m, 2 = l)
            const int pa[6] = {2, 1, 0, 1, 0, 0}, pb[6] = {0, 1, 2, 0, 1, 0};
#pragma unroll
            for (int p = 0; p < 6; ++p) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)  // 16 channels = 32 bytes of the swizzled row
                    mma_ss(tmem, dq + (uint64_t)((pa[p] * C::PART + kk * 32) >> 4),
                           dk + (uint64_t)((pb[p] * C::PART + kk * 32) >> 4), IDESC,
                           (dc > 0 || p > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(smem_u32(bar));
        }
    }
    done = done && mbar_wait(smem_u32(bar), (D / 64 - 1) & 1, wait_ns, (volatile int *)&never, 0x51, 0);
    tc_fence_after();
    // TMEM -> registers -> padded shared tile (the operand tiles are no longer read)
    float *outs = reinterpret_cast<float *>(smem);
    {
        const int lr = (warp & 3) * 32 + lane;  // TMEM lane = query row of the tile
        const int cb = (warp >> 2) * 64;        // this warp's 64 columns
        uint32_t v[32];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            tmem_ld32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + cb + c * 32, v);
#pragma unroll
            for (int e = 0; e < 32; e += 4)
                *reinterpret_cast<float4 *>(&outs[lr * C::OUT_LD + cb + c * 32 + e]) =
                    make_float4(__uint_as_float(v[e]) * scale, __uint_as_float(v[e + 1]) * scale,
                                __uint_as_float(v[e + 2]) * scale, __uint_as_float(v[e + 3]) * scale);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 128);
    if (!done) return;  // a wait ran out: the device error word says so; store nothing
    // coalesced rows: warp w stores rows w, w + 8, ...
    const int ncol = min(TC_ROWS, nb - j0);
    for (int rr = warp; rr < TC_ROWS; rr += 8) {
        const int i = i0 + rr;
        if (i >= nb) break;
        float *dst = logits + ((size_t)bh * nb + i) * nb + j0;
#pragma unroll
        for (int c = lane; c < TC_ROWS; c += 32)
            if (c < ncol) dst[c] = outs[rr * C::OUT_LD + c];
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

// The two thresholds by one bitwise search (bit 31 down to 0) over EE blocks per lane:
//   tp = the largest key T with fixed-point mass  sum{P : key >= T} >= pfix,
//   tk = the largest key T with  #{key >= T} >= kk.
// Each search keeps the invariant that its current threshold satisfies its condition, and stops
// as soon as the answer is known:
//   top-k: once exactly kk keys are >= tk, the answer is the least of them;
//   top-p: once the mass of the keys above m (m the least key >= tp) falls short of pfix, the
//          answer is m (checked every fourth bit, and at the end).
// A search that is not wanted (do_p / do_k false) is skipped.
template <int EE>
__device__ __forceinline__ void search_thresholds(const uint32_t (&key)[EE], const uint32_t (&pf)[EE],
                                                  uint32_t pfix, int kk, bool do_p, bool do_k,
                                                  uint32_t &tp, uint32_t &tk) {
    tp = 0u;
    tk = 0u;
    bool dp = !do_p, dk = !do_k;
#pragma unroll 1
    for (int bit = 31; bit >= 0 && !(dp && dk); --bit) {
        if (!dp) {
            const uint32_t cp = tp | (1u << bit);
            uint32_t ms = 0u;
#pragma unroll
            for (int r = 0; r < EE; ++r) ms += key[r] >= cp ? pf[r] : 0u;
            if (__reduce_add_sync(0xffffffffu, ms) >= pfix) tp = cp;
            if ((bit & 3) == 0) {
                uint32_t lo = 0xFFFFFFFFu;
#pragma unroll
                for (int r = 0; r < EE; ++r) lo = key[r] >= tp ? min(lo, key[r]) : lo;
                const uint32_t m = __reduce_min_sync(0xffffffffu, lo);
                uint32_t above = 0u;
#pragma unroll
                for (int r = 0; r < EE; ++r) above += key[r] > m ? pf[r] : 0u;
                if (__reduce_add_sync(0xffffffffu, above) < pfix) {
                    tp = m;
                    dp = true;
                }
            }
        }
        if (!dk) {
            const uint32_t ck = tk | (1u << bit);
            uint32_t c = 0u;
#pragma unroll
            for (int r = 0; r < EE; ++r) c += key[r] >= ck ? 1u : 0u;
            const int cc = (int)__reduce_add_sync(0xffffffffu, c);
            if (cc >= kk) {
                tk = ck;
                if (cc == kk) {
                    uint32_t lo = 0xFFFFFFFFu;
#pragma unroll
                    for (int r = 0; r < EE; ++r) lo = key[r] >= tk ? min(lo, key[r]) : lo;
                    tk = __reduce_min_sync(0xffffffffu, lo);
                    dk = true;
                }
            }
        }
    }
}

// One warp per query-block row; element e = r*32 + lane (coalesced, index order is r-major).
//
// The ranked order is (score descending, block id ascending); key[e] is the score mapped to an
// order-preserving uint32, so "rank < R" is "key > T, or key == T and among the first few
// tied ids" for the right threshold T.  Both sets the pages define are prefixes of this order:
//   top-p: T_p = the largest key value whose mass  sum{P_e : key_e >= T_p} >= p;  then the
//          tied blocks at T_p are taken in id order until the mass reaches p;  m = their count
//          plus the blocks above T_p.
//   top-k: T_k = the largest key value with  #{e : key_e >= T_k} >= k.
// The top-p threshold is found by a bitwise search: its first 11 bits over every block held in
// registers, then the blocks whose keys share those bits (a bucket of at most 64 in practice) are
// compacted in id order into shared memory and the remaining 21 bits are decided over the bucket
// alone, with the mass above the bucket added once (a crowded bucket falls back to the search
// over every block).  The top-k threshold, needed only when the top-p prefix is shorter than k,
// is found by the register search, which stops as soon as exactly k keys clear the candidate.  Masses are summed in fixed
// point (round(P * 2^26) in 32 bits), so every warp sum is exact, independent of the order of
// addition, and one redux.sync instruction; the fixed-point rounding (<= 2^-27 per block, under
// 8e-6 over a row) stays below the 1e-5 resolution of the cut.  The union is the longer prefix,
// |keep| = max(min(k, nb), m).
template <int E>
__global__ void __launch_bounds__(SEL_WARPS * 32, E <= 20 ? 8 : 4) select_rows_kernel(
    const float *logits, long long rows, int nb, int topk, float topp, uint8_t *__restrict__ mask,
    int32_t *kv_idx, int32_t *__restrict__ kv_cnt) {
    __shared__ uint32_t s_cand[SEL_WARPS][2 * 64];
    grid_dependency_wait();  // the scores of a programmatically dependent launch are complete
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * SEL_WARPS + (threadIdx.x >> 5);
    if (row >= rows) return;
    const float *lg = logits + (size_t)row * nb;
    const uint32_t lt_mask = (1u << lane) - 1u;
    constexpr float kFix = 67108864.0f;  // 2^26

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
    // per block: order key, exp(x - max) on the SFU (relative error ~2^-22, under a tenth of the
    // 1e-5 resolution of the cut), then the fixed-point probability round(P * 2^26) (sums over
    // <= 1024 blocks stay below 2^32 and differ from the exact sum by < 8e-6)
    uint32_t key[E], pf[E];
    float z = 0.f;
#pragma unroll
    for (int r = 0; r < E; ++r) {
        const bool ok = (r * 32 + lane) < nb;
        key[r] = ok ? ord_bits(x[r]) : 0u;
        x[r] = ok ? ex2((x[r] - mx) * 1.4426950408889634f) : 0.f;  // SFU exp; see the fixed point
        z += x[r];
    }
    z = warp_sum(z);
    const float to_fix = kFix / z;
    uint32_t tsum = 0u;
#pragma unroll
    for (int r = 0; r < E; ++r) {
        pf[r] = __float2uint_rn(x[r] * to_fix);
        tsum += pf[r];
    }
    const uint32_t total = __reduce_add_sync(0xffffffffu, tsum);
    // a positive p needs at least one block (the least count whose cumulative P reaches p), also
    // when p is below the fixed-point resolution
    const uint32_t pfix = max(__float2uint_rn(fminf(fmaxf(topp, 0.f), 1.f) * kFix), topp > 0.f ? 1u : 0u);
    const int kk = topk < nb ? topk : nb;
    const bool want_p = topp > 0.f && topp < 1.f && total >= pfix;
    const bool all_kept = topp >= 1.f || (topp > 0.f && !want_p) || kk >= nb;

    // ---- the top-p threshold first; the top-k one only if the top-p prefix is shorter than k
    uint32_t tp = 0u, tk = 0u;
    int m, ntake = 0, ntie_tp = -1;  // blocks tied at tp, when known
    bool counted = false;
    if (!(topp > 0.f)) {
        m = 0;
        counted = true;
    } else if (!want_p || all_kept) {
        m = nb;  // p >= 1, the fixed-point total falls short of p, or k >= nb keeps everything
        counted = true;
    } else {
        // The first PRE bits of the threshold over every block in registers.  The answer then
        // lies in the bucket [tp, tp | LOW]: the blocks in it are compacted (in id order) into
        // shared memory, the mass above the bucket is summed once, and the remaining bits are
        // decided over the bucket alone; mass{key >= c} = mass above + mass{bucket key >= c}.
        constexpr int PRE = 11, CAP = 64;
        constexpr uint32_t LOW = (1u << (32 - PRE)) - 1u;
#pragma unroll 1
        for (int bit = 31; bit >= 32 - PRE; --bit) {
            const uint32_t cp = tp | (1u << bit);
            uint32_t ms = 0u;
#pragma unroll
            for (int r = 0; r < E; ++r) ms += key[r] >= cp ? pf[r] : 0u;
            if (__reduce_add_sync(0xffffffffu, ms) >= pfix) tp = cp;
        }
        const uint32_t hi = tp | LOW;
        uint32_t am = 0u, ac = 0u;
        int n = 0;
        uint32_t *ck = s_cand[threadIdx.x >> 5], *cm = s_cand[threadIdx.x >> 5] + CAP;
#pragma unroll
        for (int r = 0; r < E; ++r) {
            const bool inb = key[r] >= tp && key[r] <= hi;
            const uint32_t bal = __ballot_sync(0xffffffffu, inb);
            const int pos = n + __popc(bal & lt_mask);
            if (inb && pos < CAP) {
                ck[pos] = key[r];
                cm[pos] = pf[r];
            }
            n += __popc(bal);
            am += key[r] > hi ? pf[r] : 0u;
            ac += key[r] > hi ? 1u : 0u;
        }
        if (n <= CAP) {
            const uint32_t above_m = __reduce_add_sync(0xffffffffu, am);
            const int above_c = (int)__reduce_add_sync(0xffffffffu, ac);
            __syncwarp();
            // position j of the bucket: slot j / 32 of lane j % 32 (id order = position order)
            const uint32_t k0 = lane < n ? ck[lane] : 0u, m0 = lane < n ? cm[lane] : 0u;
            const uint32_t k1 = lane + 32 < n ? ck[lane + 32] : 0u, m1 = lane + 32 < n ? cm[lane + 32] : 0u;
            __syncwarp();
#pragma unroll 1
            for (int bit = 31 - PRE; bit >= 0; --bit) {
                const uint32_t cp = tp | (1u << bit);
                const uint32_t ms = (k0 >= cp ? m0 : 0u) + (k1 >= cp ? m1 : 0u);
                if (above_m + __reduce_add_sync(0xffffffffu, ms) >= pfix) tp = cp;
            }
            // m: the blocks above tp, then the blocks tied at tp in id order until the mass
            // reaches p (ties can only be bucket members)
            uint32_t run = above_m + __reduce_add_sync(0xffffffffu, (k0 > tp ? m0 : 0u) + (k1 > tp ? m1 : 0u));
            const int gt = above_c + (int)__reduce_add_sync(0xffffffffu, (k0 > tp ? 1u : 0u) + (k1 > tp ? 1u : 0u));
            int need = 0, ntie = 0;
#pragma unroll
            for (int sidx = 0; sidx < 2; ++sidx) {
                const bool tied = (sidx == 0 ? k0 : k1) == tp && (sidx == 0 ? lane : lane + 32) < n;
                const uint32_t bal = __ballot_sync(0xffffffffu, tied);
                if (bal) {
                    uint32_t v = tied ? (sidx == 0 ? m0 : m1) : 0u;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const uint32_t y = __shfl_up_sync(0xffffffffu, v, o);
                        if (lane >= o) v += y;
                    }
                    need += __popc(__ballot_sync(0xffffffffu, tied && run + v < pfix));
                    run += __shfl_sync(0xffffffffu, v, 31);
                    ntie += __popc(bal);
                }
            }
            ntake = min(need + 1, ntie);
            ntie_tp = ntie;
            m = gt + ntake;
            counted = true;
        } else {
            // a crowded bucket: finish the search over the registers
            search_thresholds<E>(key, pf, pfix, kk, true, false, tp, tk);
        }
    }
    if (!counted) {
        uint32_t as = 0u, ac = 0u;
#pragma unroll
        for (int r = 0; r < E; ++r) {
            const bool gt = key[r] > tp;
            as += gt ? pf[r] : 0u;
            ac += gt ? 1u : 0u;
        }
        uint32_t run = __reduce_add_sync(0xffffffffu, as);
        const int above = (int)__reduce_add_sync(0xffffffffu, ac);
        int need = 0, ntie = 0;
#pragma unroll
        for (int r = 0; r < E; ++r) {
            const bool tied = key[r] == tp;
            const uint32_t bal = __ballot_sync(0xffffffffu, tied);
            if (bal) {  // warp-uniform; usually a single block
                uint32_t v = tied ? pf[r] : 0u;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t y = __shfl_up_sync(0xffffffffu, v, o);
                    if (lane >= o) v += y;
                }
                need += __popc(__ballot_sync(0xffffffffu, tied && run + v < pfix));
                run += __shfl_sync(0xffffffffu, v, 31);
                ntie += __popc(bal);
            }
        }
        ntake = min(need + 1, ntie);
        m = above + ntake;
    }
    const int keep = max(kk, m);

    // ---- the kept prefix: key > T, plus the first `take` blocks tied at T
    uint32_t T;
    int take;
    if (keep >= nb) {
        T = 0u;  // every valid block (valid keys are > 0, padding is 0)
        take = 0;
    } else if (keep <= 0) {
        T = 0xFFFFFFFFu;
        take = 0;
    } else if (want_p && m >= kk) {
        T = tp;
        take = ntake;
    } else {
        uint32_t unused;
        search_thresholds<E>(key, pf, pfix, kk, false, true, unused, tk);
        uint32_t above = 0u;
#pragma unroll
        for (int r = 0; r < E; ++r) above += key[r] > tk ? 1u : 0u;
        T = tk;
        take = kk - (int)__reduce_add_sync(0xffffffffu, above);
    }

    // ---- mark, write the mask row and the ascending id list
    uint8_t *mrow = mask + (size_t)row * nb;
    int32_t *idx = kv_idx + (size_t)row * nb;
    int tied_before = 0, pos = 0;
    // the usual case: every block tied at the threshold is taken (typically the one cut block)
    const bool all_tied = T == tp && ntie_tp >= 0 && take >= ntie_tp && take > 0;
    if (all_tied) {
#pragma unroll
        for (int r = 0; r < E; ++r) {
            const int e = r * 32 + lane;
            const bool kept = e < nb && key[r] >= T;
            const uint32_t kb = __ballot_sync(0xffffffffu, kept);
            if (e < nb) mrow[e] = kept ? 1 : 0;
            if (kept) idx[pos + __popc(kb & lt_mask)] = e;
            pos += __popc(kb);
        }
    } else {
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
    }
    if (lane == 0) kv_cnt[row] = pos;
}


template <int E>
static cudaError_t launch_select_rows(const float *logits, long long rows, int nb, int topk,
                                      float topp, uint8_t *mask, int32_t *kv_idx, int32_t *kv_cnt,
                                      cudaStream_t st) {
    const long long grid = (rows + SEL_WARPS - 1) / SEL_WARPS;
    return launch_dependent(select_rows_kernel<E>, dim3((unsigned)grid), dim3(SEL_WARPS * 32), 0,
                            st, logits, rows, nb, topk, topp, mask, kv_idx, kv_cnt);
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

template <int D>
static cudaError_t launch_scores_tc(const float *qp, const float *kp, float *logits, long long BH,
                                    int nb, float scale, unsigned long long wait_ns, cudaStream_t st) {
    using C = ScoresTcCfg;
    cudaError_t e = cudaFuncSetAttribute(block_scores_tc_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    const int t = (nb + TC_ROWS - 1) / TC_ROWS;
    dim3 grid((unsigned)t, (unsigned)t, (unsigned)BH);
    return launch_dependent(block_scores_tc_kernel<D>, grid, dim3(256), C::SMEM, st, qp, kp, logits,
                            nb, scale, wait_ns);
}

cudaError_t block_scores_tc(const float *qp, const float *kp, float *logits, long long BH, int nb,
                            int d, float scale, unsigned long long wait_ns, cudaStream_t st) {
    if (BH == 0 || nb == 0) return cudaSuccess;
    if (d == 128) return launch_scores_tc<128>(qp, kp, logits, BH, nb, scale, wait_ns, st);
    if (d == 64) return launch_scores_tc<64>(qp, kp, logits, BH, nb, scale, wait_ns, st);
    return cudaErrorInvalidValue;
}

}  // namespace bsa
