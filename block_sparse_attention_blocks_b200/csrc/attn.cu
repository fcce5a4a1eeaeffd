// Attention forward on the tensor cores over per-unit lists of key tiles: the block-sparse
// attention over a compacted per-query-block key-block list and its dense control (every key
// block), and attention over clusters of variable size (the kernel behind the semantic-aware
// permutation of Sparse VideoGen2, section 2.A and 2.C), in one kernel template whose tile
// addressing is a policy (BlockWalk, TileWalk).
//
// Block lists: for each query block i and each kept key block j, S = Q_i K_j^T is a dense 128 x BS x d
// contraction and O_i += P V_j a dense 128 x d x BS one, so both run on the tcgen05 tensor cores
// with fp32 accumulators in tensor memory; softmax is online as in FlashAttention (a reference
// max per row from the first kept block, P allowed to reach 2^30 before the reference moves and
// O and the row sum are rescaled).  The key-block walk is what Sparse
// VideoGen2 (section 2.C) describes: dense compute on a contiguous query tile, sparse loads of
// the kept key/value blocks.  Keys at or beyond N are masked; query rows at or beyond N (and,
// for BS = 64, rows of the next query block inside the 128-row tile) are computed but not
// stored.  A query block with an empty list writes zeros.
//
// Variable-length tiles: Q, K and V arrive already permuted (each cluster a contiguous range of
// rows of its head).  A work unit is a query tile, up to 128 consecutive rows of one query
// cluster; its key list is its cluster's list of key tiles of up to 128 consecutive permuted rows,
// each given by its first row and its number of valid keys (keys past that count belong to the
// next cluster and are masked).  A TMA row coordinate may be any row, so tiles start inside
// clusters rather than on block boundaries.  The output row of permuted query row s is written at
// its original position perm_q[s], which undoes the permutation.  The query tensor may have
// another length than the keys (Nq rows against N keys).  In the split form each query
// "cluster" is one run of the keys and the kernel writes, per cluster, the fp32 output of that run
// with its log2-sum-exp, for the caller to combine.
//
// CTA roles (256 threads, two CTAs per SM, persistent; query blocks are claimed dynamically
// from a counter in the caller's workspace, in head-major order):
//   warp 0 lane 0  TMA producer: Q tile once per unit, then K and V per key tile
//   warp 1 lane 0  MMA issuer:   S = Q K_j^T (SS form), O += P V_j (P read from tensor memory)
//   warp 2         tensor-memory allocator (256 columns: S/P at 0, O at 128)
//   warps 4..7     softmax: one thread per query row; reads S, writes P (bf16) over S, rescales
//                  O, and runs the epilogue O / l -> bf16 -> global
// Per CTA the chain S -> softmax -> PV is serial; the second CTA on the SM fills the tensor
// pipe while this one is in softmax.
#include "bsa_internal.h"
#include "softmax.cuh"

namespace bsa {

// Parameters common to the tile-addressing policies.
struct AttnCommon {
    float scale_log2;        // softmax scale * log2(e)
    unsigned long long wait_ns;
    unsigned int *progress;  // optional host-mapped [grid, 8] stage words for diagnosis
    unsigned int *next_unit; // work counter in the caller's workspace, zero at launch
};

// One work unit as the roles see it: its head, its query tile (first row, rows to store; 0
// rows: no work), its key-tile count and list, and its query cluster.
struct AttnUnit {
    int bh, q0, rows, cnt, cluster;
    const int32_t *list;
};
struct KeyTile {
    int k0, valid;  // first key row, keys in the tile
};
struct AttnOut {
    __nv_bfloat16 *row;  // bf16 output row
    float *part, *lse;   // or, in the split form, the fp32 row and its log2-sum-exp
};

// Block lists: unit u = query block i of head bh (head-major), key tile j = key block j.
template <int D, int BS>
struct BlockWalk {
    static constexpr int kD = D, kBS = BS;
    static constexpr bool kSplit = false, kGroups = false;
    const int32_t *kv_idx;  // [units, nbk] ascending key-block ids, or null for dense
    const int32_t *kv_cnt;  // [units], or null for dense
    __nv_bfloat16 *o;       // [BH, N, D]
    int N, nbq, nbk;
    long long nunits;       // BH * nbq

    __device__ __forceinline__ AttnUnit unit(long long u) const {
        AttnUnit w;
        w.bh = (int)(u / nbq);
        w.q0 = (int)(u - (long long)w.bh * nbq) * BS;
        w.rows = min(BS, N - w.q0);
        w.cnt = kv_idx ? min(max(kv_cnt[u], 0), nbk) : nbk;
        w.cluster = 0;
        w.list = kv_idx ? kv_idx + (size_t)u * nbk : nullptr;
        return w;
    }
    __device__ __forceinline__ int32_t entry(const AttnUnit &w, int t) const {
        return w.list ? w.list[t] : t;
    }
    // an id outside [0, nbk) is clamped (and flagged once, by the producer)
    __device__ __forceinline__ KeyTile key(int32_t j, bool flag) const {
        if (j < 0 || j >= nbk) {
            if (flag) atomicOr(&g_bsa_device_error, BSA_DEVERR_BOUNDS);
            j = j < 0 ? 0 : nbk - 1;
        }
        return KeyTile{j * BS, min(BS, N - j * BS)};
    }
    __device__ __forceinline__ AttnOut out(const AttnUnit &w, int r, bool row_ok) const {
        return AttnOut{o + ((size_t)w.bh * N + (row_ok ? w.q0 + r : 0)) * D, nullptr, nullptr};
    }
};

// Variable-length tiles: unit u = entry u of the query-tile table (units_per_head per head),
// key tile = entry (k_row0 << 7) | (valid - 1) of its cluster's list.
template <int D>
struct TileWalk {
    static constexpr int kD = D;
    static constexpr bool kSplit = true, kGroups = false;
    const int2 *units;      // [BH * units_per_head] {q_row0, q_rows << 16 | cluster}; q_rows = 0: none
    const int32_t *tiles;   // [BH * Cq, tstride] key tiles (k_row0 << 7) | (valid - 1)
    const int32_t *tcnt;    // [BH * Cq] key tiles in each query cluster's list
    const int32_t *perm_q;  // [BH, Nq] original position of each permuted query row
    __nv_bfloat16 *o;       // [BH, Nq, D] in the original order
    float *part_o;          // or, when set: [Cq, BH, Nq, D] fp32 O / l per query cluster ...
    float *part_lse;        // ... and [Cq, BH, Nq] its log2-sum-exp (log2 l + the row's max)
    long long BH, nunits;   // nunits = BH * units_per_head
    int N, Nq, Cq, tstride, units_per_head;  // N keys, Nq query (and output) rows

    __device__ __forceinline__ AttnUnit unit(long long u) const {
        const int2 e = units[u];
        AttnUnit w;
        w.bh = (int)(u / units_per_head);
        w.rows = (int)((uint32_t)e.y >> 16);
        w.cluster = e.y & 0xFFFF;
        w.q0 = e.x;
        if (w.rows > 0 && (w.rows > 128 || w.q0 < 0 || w.q0 > Nq - w.rows || w.cluster >= Cq)) {
            atomicOr(&g_bsa_device_error, BSA_DEVERR_BOUNDS);
            w.rows = 0;  // a malformed unit is skipped by every role alike
        }
        const size_t row = (size_t)w.bh * Cq + (w.rows ? w.cluster : 0);
        w.cnt = w.rows ? min(max(tcnt[row], 0), tstride) : 0;
        w.list = tiles + row * tstride;
        return w;
    }
    __device__ __forceinline__ int32_t entry(const AttnUnit &w, int t) const { return w.list[t]; }
    // first row and valid count of a key tile entry, clamped into the head
    __device__ __forceinline__ KeyTile key(int32_t e, bool flag) const {
        KeyTile k;
        k.k0 = (int)((uint32_t)e >> 7);
        k.valid = (e & 127) + 1;
        if (k.k0 >= N) {
            if (flag) atomicOr(&g_bsa_device_error, BSA_DEVERR_BOUNDS);
            k.k0 = N - 1;
        }
        k.valid = min(k.valid, N - k.k0);
        return k;
    }
    __device__ __forceinline__ AttnOut out(const AttnUnit &w, int r, bool row_ok) const {
        int orig = 0;
        if (row_ok) {
            orig = perm_q[(size_t)w.bh * Nq + w.q0 + r];
            if (orig < 0 || orig >= Nq) {
                atomicOr(&g_bsa_device_error, BSA_DEVERR_BOUNDS);
                orig = 0;
            }
        }
        const size_t prow = ((size_t)w.cluster * BH + w.bh) * Nq + orig;
        return AttnOut{o ? o + ((size_t)w.bh * Nq + orig) * D : nullptr,
                       part_o ? part_o + prow * D : nullptr, part_lse ? part_lse + prow : nullptr};
    }
};

// Many short independent sequences (W tokens each, stored one after another: Ntot rows in all)
// packed into 128-row tiles: unit u = rows [u P W, u P W + P W) with P = 128 / W sequences, one
// key tile over the same rows, and row r of the tile attends only to the keys of its own
// sequence (a block-diagonal mask in the softmax).
template <int D>
struct GroupWalk {
    static constexpr int kD = D;
    static constexpr bool kSplit = false, kGroups = true;
    __nv_bfloat16 *o;  // [Ntot, D]
    long long nunits;  // ceil(Ntot / per_tile)
    int Ntot, W, per_tile;  // rows, tokens per sequence, rows per tile (P W)

    __device__ __forceinline__ AttnUnit unit(long long u) const {
        AttnUnit w;
        w.bh = 0;
        w.q0 = (int)(u * per_tile);
        w.rows = min(per_tile, Ntot - w.q0);
        w.cnt = 1;
        w.cluster = 0;
        w.list = nullptr;
        return w;
    }
    __device__ __forceinline__ int32_t entry(const AttnUnit &w, int) const { return w.q0; }
    __device__ __forceinline__ KeyTile key(int32_t k0, bool) const {
        return KeyTile{k0, min(per_tile, Ntot - k0)};
    }
    __device__ __forceinline__ AttnOut out(const AttnUnit &w, int r, bool row_ok) const {
        return AttnOut{o + (size_t)(row_ok ? w.q0 + r : 0) * D, nullptr, nullptr};
    }
};

// Stage report for diagnosis: word (cta, role) = stage << 24 | step << 12 | unit (low bits).
__device__ __forceinline__ void report(unsigned int *progress, int role, int stage, int step,
                                       long long unit) {
    if (progress && (threadIdx.x & 31) == 0) {
        volatile unsigned int *w = progress + blockIdx.x * 8 + role;
        *w = ((unsigned)stage << 24) | (((unsigned)step & 0xFFFu) << 12) | ((unsigned)unit & 0xFFFu);
    }
}

template <int D, int BS>
struct AttnCfg {
    static constexpr int QROWS = 128;
    static constexpr int CHUNKS = D / 64;           // 64-column (128-byte) swizzle chunks
    static constexpr int Q_CHUNK = QROWS * 128;     // bytes per Q chunk
    static constexpr int KV_CHUNK = BS * 128;       // bytes per K or V chunk
    static constexpr int Q_BYTES = CHUNKS * Q_CHUNK;
    static constexpr int KV_BYTES = CHUNKS * KV_CHUNK;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + KV_BYTES;
    static constexpr int OFF_BAR = OFF_V + KV_BYTES;
    static constexpr int OFF_UNITS = OFF_BAR + 8 * 24;  // after the barriers and two words
    static constexpr int SMEM = OFF_UNITS + 16 + 1024;  // unit ring + slack for 1024-byte alignment
    static constexpr uint32_t TMEM_COLS = 256;
    static constexpr uint32_t COL_S = 0, COL_O = 128;
    // Register split per thread: the launch gives every thread LAUNCH_REGS (256 threads, two
    // CTAs per SM); warps 0-3 (producer, MMA issuer, allocator, idle) give registers to the
    // softmax warpgroup, which holds a whole S row.  REGS_LO + REGS_HI == 2 * LAUNCH_REGS.
    static constexpr int LAUNCH_REGS = 128;
    static constexpr int REGS_LO = 56;
    static constexpr int REGS_HI = 200;
    static_assert(REGS_LO + REGS_HI == 2 * LAUNCH_REGS, "register split must match the launch");
};

enum { B_QF, B_QE, B_KF, B_KE, B_VF, B_VE, B_SF, B_PF, B_OD, B_ED, B_FIN,
       B_UF0, B_UF1, B_UF2, B_UF3,   // unit ring slot published (producer -> consumers)
       B_UE0, B_UE1, B_UE2, B_UE3,   // unit ring slot consumed (MMA warp + 4 softmax warps)
       B_COUNT };
constexpr int UNIT_RING = 4;

template <int D, int BS, class Walk>
__global__ void __launch_bounds__(256, 2)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const Walk walk, const AttnCommon prm) {
    using C = AttnCfg<D, BS>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::OFF_BAR + 8 * B_COUNT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_BAR + 8 * B_COUNT + 4);
    volatile int *s_unit = reinterpret_cast<volatile int *>(smem + C::OFF_UNITS);
    static_assert(8 * B_COUNT + 8 <= C::OFF_UNITS - C::OFF_BAR, "barrier area overflow");

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t sQ = smem_u32(smem + C::OFF_Q);
    const uint32_t sK = smem_u32(smem + C::OFF_K);
    const uint32_t sV = smem_u32(smem + C::OFF_V);
    auto bar = [&](int b) { return smem_u32(&bars[b]); };

    if (threadIdx.x == 0) {
        mbar_init(bar(B_QF), 1);
        mbar_init(bar(B_QE), 1);
        mbar_init(bar(B_KF), 1);
        mbar_init(bar(B_KE), 1);
        mbar_init(bar(B_VF), 1);
        mbar_init(bar(B_VE), 1);
        mbar_init(bar(B_SF), 1);
        mbar_init(bar(B_PF), 128);
        mbar_init(bar(B_OD), 1);
        mbar_init(bar(B_ED), 128);
        mbar_init(bar(B_FIN), 1);
        for (int r = 0; r < UNIT_RING; ++r) {
            mbar_init(bar(B_UF0 + r), 1);
            mbar_init(bar(B_UE0 + r), 5);
        }
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    if (warp == 2) {
        report(prm.progress, 2, 0, 0, 0);
        tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
        tmem_relinquish();
        report(prm.progress, 2, 1, 0, 0);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_holder;
    const uint32_t tS = tbase + C::COL_S;
    const uint32_t tO = tbase + C::COL_O;
    const unsigned long long wns = prm.wait_ns;

    if (warp == 0) {
        regs_dec<C::REGS_LO>();
        // ---------------------------------------------------------------- TMA producer
        // The whole warp walks the loop (so it reaches the final CTA barrier converged); lane 0
        // arms the barriers and issues the copies.
        // Units (query blocks) are claimed from a global counter in head-major order, so all
        // CTAs stay within about one head of each other and that head's K/V stay in L2; each
        // claimed index is published to the MMA and softmax warps through a 4-slot ring.
        uint32_t nq = 0, nk = 0, nv = 0;
        bool ok = true;
        for (uint32_t kth = 0; ok; ++kth) {
            const int slot = kth & (UNIT_RING - 1);
            if (kth >= UNIT_RING &&
                !(ok = warp_wait(bar(B_UE0 + slot), ((kth / UNIT_RING) - 1) & 1, wns, abort_flag, 0x14, kth)))
                break;
            long long u = 0;
            if (lane == 0) {
                u = (long long)atomicAdd(prm.next_unit, 1u);
                s_unit[slot] = u < walk.nunits ? (int)u : -1;
                mbar_arrive(bar(B_UF0 + slot));
            }
            u = __shfl_sync(0xffffffffu, u, 0);
            if (u >= walk.nunits) break;
            const AttnUnit w = walk.unit(u);
            const int cnt = w.cnt;
            if (w.rows == 0 || cnt == 0) continue;
            report(prm.progress, 0, 1, 0, u);
            if (nq > 0 && !(ok = warp_wait(bar(B_QE), (nq - 1) & 1, wns, abort_flag, 0x11, (uint32_t)u)))
                break;
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(B_QF), C::Q_BYTES);
#pragma unroll
                for (int c = 0; c < C::CHUNKS; ++c)
                    tma_load_3d(sQ + c * C::Q_CHUNK, &tmQ, bar(B_QF), c * 64, w.q0, w.bh);
            }
            ++nq;
            int32_t en = walk.entry(w, 0);
            for (int t = 0; t < cnt; ++t) {
                const uint32_t where = ((uint32_t)t << 16) | ((uint32_t)u & 0xFFFFu);
                const KeyTile kt = walk.key(en, true);
                if (t + 1 < cnt) en = walk.entry(w, t + 1);  // next entry, fetched early
                report(prm.progress, 0, 2, t, u);
                if (nk > 0 && !(ok = warp_wait(bar(B_KE), (nk - 1) & 1, wns, abort_flag, 0x12, where)))
                    break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar(B_KF), C::KV_BYTES);
#pragma unroll
                    for (int c = 0; c < C::CHUNKS; ++c)
                        tma_load_3d(sK + c * C::KV_CHUNK, &tmK, bar(B_KF), c * 64, kt.k0, w.bh);
                }
                ++nk;
                report(prm.progress, 0, 3, t, u);
                if (nv > 0 && !(ok = warp_wait(bar(B_VE), (nv - 1) & 1, wns, abort_flag, 0x13, where)))
                    break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar(B_VF), C::KV_BYTES);
#pragma unroll
                    for (int c = 0; c < C::CHUNKS; ++c)
                        tma_load_3d(sV + c * C::KV_CHUNK, &tmV, bar(B_VF), c * 64, kt.k0, w.bh);
                }
                ++nv;
            }
        }
        report(prm.progress, 0, 4, 0, 0);
        if (!ok && lane == 0) {  // let every copy that was started land before the CTA leaves
            if (nq) drain_wait(bar(B_QF), (nq - 1) & 1, wns, 0x41);
            if (nk) drain_wait(bar(B_KF), (nk - 1) & 1, wns, 0x42);
            if (nv) drain_wait(bar(B_VF), (nv - 1) & 1, wns, 0x43);
        }
    } else if (warp == 1) {
        regs_dec<C::REGS_LO>();
        // ---------------------------------------------------------------- MMA issuer
        // Converged warp like the producer; lane 0 issues the MMAs and the commits (a commit
        // tracks the MMAs of the thread that issues it).
        constexpr uint32_t IDESC_S = idesc_bf16_f32(128, BS, 0, 0);
        constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, 0, 1);
        uint32_t nq = 0, nk = 0, nv = 0, np = 0, npv = 0, ned = 0, units_done = 0;
        bool ok = true;
        // Descriptors of the first 16-column step of each operand; step kk is reached by adding
        // its byte offset / 16 to the start-address field (shared addresses stay below 2^18, so
        // the 14-bit field never carries).  Few instructions per MMA matter: this warp shares
        // its issue slots with softmax warps.
        const uint64_t dQ = smem_desc_sw128(sQ, 16, 1024);
        const uint64_t dK = smem_desc_sw128(sK, 16, 1024);
        const uint64_t dV = smem_desc_sw128(sV, C::KV_CHUNK, 1024);
        for (uint32_t kth = 0; ok; ++kth) {
            const int slot = kth & (UNIT_RING - 1);
            if (!(ok = warp_wait(bar(B_UF0 + slot), (kth / UNIT_RING) & 1, wns, abort_flag, 0x27, kth)))
                break;
            const long long u = s_unit[slot];
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_UE0 + slot));
            if (u < 0) break;
            const AttnUnit w = walk.unit(u);
            const int cnt = w.cnt;
            if (w.rows == 0 || cnt == 0) continue;
            report(prm.progress, 1, 1, 0, u);
            if (!(ok = warp_wait(bar(B_QF), nq & 1, wns, abort_flag, 0x21, (uint32_t)u))) break;
            ++nq;
            for (int t = 0; t < cnt; ++t) {
                const uint32_t where = ((uint32_t)t << 16) | ((uint32_t)u & 0xFFFFu);
                report(prm.progress, 1, 2, t, u);
                if (!(ok = warp_wait(bar(B_KF), nk & 1, wns, abort_flag, 0x22, where))) break;
                report(prm.progress, 1, 3, t, u);
                ++nk;
                // S overwrites the columns the previous P V reads P from: tcgen05.mma operations
                // issued by one thread execute in issue order, so no wait is needed here.
                tc_fence_after();
                if (lane == 0) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        // K step kk: 32 bytes inside the 128-byte swizzled row, then the next chunk
                        const uint64_t oq = (uint64_t)(((kk >> 2) * C::Q_CHUNK + (kk & 3) * 32) >> 4);
                        const uint64_t ok = (uint64_t)(((kk >> 2) * C::KV_CHUNK + (kk & 3) * 32) >> 4);
                        mma_ss(tS, dQ + oq, dK + ok, IDESC_S, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(bar(B_SF));
                    mma_commit(bar(B_KE));
                    if (t == cnt - 1) mma_commit(bar(B_QE));
                }
                __syncwarp();
                report(prm.progress, 1, 4, t, u);
                if (!(ok = warp_wait(bar(B_PF), np & 1, wns, abort_flag, 0x24, where))) break;
                report(prm.progress, 1, 5, t, u);
                ++np;
                if (t == 0 && units_done > 0) {
                    // O is about to be overwritten: the previous epilogue must have read it
                    if (!(ok = warp_wait(bar(B_ED), ned & 1, wns, abort_flag, 0x25, (uint32_t)u))) break;
                    ++ned;
                }
                report(prm.progress, 1, 6, t, u);
                if (!(ok = warp_wait(bar(B_VF), nv & 1, wns, abort_flag, 0x26, where))) break;
                report(prm.progress, 1, 7, t, u);
                ++nv;
                tc_fence_after();
                if (lane == 0) {
#pragma unroll
                    for (int kk = 0; kk < BS / 16; ++kk) {
                        // 16 keys = 16 rows of 128 bytes
                        mma_ts(tO, tS + kk * 8, dV + (uint64_t)((kk * 2048) >> 4), IDESC_PV,
                               (t > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(bar(B_VE));
                    mma_commit(bar(B_OD));
                }
                __syncwarp();
                report(prm.progress, 1, 8, t, u);
                ++npv;
            }
            ++units_done;
        }
        // every MMA this warp issued must be complete before tensor memory is released
        report(prm.progress, 1, 9, 0, 0);
        if (lane == 0) {
            mma_commit(bar(B_FIN));
            drain_wait(bar(B_FIN), 0, wns, 0x44);
        }
        report(prm.progress, 1, 10, 0, 0);
    } else if (warp < 4) {
        regs_dec<C::REGS_LO>();  // allocator and idle warp: nothing to do until the end
    } else {
        regs_inc<C::REGS_HI>();
        // ---------------------------------------------------------------- softmax + epilogue
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;  // query row inside the tile == TMEM lane
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        const uint32_t tSr = tS + lane_off, tOr = tO + lane_off;
        const float sl2 = prm.scale_log2;
        uint32_t ns = 0, npv = 0;
        bool ok = true;
        for (uint32_t kth = 0; ok; ++kth) {
            const int slot = kth & (UNIT_RING - 1);
            if (!(ok = warp_wait(bar(B_UF0 + slot), (kth / UNIT_RING) & 1, wns, abort_flag, 0x33, kth)))
                break;
            const long long u = s_unit[slot];
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_UE0 + slot));
            if (u < 0) break;
            const AttnUnit w = walk.unit(u);
            if (w.rows == 0) continue;  // no query rows in this unit
            const int cnt = w.cnt;
            const bool row_ok = r < w.rows;
            const AttnOut out = walk.out(w, r, row_ok);
            if (cnt == 0) {  // nothing kept: zeros
                if (row_ok) {
                    if (Walk::kSplit && out.part) {
                        float4 *dst = reinterpret_cast<float4 *>(out.part);
#pragma unroll 4
                        for (int c = 0; c < D / 4; ++c) dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
                        *out.lse = -INFINITY;
                    } else {
                        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                        for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4 *>(out.row)[c] = z;
                    }
                }
                continue;
            }
            float m_ref = 0.f;        // reference max, log2 domain (set by the first block)
            float l = 0.f;            // running sum
            int32_t en = walk.entry(w, 0);
            for (int t = 0; t < cnt; ++t) {
                const KeyTile kt = walk.key(en, false);
                if (t + 1 < cnt) en = walk.entry(w, t + 1);  // next entry, fetched early
                const int valid = kt.valid;
                report(prm.progress, 4 + q4, 1, t, u);
                if (!(ok = warp_wait(bar(B_SF), ns & 1, wns, abort_flag, 0x31, ((uint32_t)t << 16) | ((uint32_t)u & 0xFFFFu)))) break;
                ++ns;
                tc_fence_after();
                // the whole S row of this thread: BS fp32 scores, one TMEM round trip
                uint32_t s[BS];
                tmem_ld_cols<BS>(tSr, s);
                // keys this row may see: [klo, khi) of the tile (its own sequence for packed
                // sequences; otherwise the tile's valid keys)
                int klo = 0, khi = valid;
                if constexpr (Walk::kGroups) {
                    if (row_ok) {
                        klo = (r / walk.W) * walk.W;
                        khi = min(klo + walk.W, valid);
                    }
                }
                auto mask_keys = [&](uint32_t (&sv)[BS]) {
                    if constexpr (Walk::kGroups) {
#pragma unroll
                        for (int e = 0; e < BS; ++e)
                            if (e < klo || e >= khi) sv[e] = __float_as_uint(-INFINITY);
                    } else if (valid < BS) {  // keys past the tile's valid count (warp-uniform)
#pragma unroll
                        for (int e = 0; e < BS; ++e)
                            if (e >= valid) sv[e] = __float_as_uint(-INFINITY);
                    }
                };
                mask_keys(s);
                // Reference max: the first block of a query block sets it from its own scores.
                // Later blocks reuse it while their P stays below 2^30 (bf16 and the fp32 sums
                // have room for that), which the block's row sum shows, so the row max is not
                // needed per block.  A block that overflows moves the reference to its max,
                // rescales O and l, and is exponentiated again.
                if (t == 0) m_ref = row_max<BS>(s) * sl2;
                uint32_t pk[BS / 2];
                float xpoly;
                float ts = exp_row<BS>(s, sl2, m_ref, pk, xpoly);
                // warp-uniform (tcgen05.ld/st are .sync.aligned); a NaN sum also overflows
                if (__any_sync(0xffffffffu, !(ts < kMaxP) || xpoly > kMaxLog2P)) {
                    // rare: S is read again from tensor memory (still intact: P is written below)
                    tmem_ld_cols<BS>(tSr, s);
                    mask_keys(s);
                    const float m_new = fmaxf(m_ref, row_max<BS>(s) * sl2);
                    const float alpha = ex2(m_ref - m_new);  // 1 for rows that keep theirs
                    if (t > 0) {
                        // the previous P V is complete: this S was issued after it, in order
#pragma unroll 1
                        for (int c = 0; c < D / 32; ++c) {
                            uint32_t v[32];
                            tmem_ld32(tOr + c * 32, v);
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
                            tmem_st32(tOr + c * 32, v);
                        }
                    }
                    l *= alpha;
                    m_ref = m_new;
                    ts = exp_row<BS>(s, sl2, m_ref, pk, xpoly);  // now every P <= 1
                }
                l += ts;
#pragma unroll
                for (int c = 0; c < BS / 64; ++c)
                    tmem_st32(tSr + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[c * 32]));
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(B_PF));
                report(prm.progress, 4 + q4, 3, t, u);
            }
            if (!ok) break;
            // epilogue: wait for the last P V of this query block
            npv += cnt;
            report(prm.progress, 4 + q4, 4, 0, u);
            if (!(ok = warp_wait(bar(B_OD), (npv - 1) & 1, wns, abort_flag, 0x32, (uint32_t)u))) break;
            tc_fence_after();
            const float inv_l = 1.f / l;
            if (Walk::kSplit && out.part) {  // fp32 output of this key run and its log2-sum-exp
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t v[32];
                    tmem_ld32(tOr + c * 32, v);
                    if (row_ok) {
                        float4 *dst = reinterpret_cast<float4 *>(out.part + c * 32);
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            dst[q] = make_float4(__uint_as_float(v[4 * q]) * inv_l, __uint_as_float(v[4 * q + 1]) * inv_l,
                                                 __uint_as_float(v[4 * q + 2]) * inv_l, __uint_as_float(v[4 * q + 3]) * inv_l);
                    }
                }
                if (row_ok) *out.lse = m_ref + log2f(l);
                tc_fence_before();
                mbar_arrive(bar(B_ED));
                continue;
            }
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t v[32];
                tmem_ld32(tOr + c * 32, v);
                if (row_ok) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 32; e += 2)
                        pk[e >> 1] = pack_bf16(__uint_as_float(v[e]) * inv_l,
                                               __uint_as_float(v[e + 1]) * inv_l);
                    uint4 *dst = reinterpret_cast<uint4 *>(out.row + c * 32);
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        dst[w] = make_uint4(pk[4 * w], pk[4 * w + 1], pk[4 * w + 2], pk[4 * w + 3]);
                }
            }
            tc_fence_before();
            mbar_arrive(bar(B_ED));
            report(prm.progress, 4 + q4, 5, 0, u);
        }
        report(prm.progress, 4 + q4, 6, 0, 0);
    }

    __syncwarp();
    if (warp == 2) report(prm.progress, 2, 2, 0, 0);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 2) {
        tmem_dealloc(tbase, C::TMEM_COLS);
        report(prm.progress, 2, 3, 0, 0);
    }
}

// ------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------
template <int D, int BS, class Walk>
static cudaError_t launch_attn_t(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                 const Walk &w, const AttnCommon &cm, int num_sms, cudaStream_t st) {
    using C = AttnCfg<D, BS>;
    auto *kern = attn_fwd_kernel<D, BS, Walk>;
    // at least 80 KB per CTA so that no more than two CTAs (2 x 256 TMEM columns) share an SM
    const int smem = C::SMEM > 80 * 1024 ? C::SMEM : 80 * 1024;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    // setmaxnreg.inc only succeeds within the registers the CTA was launched with: refuse to
    // launch a build whose per-thread count differs from the split's assumption.
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != C::LAUNCH_REGS) return cudaErrorInvalidConfiguration;
    long long grid = 2LL * num_sms;
    if (grid > w.nunits) grid = w.nunits;
    if (grid <= 0) return cudaSuccess;
    e = cudaMemsetAsync(cm.next_unit, 0, sizeof(unsigned int), st);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)grid, 256, smem, st>>>(tq, tk, tv, w, cm);
    return cudaGetLastError();
}

cudaError_t attn_fwd(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                     const int32_t *kv_idx, const int32_t *kv_cnt, void *o, long long BH, int N,
                     int d, int bs, float scale, unsigned long long wait_ns, int num_sms,
                     unsigned int *progress, unsigned int *workspace, cudaStream_t st) {
    AttnCommon cm;
    cm.scale_log2 = scale * 1.4426950408889634f;
    cm.wait_ns = wait_ns;
    cm.progress = progress;
    cm.next_unit = workspace;
    auto run = [&](auto walk) {
        using W = decltype(walk);
        walk.kv_idx = kv_idx;
        walk.kv_cnt = kv_cnt;
        walk.o = reinterpret_cast<__nv_bfloat16 *>(o);
        walk.N = N;
        walk.nbq = (N + bs - 1) / bs;
        walk.nbk = walk.nbq;
        walk.nunits = BH * walk.nbq;
        return launch_attn_t<W::kD, W::kBS, W>(tq, tk, tv, walk, cm, num_sms, st);
    };
    if (d == 128 && bs == 128) return run(BlockWalk<128, 128>{});
    if (d == 128 && bs == 64) return run(BlockWalk<128, 64>{});
    if (d == 64 && bs == 128) return run(BlockWalk<64, 128>{});
    if (d == 64 && bs == 64) return run(BlockWalk<64, 64>{});
    return cudaErrorInvalidValue;
}

cudaError_t attn_group_fwd(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                           void *o, long long Ntot, int W, int d, float scale,
                           unsigned long long wait_ns, int num_sms, unsigned int *workspace,
                           cudaStream_t st) {
    if (W < 1 || W > 128 || Ntot < 1 || Ntot > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
    AttnCommon cm;
    cm.scale_log2 = scale * 1.4426950408889634f;
    cm.wait_ns = wait_ns;
    cm.progress = nullptr;
    cm.next_unit = workspace;
    auto run = [&](auto walk) {
        using W_ = decltype(walk);
        walk.o = reinterpret_cast<__nv_bfloat16 *>(o);
        walk.Ntot = (int)Ntot;
        walk.W = W;
        walk.per_tile = (128 / W) * W;
        walk.nunits = (Ntot + walk.per_tile - 1) / walk.per_tile;
        return launch_attn_t<W_::kD, 128, W_>(tq, tk, tv, walk, cm, num_sms, st);
    };
    if (d == 128) return run(GroupWalk<128>{});
    if (d == 64) return run(GroupWalk<64>{});
    return cudaErrorInvalidValue;
}

cudaError_t attn_varlen_fwd(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                            const int2 *units, int units_per_head, const int32_t *tiles,
                            const int32_t *tcnt, int tstride, const int32_t *perm_q, void *o,
                            long long BH, int N, int Nq, int Cq, int d, float scale,
                            unsigned long long wait_ns, int num_sms, unsigned int *workspace,
                            cudaStream_t st, float *part_o, float *part_lse) {
    AttnCommon cm;
    cm.scale_log2 = scale * 1.4426950408889634f;
    cm.wait_ns = wait_ns;
    cm.progress = nullptr;
    cm.next_unit = workspace;
    auto run = [&](auto walk) {
        using W = decltype(walk);
        walk.units = units;
        walk.tiles = tiles;
        walk.tcnt = tcnt;
        walk.perm_q = perm_q;
        walk.o = reinterpret_cast<__nv_bfloat16 *>(o);
        walk.part_o = part_o;
        walk.part_lse = part_lse;
        walk.BH = BH;
        walk.nunits = BH * units_per_head;
        walk.N = N;
        walk.Nq = Nq;
        walk.Cq = Cq;
        walk.tstride = tstride;
        walk.units_per_head = units_per_head;
        return launch_attn_t<W::kD, 128, W>(tq, tk, tv, walk, cm, num_sms, st);
    };
    if (d == 128) return run(TileWalk<128>{});
    if (d == 64) return run(TileWalk<64>{});
    return cudaErrorInvalidValue;
}

}  // namespace bsa
