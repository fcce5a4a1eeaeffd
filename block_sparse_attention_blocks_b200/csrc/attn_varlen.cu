// Attention over clusters of variable size: the kernel behind the semantic-aware permutation of
// Sparse VideoGen2 (section 2.A: tokens reordered so that each cluster is contiguous; section
// 2.C: a kernel for dynamic block sizes, sparse loads of the selected key/value tokens and dense
// compute on contiguous query tokens).
//
// Q, K and V arrive already permuted (each cluster a contiguous range of rows of its head).  A
// work unit is a query tile: up to 128 consecutive rows of one query cluster.  Its key list is
// the list of its cluster: key tiles of up to 128 consecutive permuted rows, each given by its
// first row and its number of valid keys, covering exactly the keys of the selected key
// clusters.  Keys of a tile past its valid count (they belong to the next cluster) are masked;
// query rows past the tile's count are computed but not stored.  The output row of permuted
// query row s is written at its original position perm_q[s], which undoes the permutation.
// The query tensor may have another length than the keys (Nq rows against N keys), e.g. a set
// of gathered query rows attending to every key.  In the split form each query "cluster" is one
// run of the keys and the kernel writes, per cluster, the fp32 output of that run with its
// log2-sum-exp, for the caller to combine.
//
// The pipeline and the roles are those of the block-sparse kernel (one TMA producer lane, one
// MMA issuer lane, a tensor-memory allocator warp and four softmax warps; S = Q K^T and O += P V
// on the tcgen05 tensor cores with fp32 accumulators in tensor memory, P kept in tensor memory;
// online softmax with a reference max from the first key tile and P allowed up to 2^30).  What
// differs is where tiles start: a TMA row coordinate may be any row, so tiles start inside
// clusters rather than on block boundaries.
#include "bsa_internal.h"
#include "softmax.cuh"

namespace bsa {

struct VarlenParams {
    const int2 *units;      // [BH * units_per_head] {q_row0, q_rows << 16 | cluster}; q_rows = 0: no work
    const int32_t *tiles;   // [BH * Cq, tstride] key tiles (k_row0 << 7) | (valid - 1)
    const int32_t *tcnt;    // [BH * Cq] key tiles in each query cluster's list
    const int32_t *perm_q;  // [BH, Nq] original position of each permuted query row
    __nv_bfloat16 *o;       // [BH, Nq, D] in the original order
    float *part_o;          // or, when set: [Cq, BH, Nq, D] fp32 O / l per query cluster ...
    float *part_lse;        // ... and [Cq, BH, Nq] its log2-sum-exp (log2 l + the row's max)
    long long BH;
    int N, Nq, Cq, tstride, units_per_head;  // N keys, Nq query (and output) rows
    long long nunits;       // BH * units_per_head
    float scale_log2;       // softmax scale * log2(e)
    unsigned long long wait_ns;
    unsigned int *next_unit;  // work counter in the caller's workspace, zero at launch
};

template <int D>
struct VarlenCfg {
    static constexpr int ROWS = 128;                  // query rows and key rows per tile
    static constexpr int CHUNKS = D / 64;             // 64-column (128-byte) swizzle chunks
    static constexpr int CHUNK = ROWS * 128;          // bytes per chunk of a tile
    static constexpr int TILE_BYTES = CHUNKS * CHUNK;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + TILE_BYTES;
    static constexpr int OFF_V = OFF_K + TILE_BYTES;
    static constexpr int OFF_BAR = OFF_V + TILE_BYTES;
    static constexpr int OFF_UNITS = OFF_BAR + 8 * 24;
    static constexpr int SMEM = OFF_UNITS + 16 + 1024;
    static constexpr uint32_t TMEM_COLS = 256;
    static constexpr uint32_t COL_S = 0, COL_O = 128;
    static constexpr int LAUNCH_REGS = 128;
    static constexpr int REGS_LO = 56;
    static constexpr int REGS_HI = 200;
    static_assert(REGS_LO + REGS_HI == 2 * LAUNCH_REGS, "register split must match the launch");
};

enum { V_QF, V_QE, V_KF, V_KE, V_VF, V_VE, V_SF, V_PF, V_OD, V_ED, V_FIN,
       V_UF0, V_UF1, V_UF2, V_UF3, V_UE0, V_UE1, V_UE2, V_UE3, V_COUNT };
constexpr int VUNIT_RING = 4;

struct VarUnit {
    int bh, row0, rows, cluster;
};

__device__ __forceinline__ VarUnit decode_unit(const VarlenParams &p, long long u) {
    const int2 e = p.units[u];
    VarUnit r;
    r.bh = (int)(u / p.units_per_head);
    r.rows = (int)((uint32_t)e.y >> 16);
    r.cluster = e.y & 0xFFFF;
    r.row0 = e.x;
    if (r.rows > 0 &&
        (r.rows > 128 || r.row0 < 0 || r.row0 > p.Nq - r.rows || r.cluster >= p.Cq)) {
        atomicOr(&g_bsa_device_error, BSA_DEVERR_BOUNDS);
        r.rows = 0;  // a malformed unit is skipped by every role alike
    }
    return r;
}

__device__ __forceinline__ int unit_tiles(const VarlenParams &p, const VarUnit &w) {
    if (w.rows == 0) return -1;
    const int c = p.tcnt[(size_t)w.bh * p.Cq + w.cluster];
    return min(max(c, 0), p.tstride);
}

// First row and valid count of a key tile entry, clamped into the head.
__device__ __forceinline__ void decode_tile(int32_t e, int N, int &row0, int &valid) {
    row0 = (int)((uint32_t)e >> 7);
    valid = (e & 127) + 1;
    if (row0 >= N) {
        atomicOr(&g_bsa_device_error, BSA_DEVERR_BOUNDS);
        row0 = N - 1;
    }
    valid = min(valid, N - row0);
}

template <int D>
__global__ void __launch_bounds__(256, 2)
    attn_varlen_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const VarlenParams prm) {
    using C = VarlenCfg<D>;
    constexpr int BS = C::ROWS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::OFF_BAR + 8 * V_COUNT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_BAR + 8 * V_COUNT + 4);
    volatile int *s_unit = reinterpret_cast<volatile int *>(smem + C::OFF_UNITS);
    static_assert(8 * V_COUNT + 8 <= C::OFF_UNITS - C::OFF_BAR, "barrier area overflow");

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t sQ = smem_u32(smem + C::OFF_Q);
    const uint32_t sK = smem_u32(smem + C::OFF_K);
    const uint32_t sV = smem_u32(smem + C::OFF_V);
    auto bar = [&](int b) { return smem_u32(&bars[b]); };

    if (threadIdx.x == 0) {
        mbar_init(bar(V_QF), 1);
        mbar_init(bar(V_QE), 1);
        mbar_init(bar(V_KF), 1);
        mbar_init(bar(V_KE), 1);
        mbar_init(bar(V_VF), 1);
        mbar_init(bar(V_VE), 1);
        mbar_init(bar(V_SF), 1);
        mbar_init(bar(V_PF), 128);
        mbar_init(bar(V_OD), 1);
        mbar_init(bar(V_ED), 128);
        mbar_init(bar(V_FIN), 1);
        for (int r = 0; r < VUNIT_RING; ++r) {
            mbar_init(bar(V_UF0 + r), 1);
            mbar_init(bar(V_UE0 + r), 5);
        }
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    if (warp == 2) {
        tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
        tmem_relinquish();
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
        uint32_t nq = 0, nk = 0, nv = 0;
        bool ok = true;
        for (uint32_t kth = 0; ok; ++kth) {
            const int slot = kth & (VUNIT_RING - 1);
            if (kth >= VUNIT_RING &&
                !(ok = warp_wait(bar(V_UE0 + slot), ((kth / VUNIT_RING) - 1) & 1, wns, abort_flag, 0x54, kth)))
                break;
            long long u = 0;
            if (lane == 0) {
                u = (long long)atomicAdd(prm.next_unit, 1u);
                s_unit[slot] = u < prm.nunits ? (int)u : -1;
                mbar_arrive(bar(V_UF0 + slot));
            }
            u = __shfl_sync(0xffffffffu, u, 0);
            if (u >= prm.nunits) break;
            const VarUnit w = decode_unit(prm, u);
            const int cnt = unit_tiles(prm, w);
            if (cnt <= 0) continue;
            const int32_t *list = prm.tiles + ((size_t)w.bh * prm.Cq + w.cluster) * prm.tstride;
            if (nq > 0 && !(ok = warp_wait(bar(V_QE), (nq - 1) & 1, wns, abort_flag, 0x51, (uint32_t)u)))
                break;
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(V_QF), C::TILE_BYTES);
#pragma unroll
                for (int c = 0; c < C::CHUNKS; ++c)
                    tma_load_3d(sQ + c * C::CHUNK, &tmQ, bar(V_QF), c * 64, w.row0, w.bh);
            }
            ++nq;
            int32_t en = list[0];
            for (int t = 0; t < cnt; ++t) {
                const uint32_t where = ((uint32_t)t << 16) | ((uint32_t)u & 0xFFFFu);
                int k0, valid;
                decode_tile(en, prm.N, k0, valid);
                if (t + 1 < cnt) en = list[t + 1];  // next entry, fetched early
                if (nk > 0 && !(ok = warp_wait(bar(V_KE), (nk - 1) & 1, wns, abort_flag, 0x52, where)))
                    break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar(V_KF), C::TILE_BYTES);
#pragma unroll
                    for (int c = 0; c < C::CHUNKS; ++c)
                        tma_load_3d(sK + c * C::CHUNK, &tmK, bar(V_KF), c * 64, k0, w.bh);
                }
                ++nk;
                if (nv > 0 && !(ok = warp_wait(bar(V_VE), (nv - 1) & 1, wns, abort_flag, 0x53, where)))
                    break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar(V_VF), C::TILE_BYTES);
#pragma unroll
                    for (int c = 0; c < C::CHUNKS; ++c)
                        tma_load_3d(sV + c * C::CHUNK, &tmV, bar(V_VF), c * 64, k0, w.bh);
                }
                ++nv;
            }
        }
        if (!ok && lane == 0) {  // let every copy that was started land before the CTA leaves
            if (nq) drain_wait(bar(V_QF), (nq - 1) & 1, wns, 0x61);
            if (nk) drain_wait(bar(V_KF), (nk - 1) & 1, wns, 0x62);
            if (nv) drain_wait(bar(V_VF), (nv - 1) & 1, wns, 0x63);
        }
    } else if (warp == 1) {
        regs_dec<C::REGS_LO>();
        // ---------------------------------------------------------------- MMA issuer
        constexpr uint32_t IDESC_S = idesc_bf16_f32(128, BS, 0, 0);
        constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, 0, 1);
        uint32_t nq = 0, nk = 0, nv = 0, np = 0, ned = 0, units_done = 0;
        bool ok = true;
        const uint64_t dQ = smem_desc_sw128(sQ, 16, 1024);
        const uint64_t dK = smem_desc_sw128(sK, 16, 1024);
        const uint64_t dV = smem_desc_sw128(sV, C::CHUNK, 1024);
        for (uint32_t kth = 0; ok; ++kth) {
            const int slot = kth & (VUNIT_RING - 1);
            if (!(ok = warp_wait(bar(V_UF0 + slot), (kth / VUNIT_RING) & 1, wns, abort_flag, 0x67, kth)))
                break;
            const long long u = s_unit[slot];
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(V_UE0 + slot));
            if (u < 0) break;
            const VarUnit w = decode_unit(prm, u);
            const int cnt = unit_tiles(prm, w);
            if (cnt <= 0) continue;
            if (!(ok = warp_wait(bar(V_QF), nq & 1, wns, abort_flag, 0x71, (uint32_t)u))) break;
            ++nq;
            for (int t = 0; t < cnt; ++t) {
                const uint32_t where = ((uint32_t)t << 16) | ((uint32_t)u & 0xFFFFu);
                if (!(ok = warp_wait(bar(V_KF), nk & 1, wns, abort_flag, 0x72, where))) break;
                ++nk;
                tc_fence_after();
                if (lane == 0) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t oq = (uint64_t)(((kk >> 2) * C::CHUNK + (kk & 3) * 32) >> 4);
                        mma_ss(tS, dQ + oq, dK + oq, IDESC_S, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(bar(V_SF));
                    mma_commit(bar(V_KE));
                    if (t == cnt - 1) mma_commit(bar(V_QE));
                }
                __syncwarp();
                if (!(ok = warp_wait(bar(V_PF), np & 1, wns, abort_flag, 0x74, where))) break;
                ++np;
                if (t == 0 && units_done > 0) {
                    // O is about to be overwritten: the previous epilogue must have read it
                    if (!(ok = warp_wait(bar(V_ED), ned & 1, wns, abort_flag, 0x75, (uint32_t)u))) break;
                    ++ned;
                }
                if (!(ok = warp_wait(bar(V_VF), nv & 1, wns, abort_flag, 0x76, where))) break;
                ++nv;
                tc_fence_after();
                if (lane == 0) {
#pragma unroll
                    for (int kk = 0; kk < BS / 16; ++kk)
                        mma_ts(tO, tS + kk * 8, dV + (uint64_t)((kk * 2048) >> 4), IDESC_PV,
                               (t > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(bar(V_VE));
                    mma_commit(bar(V_OD));
                }
                __syncwarp();
            }
            ++units_done;
        }
        if (lane == 0) {
            mma_commit(bar(V_FIN));
            drain_wait(bar(V_FIN), 0, wns, 0x64);
        }
    } else if (warp < 4) {
        regs_dec<C::REGS_LO>();
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
            const int slot = kth & (VUNIT_RING - 1);
            if (!(ok = warp_wait(bar(V_UF0 + slot), (kth / VUNIT_RING) & 1, wns, abort_flag, 0x73, kth)))
                break;
            const long long u = s_unit[slot];
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(V_UE0 + slot));
            if (u < 0) break;
            const VarUnit w = decode_unit(prm, u);
            const int cnt = unit_tiles(prm, w);
            if (cnt < 0) continue;  // no query rows in this slot
            const bool row_ok = r < w.rows;
            int orig = 0;
            if (row_ok) {
                orig = prm.perm_q[(size_t)w.bh * prm.Nq + w.row0 + r];
                if (orig < 0 || orig >= prm.Nq) {
                    atomicOr(&g_bsa_device_error, BSA_DEVERR_BOUNDS);
                    orig = 0;
                }
            }
            __nv_bfloat16 *orow = prm.o ? prm.o + ((size_t)w.bh * prm.Nq + orig) * D : nullptr;
            const size_t prow = ((size_t)w.cluster * prm.BH + w.bh) * prm.Nq + orig;
            if (cnt == 0) {  // the cluster selected nothing: zeros
                if (row_ok && prm.part_o) {
                    float4 *dst = reinterpret_cast<float4 *>(prm.part_o + prow * D);
#pragma unroll 4
                    for (int c = 0; c < D / 4; ++c) dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
                    prm.part_lse[prow] = -INFINITY;
                } else if (row_ok) {
                    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                    for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4 *>(orow)[c] = z;
                }
                continue;
            }
            const int32_t *list = prm.tiles + ((size_t)w.bh * prm.Cq + w.cluster) * prm.tstride;
            float m_ref = 0.f;
            float l = 0.f;
            int32_t en = list[0];
            for (int t = 0; t < cnt; ++t) {
                int k0, valid;
                decode_tile(en, prm.N, k0, valid);
                if (t + 1 < cnt) en = list[t + 1];
                if (!(ok = warp_wait(bar(V_SF), ns & 1, wns, abort_flag, 0x81, ((uint32_t)t << 16) | ((uint32_t)u & 0xFFFFu)))) break;
                ++ns;
                tc_fence_after();
                uint32_t s[BS];
                tmem_ld_cols<BS>(tSr, s);
                if (valid < BS) {  // keys of the next cluster (warp-uniform branch)
#pragma unroll
                    for (int e = 0; e < BS; ++e)
                        if (e >= valid) s[e] = __float_as_uint(-INFINITY);
                }
                if (t == 0) m_ref = row_max<BS>(s) * sl2;
                uint32_t pk[BS / 2];
                float xpoly;
                float ts = exp_row<BS>(s, sl2, m_ref, pk, xpoly);
                if (__any_sync(0xffffffffu, !(ts < kMaxP) || xpoly > kMaxLog2P)) {
                    tmem_ld_cols<BS>(tSr, s);
                    if (valid < BS) {
#pragma unroll
                        for (int e = 0; e < BS; ++e)
                            if (e >= valid) s[e] = __float_as_uint(-INFINITY);
                    }
                    const float m_new = fmaxf(m_ref, row_max<BS>(s) * sl2);
                    const float alpha = ex2(m_ref - m_new);
                    if (t > 0) {
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
                    ts = exp_row<BS>(s, sl2, m_ref, pk, xpoly);
                }
                l += ts;
#pragma unroll
                for (int c = 0; c < BS / 64; ++c)
                    tmem_st32(tSr + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[c * 32]));
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(V_PF));
            }
            if (!ok) break;
            npv += cnt;
            if (!(ok = warp_wait(bar(V_OD), (npv - 1) & 1, wns, abort_flag, 0x82, (uint32_t)u))) break;
            tc_fence_after();
            const float inv_l = 1.f / l;
            if (prm.part_o) {  // fp32 partial output of this key list and its log2-sum-exp
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t v[32];
                    tmem_ld32(tOr + c * 32, v);
                    if (row_ok) {
                        float4 *dst = reinterpret_cast<float4 *>(prm.part_o + prow * D + c * 32);
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            dst[q] = make_float4(__uint_as_float(v[4 * q]) * inv_l, __uint_as_float(v[4 * q + 1]) * inv_l,
                                                 __uint_as_float(v[4 * q + 2]) * inv_l, __uint_as_float(v[4 * q + 3]) * inv_l);
                    }
                }
                if (row_ok) prm.part_lse[prow] = m_ref + log2f(l);
                tc_fence_before();
                mbar_arrive(bar(V_ED));
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
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                }
            }
            tc_fence_before();
            mbar_arrive(bar(V_ED));
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 2) tmem_dealloc(tbase, C::TMEM_COLS);
}

template <int D>
static cudaError_t launch_varlen_t(const CUtensorMap &tq, const CUtensorMap &tk,
                                   const CUtensorMap &tv, const VarlenParams &p, int num_sms,
                                   cudaStream_t st) {
    using C = VarlenCfg<D>;
    const int smem = C::SMEM > 80 * 1024 ? C::SMEM : 80 * 1024;
    cudaError_t e = cudaFuncSetAttribute(attn_varlen_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    // setmaxnreg.inc only succeeds within the registers the CTA was launched with
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, attn_varlen_kernel<D>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != C::LAUNCH_REGS) return cudaErrorInvalidConfiguration;
    long long grid = 2LL * num_sms;
    if (grid > p.nunits) grid = p.nunits;
    if (grid <= 0) return cudaSuccess;
    e = cudaMemsetAsync(p.next_unit, 0, sizeof(unsigned int), st);
    if (e != cudaSuccess) return e;
    attn_varlen_kernel<D><<<(unsigned)grid, 256, smem, st>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

cudaError_t attn_varlen_fwd(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                            const int2 *units, int units_per_head, const int32_t *tiles,
                            const int32_t *tcnt, int tstride, const int32_t *perm_q, void *o,
                            long long BH, int N, int Nq, int Cq, int d, float scale,
                            unsigned long long wait_ns, int num_sms, unsigned int *workspace,
                            cudaStream_t st, float *part_o, float *part_lse) {
    VarlenParams p;
    p.part_o = part_o;
    p.part_lse = part_lse;
    p.BH = BH;
    p.units_per_head = units_per_head;
    p.tiles = tiles;
    p.tcnt = tcnt;
    p.perm_q = perm_q;
    p.o = reinterpret_cast<__nv_bfloat16 *>(o);
    p.N = N;
    p.Nq = Nq;
    p.Cq = Cq;
    p.tstride = tstride;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.wait_ns = wait_ns;
    p.next_unit = workspace;
    p.units = units;
    p.nunits = BH * units_per_head;
    if (d == 128) return launch_varlen_t<128>(tq, tk, tv, p, num_sms, st);
    if (d == 64) return launch_varlen_t<64>(tq, tk, tv, p, num_sms, st);
    return cudaErrorInvalidValue;
}

}  // namespace bsa
