// SparsePR's probe-fitted residual correction of block-sparse attention (page "Partition the
// Support, Reconstruct the Residual: Training-Free Sparse Attention for Video Generation and
// World Models", abstract and summary section 3).  Per call and head, a few probe query rows are
// computed exactly; their residuals against the block-sparse output are fitted by an affine map
// of the sparse output, and that map corrects every row.
//
// Per head, with P the probe rows (m of them, chosen by the caller), O_s the block-sparse output
// and E the exact outputs of the probe rows:
//   X = [O_s[P], 1]  (m x (d + 1)),   R = E - O_s[P]  (m x d)
//   W = X^+ R, the minimum-norm least-squares map, and O = O_s + [O_s, 1] W for every row.
// At the full numerical rank this is the page's fit limited to the span of the residuals: the
// minimum-norm least-squares map of the residuals is already a combination of the rows of R.
//
// Steps (one stream, no host synchronisation):
//   1. O_s by the block-sparse attention kernel;
//   2. the probe rows of Q gathered into [BH, m, d]; their exact outputs by the attention kernel
//      over variable-length tiles in its split form: the keys of each head cut into S runs of
//      128-key tiles (enough units to fill the GPU), each run's fp32 output and log2-sum-exp
//      combined in fp64 (probe_merge_kernel);
//   3. [O_s[P] | R] in fp64; the Gram products tiled over CTAs; W by d / 32 CTAs per head in
//      fp64 (32 right-hand-side columns each): the normal equations of the smaller side,
//      Cholesky in shared memory with a ridge of 1e-12 times the mean diagonal (which keeps a
//      rank-deficient X solvable and approximates the pseudo-inverse's minimum-norm choice);
//   4. O += [O, 1] W in place on the bf16 output, on the tensor cores (W in two bf16 parts).
#include "bsa_internal.h"
#include "sparse_attn.h"

namespace bsa {

// Qpr[bh, i, :] = Q[bh, probes[bh, i], :]   (16-byte vectors)
__global__ void __launch_bounds__(256) gather_probe_rows_kernel(const uint4 *__restrict__ q,
                                                                const int32_t *__restrict__ probes,
                                                                uint4 *__restrict__ qpr,
                                                                long long BH, int N, int m,
                                                                int vec) {
    const long long total = BH * m * vec;
    for (long long x = (long long)blockIdx.x * blockDim.x + threadIdx.x; x < total;
         x += (long long)gridDim.x * blockDim.x) {
        const long long row = x / vec;  // bh * m + i
        const int c = (int)(x - row * vec);
        const long long bh = row / m;
        const int t = min(max(probes[row], 0), N - 1);
        qpr[x] = q[(bh * N + t) * vec + c];
    }
}

// E = the exact probe outputs, combined from the S key splits by their log2-sum-exp weights
// (fp64), and M [BH, m, 2 d] = [O_s[P] | E - O_s[P]] with O_s bf16 [BH, N, d].
// po [S, BH, m, d] fp32 and plse [S, BH, m] are the split outputs of the variable-length kernel.
// CTA of 256 threads = 256 / d rows at a time, thread = (row, column); a row's S weights are
// computed once into shared memory.
__global__ void __launch_bounds__(256) probe_merge_kernel(
    const __nv_bfloat16 *__restrict__ os, const float *__restrict__ po, const float *__restrict__ plse,
    const int32_t *__restrict__ probes, double *__restrict__ M, long long BH, int N, int m, int d, int S) {
    __shared__ double s_w[4][64];
    const long long rows = BH * m;
    const int per = 256 / d, rr = threadIdx.x / d, c = threadIdx.x % d;
    for (long long r0 = (long long)blockIdx.x * per; r0 < rows; r0 += (long long)gridDim.x * per) {
        const long long row = r0 + rr;  // bh * m + i
        const bool live = row < rows;
        float lmax = -INFINITY;
        if (live)
            for (int sp = 0; sp < S; ++sp) lmax = fmaxf(lmax, plse[sp * rows + row]);
        if (live && c < S) s_w[rr][c] = exp2((double)plse[c * rows + row] - (double)lmax);
        __syncthreads();
        if (live) {
            double num = 0.0, den = 0.0;
            for (int sp = 0; sp < S; ++sp) {
                const double w = s_w[rr][sp];
                num += w * (double)po[(sp * rows + row) * d + c];
                den += w;
            }
            const long long bh = row / m;
            const int t = min(max(probes[row], 0), N - 1);
            const double o = (double)__bfloat162float(os[(bh * N + t) * d + c]);
            M[row * 2 * d + c] = o;
            M[row * 2 * d + d + c] = num / den - o;
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------------------------------------
// the per-head fit W = X^+ R, X = [O_s[P], 1], fp64
// ------------------------------------------------------------------------------------------
// With m >= d + 1 probes (the usual case) W solves the normal equations
//   (X^T X + ridge) W = X^T R,  X^T X = [[O^T O, O^T 1], [1^T O, m]],  X^T R = [O^T R; 1^T R]
// (O = O_s[P]); the products O^T [O | R] and the column sums of [O | R] come from
// probe_gram_kernel, tiled over many CTAs.  With fewer probes the smaller side is solved:
// (X X^T + ridge) Y = R, W = X^T Y.  The ridge is 1e-12 times the mean diagonal.

// C [BH, d, 2 d] = O^T [O | R] over the m probe rows (only tiles on or below the diagonal of
// the O^T O block), sums [BH, 2 d] = column sums of [O | R].  CTA = one 64 x 64 tile of one
// head (blockIdx.x < tiles) or the sums (blockIdx.x == tiles); thread = 4 x 4 outputs, rows
// staged through shared memory 32 at a time.
__global__ void __launch_bounds__(256) probe_gram_kernel(const double *__restrict__ M,
                                                         double *__restrict__ C,
                                                         double *__restrict__ sums, int m, int d) {
    const long long bh = blockIdx.y;
    const int w2 = 2 * d;
    const double *Mh = M + bh * m * w2;
    const int tcols = w2 / 64, tiles = (d / 64) * tcols;
    if ((int)blockIdx.x == tiles) {
        for (int j = threadIdx.x; j < w2; j += blockDim.x) {
            double s = 0.0;
            for (int r = 0; r < m; ++r) s += Mh[(long long)r * w2 + j];
            sums[bh * w2 + j] = s;
        }
        return;
    }
    const int ti = blockIdx.x / tcols, tj = blockIdx.x % tcols;
    if (tj < d / 64 && tj > ti) return;  // above the diagonal of the symmetric block
    __shared__ double As[32][64];
    __shared__ double Bs[32][64];
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
    double acc[4][4] = {};
    for (int r0 = 0; r0 < m; r0 += 32) {
        for (int p = threadIdx.x; p < 32 * 64; p += 256) {
            const int rr = p >> 6, cc = p & 63;
            const bool in = r0 + rr < m;
            const double *row = Mh + (long long)(r0 + rr) * w2;
            As[rr][cc] = in ? row[ti * 64 + cc] : 0.0;
            Bs[rr][cc] = in ? row[tj * 64 + cc] : 0.0;
        }
        __syncthreads();
#pragma unroll 4
        for (int k = 0; k < 32; ++k) {
            const double2 a01 = *reinterpret_cast<const double2 *>(&As[k][ty * 4]);
            const double2 a23 = *reinterpret_cast<const double2 *>(&As[k][ty * 4 + 2]);
            const double2 b01 = *reinterpret_cast<const double2 *>(&Bs[k][tx * 4]);
            const double2 b23 = *reinterpret_cast<const double2 *>(&Bs[k][tx * 4 + 2]);
            const double av[4] = {a01.x, a01.y, a23.x, a23.y};
            const double bv[4] = {b01.x, b01.y, b23.x, b23.y};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fma(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }
    double *Ch = C + bh * d * w2;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) Ch[(long long)(ti * 64 + ty * 4 + i) * w2 + tj * 64 + tx * 4 + j] = acc[i][j];
}

constexpr int kSolveThreads = 512;
constexpr int kSolveCols = 32;  // right-hand-side columns per CTA

__device__ __forceinline__ int tri(int i) { return i * (i + 1) / 2; }  // packed lower-row start

__device__ __forceinline__ void tri_decode(int p, int &i, int &j) {  // p -> (i, j), j <= i
    i = (int)((sqrt(8.0 * (double)p + 1.0) - 1.0) * 0.5);
    while (tri(i + 1) <= p) ++i;
    while (tri(i) > p) --i;
    j = p - tri(i);
}

// CTA (column block cb, head bh): forms the k x k system (k = d + 1, or m when m <= d), factors
// it in shared memory (packed lower triangle; every column block factors its own copy) and
// solves for its 32 right-hand-side columns, then writes those columns of W: the first d rows
// as two bf16 parts [BH, 2 d, d] (W_hi; W - W_hi) and the offset row [BH, d] fp32.
__global__ void __launch_bounds__(kSolveThreads, 2)
    probe_solve_kernel(const double *__restrict__ M, const double *__restrict__ C,
                       const double *__restrict__ sums, __nv_bfloat16 *__restrict__ wparts,
                       float *__restrict__ woff, int m, int d, double eps) {
    extern __shared__ double sm_solve[];
    constexpr int NC = kSolveCols;
    const long long bh = blockIdx.y;
    const int c0 = blockIdx.x * NC;
    const int n = d + 1, w2 = 2 * d;
    const bool tall = m >= n;
    const int k = tall ? n : m;
    double *__restrict__ L = sm_solve;                 // packed lower triangle, tri(k) entries
    double *__restrict__ invd = sm_solve + tri(k);     // [k] reciprocals of the factor's diagonal
    double *__restrict__ Z = sm_solve + tri(k) + k;    // [k][NC] right-hand sides, then the solution
    __shared__ double s_red[kSolveThreads / 32];
    const int tid = threadIdx.x, nt = blockDim.x;
    const int warp = tid >> 5, lane = tid & 31, nw = nt >> 5;
    const double *Mh = M + bh * m * w2;

    // 1. the system
    if (tall) {
        const double *Ch = C + bh * d * w2;
        const double *sh = sums + bh * w2;
        for (int p = tid; p < tri(k); p += nt) {
            int i, j;
            tri_decode(p, i, j);
            L[p] = i < d ? Ch[(long long)i * w2 + j] : (j < d ? sh[j] : (double)m);
        }
        for (int p = tid; p < k * NC; p += nt) {
            const int i = p / NC, c = c0 + p % NC;
            Z[p] = i < d ? Ch[(long long)i * w2 + d + c] : sh[d + c];
        }
    } else {
        for (int p = tid; p < tri(k); p += nt) {
            int i, j;
            tri_decode(p, i, j);
            const double *xi = Mh + (long long)i * w2, *xj = Mh + (long long)j * w2;
            double sum = 1.0;  // the ones column
            for (int e = 0; e < d; ++e) sum = fma(xi[e], xj[e], sum);
            L[p] = sum;
        }
        for (int p = tid; p < k * NC; p += nt) Z[p] = Mh[(long long)(p / NC) * w2 + d + c0 + p % NC];
    }
    __syncthreads();
    // ridge: eps times the mean diagonal
    {
        double sum = 0.0;
        for (int i = tid; i < k; i += nt) sum += L[tri(i) + i];
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0) s_red[warp] = sum;
        __syncthreads();
        double tr = 0.0;
        for (int w = 0; w < nw; ++w) tr += s_red[w];
        __syncthreads();
        for (int i = tid; i < k; i += nt) L[tri(i) + i] += eps * tr / k;
    }
    __syncthreads();

    // 2. factor G = L L^T in 8-column panels (right-looking): warp 0 factors the panel
    // (columns i0 .. i1 - 1, every row below) column by column, lane = row; then every warp
    // (warp = row, lane = column) subtracts the panel's rank-8 term from the trailing matrix.
    // Non-positive pivots (rounding in a rank-deficient system) count as 1e-300.
    constexpr int KB = 8;
    for (int i0 = 0; i0 < k; i0 += KB) {
        const int nb = min(KB, k - i0), i1 = i0 + nb;
        if (warp == 0) {
            for (int j = 0; j < nb; ++j) {
                const int cj = i0 + j;
                double piv = L[tri(cj) + cj];
                piv = piv > 0.0 ? piv : 1e-300;
                const double sq = sqrt(piv), inv = 1.0 / sq;
                __syncwarp();
                if (lane == 0) L[tri(cj) + cj] = sq;
                for (int r = cj + 1 + lane; r < k; r += 32) L[tri(r) + cj] *= inv;
                __syncwarp();
                for (int cc = cj + 1; cc < i1; ++cc) {
                    const double lcj = L[tri(cc) + cj];
                    for (int r = cc + lane; r < k; r += 32) L[tri(r) + cc] -= L[tri(r) + cj] * lcj;
                }
                __syncwarp();
            }
        }
        __syncthreads();
        for (int t = 0; i1 + 32 * t < k; ++t) {
            const int c = i1 + lane + 32 * t;
            const bool valid = c < k;
            double cp[KB];
#pragma unroll
            for (int e = 0; e < KB; ++e) cp[e] = valid && e < nb ? L[tri(c) + i0 + e] : 0.0;
            for (int i = i1 + 32 * t + warp; i < k; i += nw) {
                if (valid && c <= i) {
                    const double *li = L + tri(i) + i0;
                    double s0 = 0.0, s1 = 0.0;
#pragma unroll
                    for (int e = 0; e < KB; e += 2) {
                        if (e < nb) s0 = fma(li[e], cp[e], s0);
                        if (e + 1 < nb) s1 = fma(li[e + 1], cp[e + 1], s1);
                    }
                    L[tri(i) + c] -= s0 + s1;
                }
            }
        }
        __syncthreads();
    }
    for (int i = tid; i < k; i += nt) invd[i] = 1.0 / L[tri(i) + i];
    __syncthreads();

    // 3. L Y = Z (forward), then L^T W = Y (backward), 8 rows per step: warp 0 (lane = column)
    // solves the step's 8 x 8 diagonal block in registers; then every warp (a row group, lane =
    // column) subtracts the block's contribution from the remaining rows.
    const int c = lane;
    for (int i0 = 0; i0 < k; i0 += KB) {
        const int i1 = min(i0 + KB, k);
        if (warp == 0) {
            double zb[KB];
#pragma unroll
            for (int e = 0; e < KB; ++e) zb[e] = i0 + e < i1 ? Z[(i0 + e) * NC + c] : 0.0;
#pragma unroll
            for (int i = 0; i < KB; ++i) {
                if (i0 + i < i1) {
                    const double *li = L + tri(i0 + i) + i0;
                    double sum = zb[i];
#pragma unroll
                    for (int e = 0; e < i; ++e) sum -= li[e] * zb[e];
                    zb[i] = sum * invd[i0 + i];
                }
            }
#pragma unroll
            for (int e = 0; e < KB; ++e)
                if (i0 + e < i1) Z[(i0 + e) * NC + c] = zb[e];
        }
        __syncthreads();
        double y[KB];
#pragma unroll
        for (int e = 0; e < KB; ++e) y[e] = i0 + e < i1 ? Z[(i0 + e) * NC + c] : 0.0;
        for (int j = i1 + warp; j < k; j += nw) {
            const double *lj = L + tri(j) + i0;
            double lv[KB];
#pragma unroll
            for (int e = 0; e < KB; ++e) lv[e] = i0 + e < i1 ? lj[e] : 0.0;
            double s0 = Z[j * NC + c], s1 = 0.0;
#pragma unroll
            for (int e = 0; e < KB; e += 2) {
                s0 -= lv[e] * y[e];
                s1 -= lv[e + 1] * y[e + 1];
            }
            Z[j * NC + c] = s0 + s1;
        }
        __syncthreads();
    }
    for (int i1 = k; i1 > 0; i1 -= KB) {
        const int i0 = max(i1 - KB, 0);
        if (warp == 0) {
            double xb[KB];
#pragma unroll
            for (int e = 0; e < KB; ++e) xb[e] = i0 + e < i1 ? Z[(i0 + e) * NC + c] : 0.0;
#pragma unroll
            for (int i = KB - 1; i >= 0; --i) {
                if (i0 + i < i1) {
                    double sum = xb[i];
#pragma unroll
                    for (int e = i + 1; e < KB; ++e)
                        if (i0 + e < i1) sum -= L[tri(i0 + e) + i0 + i] * xb[e];
                    xb[i] = sum * invd[i0 + i];
                }
            }
#pragma unroll
            for (int e = 0; e < KB; ++e)
                if (i0 + e < i1) Z[(i0 + e) * NC + c] = xb[e];
        }
        __syncthreads();
        double x[KB];
#pragma unroll
        for (int e = 0; e < KB; ++e) x[e] = i0 + e < i1 ? Z[(i0 + e) * NC + c] : 0.0;
        for (int j = warp; j < i0; j += nw) {
            double lv[KB];
#pragma unroll
            for (int e = 0; e < KB; ++e) lv[e] = i0 + e < i1 ? L[tri(i0 + e) + j] : 0.0;
            double s0 = Z[j * NC + c], s1 = 0.0;
#pragma unroll
            for (int e = 0; e < KB; e += 2) {
                s0 -= lv[e] * x[e];
                s1 -= lv[e + 1] * x[e + 1];
            }
            Z[j * NC + c] = s0 + s1;
        }
        __syncthreads();
    }

    // 4. this CTA's columns of W (n x d): the solution itself, or X^T Y on the smaller side
    __nv_bfloat16 *wp = wparts + bh * 2 * d * d;
    for (int p = tid; p < n * NC; p += nt) {
        const int e = p / NC, cl = p % NC, cc = c0 + cl;
        double w;
        if (tall) {
            w = Z[p];
        } else {
            w = 0.0;
            for (int r = 0; r < m; ++r)
                w = fma(e < d ? Mh[(long long)r * w2 + e] : 1.0, Z[r * NC + cl], w);
        }
        if (e < d) {
            const __nv_bfloat16 h = __double2bfloat16(w);
            wp[e * d + cc] = h;
            wp[(d + e) * d + cc] = __double2bfloat16(w - (double)__bfloat162float(h));
        } else {
            woff[bh * d + cc] = (float)w;
        }
    }
}

size_t probe_solve_smem(int m, int d) {
    const int n = d + 1, k = m >= n ? n : m;
    return ((size_t)k * (k + 1) / 2 + k + (size_t)k * kSolveCols) * sizeof(double);
}

cudaError_t sparsepr_solve(const double *M, double *C, double *sums, __nv_bfloat16 *wparts,
                           float *woff, long long BH, int m, int d, cudaStream_t st) {
    if (m >= d + 1) {
        const int tiles = (d / 64) * (2 * d / 64);
        probe_gram_kernel<<<dim3((unsigned)tiles + 1, (unsigned)BH), 256, 0, st>>>(M, C, sums, m, d);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const size_t smem = probe_solve_smem(m, d);
    cudaError_t e = cudaFuncSetAttribute(probe_solve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    probe_solve_kernel<<<dim3((unsigned)(d / kSolveCols), (unsigned)BH), kSolveThreads, smem, st>>>(
        M, C, sums, wparts, woff, m, d, 1e-12);
    return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// O += [O, 1] W on the tensor cores, in place on the bf16 output
// ------------------------------------------------------------------------------------------
// Per 128-row tile of one head the product O W is a dense 128 x D x D contraction: A is the bf16
// tile of O itself (exact), B is W's first D rows split into two bf16 parts (W ~ W_hi + W_lo,
// relative error 2^-17), both accumulated in fp32 in tensor memory; the epilogue adds O and the
// offset row (fp32) and rounds to bf16 once.  The kernel is bound by reading and writing O.
//
// Persistent CTAs (one per SM), each owning a contiguous run of the head-major tile sequence,
// so W is loaded once per head change:
//   warp 0 lane 0  TMA producer: W parts per head, O tiles into a 4-slot ring
//   warp 1 lane 0  MMA issuer:   acc[i % 2] = O_i W_hi + O_i W_lo
//   warp 2         tensor-memory allocator (2 accumulators of D columns)
//   warps 4..7     epilogue: thread = tile row; result written over the O slot, then stored by
//                  TMA (32 rows per warp), the slot released once the store has read it
template <int D>
struct ApplyCfg {
    static constexpr int CHUNKS = D / 64;        // 64-column (128-byte) swizzle chunks
    static constexpr int O_CHUNK = 128 * 128;    // 128 rows x 128 bytes
    static constexpr int O_BYTES = CHUNKS * O_CHUNK;
    static constexpr int W_CHUNK = D * 128;      // D rows x 128 bytes
    static constexpr int W_PART = CHUNKS * W_CHUNK;
    static constexpr int W_BYTES = 2 * W_PART;
    static constexpr int NSLOT = 4, NACC = 2;
    static constexpr int OFF_W = 0;
    static constexpr int OFF_O = W_BYTES;
    static constexpr int OFF_BAR = OFF_O + NSLOT * O_BYTES;
    static constexpr int SMEM = OFF_BAR + 256 + 1024;  // barriers + slack for 1024-byte alignment
    static constexpr uint32_t TMEM_COLS = NACC * D;
};

enum { A_WF, A_WE, A_OF0, A_OE0 = A_OF0 + 4, A_AF0 = A_OE0 + 4, A_AE0 = A_AF0 + 2, A_FIN = A_AE0 + 2,
       A_COUNT };

struct ApplyParams {
    const float *woff;   // [BH, D] the offset row of W (fp32)
    int N, tiles;        // rows per head, 128-row tiles per head
    long long total;     // BH * tiles
    unsigned long long wait_ns;
};

template <int D>
__global__ void __launch_bounds__(256, 1)
    apply_correction_tc_kernel(const __grid_constant__ CUtensorMap tmO,
                               const __grid_constant__ CUtensorMap tmOst,
                               const __grid_constant__ CUtensorMap tmW, const ApplyParams prm) {
    using C = ApplyCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::OFF_BAR + 8 * A_COUNT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_BAR + 8 * A_COUNT + 4);
    static_assert(8 * A_COUNT + 8 <= 256, "barrier area overflow");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t sW = smem_u32(smem + C::OFF_W), sO = smem_u32(smem + C::OFF_O);
    auto bar = [&](int b) { return smem_u32(&bars[b]); };
    // this CTA's run of the head-major tile sequence
    const long long lo = prm.total * blockIdx.x / gridDim.x;
    const long long hi = prm.total * (blockIdx.x + 1) / gridDim.x;

    if (threadIdx.x == 0) {
        mbar_init(bar(A_WF), 1);
        mbar_init(bar(A_WE), 1);
        for (int s = 0; s < C::NSLOT; ++s) {
            mbar_init(bar(A_OF0 + s), 1);
            mbar_init(bar(A_OE0 + s), 4);
        }
        for (int a = 0; a < C::NACC; ++a) {
            mbar_init(bar(A_AF0 + a), 1);
            mbar_init(bar(A_AE0 + a), 4);
        }
        mbar_init(bar(A_FIN), 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmO);
        prefetch_tmap(&tmOst);
        prefetch_tmap(&tmW);
    }
    if (warp == 2) {
        tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tacc = *tmem_holder;
    const unsigned long long wns = prm.wait_ns;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        uint32_t nw = 0, no = 0;
        long long cur = -1;
        bool ok = true;
        for (long long t = lo; t < hi && ok; ++t) {
            const long long bh = t / prm.tiles;
            const int tile = (int)(t - bh * prm.tiles);
            if (bh != cur) {
                // W of the previous head must be consumed by its last MMA
                if (nw > 0 && !(ok = warp_wait(bar(A_WE), (nw - 1) & 1, wns, abort_flag, 0x51, (uint32_t)t)))
                    break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar(A_WF), C::W_BYTES);
#pragma unroll
                    for (int part = 0; part < 2; ++part)
#pragma unroll
                        for (int c = 0; c < C::CHUNKS; ++c)
                            tma_load_3d(sW + part * C::W_PART + c * C::W_CHUNK, &tmW, bar(A_WF), c * 64,
                                        part * D, (int)bh);
                }
                ++nw;
                cur = bh;
            }
            const int slot = no % C::NSLOT;
            if (no >= C::NSLOT &&
                !(ok = warp_wait(bar(A_OE0 + slot), ((no / C::NSLOT) - 1) & 1, wns, abort_flag, 0x52, (uint32_t)t)))
                break;
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(A_OF0 + slot), C::O_BYTES);
#pragma unroll
                for (int c = 0; c < C::CHUNKS; ++c)
                    tma_load_3d(sO + slot * C::O_BYTES + c * C::O_CHUNK, &tmO, bar(A_OF0 + slot), c * 64,
                                tile * 128, (int)bh);
            }
            ++no;
        }
        if (!ok && lane == 0) {  // let every copy that was started land before the CTA leaves
            if (nw) drain_wait(bar(A_WF), (nw - 1) & 1, wns, 0x55);
            for (uint32_t i = no > C::NSLOT ? no - C::NSLOT : 0; i < no; ++i)
                drain_wait(bar(A_OF0 + i % C::NSLOT), (i / C::NSLOT) & 1, wns, 0x56);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        constexpr uint32_t IDESC = idesc_bf16_f32(128, D, 0, 1);
        const uint64_t dO = smem_desc_sw128(sO, 16, 1024);               // A: K-major tile of O
        const uint64_t dW = smem_desc_sw128(sW, C::W_CHUNK, 1024);       // B: W rows, N innermost
        uint32_t nw = 0, no = 0;
        long long cur = -1;
        bool ok = true;
        for (long long t = lo; t < hi && ok; ++t) {
            const long long bh = t / prm.tiles;
            if (bh != cur) {
                if (!(ok = warp_wait(bar(A_WF), nw & 1, wns, abort_flag, 0x61, (uint32_t)t))) break;
                ++nw;
                cur = bh;
            }
            const int slot = no % C::NSLOT, a = no % C::NACC;
            if (!(ok = warp_wait(bar(A_OF0 + slot), (no / C::NSLOT) & 1, wns, abort_flag, 0x62, (uint32_t)t)))
                break;
            if (no >= C::NACC &&
                !(ok = warp_wait(bar(A_AE0 + a), ((no / C::NACC) - 1) & 1, wns, abort_flag, 0x63, (uint32_t)t)))
                break;
            tc_fence_after();
            const bool last_of_head = t + 1 >= hi || (t + 1) / prm.tiles != bh;
            if (lane == 0) {
                const uint64_t oslot = (uint64_t)((slot * C::O_BYTES) >> 4);
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        // A step kk: 32 bytes inside the swizzled row, then the next chunk;
                        // B step kk: 16 rows of 128 bytes
                        const uint64_t oa = oslot + (uint64_t)(((kk >> 2) * C::O_CHUNK + (kk & 3) * 32) >> 4);
                        const uint64_t ob = (uint64_t)((part * C::W_PART + kk * 2048) >> 4);
                        mma_ss(tacc + a * D, dO + oa, dW + ob, IDESC, (part | kk) ? 1u : 0u);
                    }
                mma_commit(bar(A_AF0 + a));
                if (last_of_head) mma_commit(bar(A_WE));
            }
            __syncwarp();
            ++no;
        }
        // every MMA this warp issued must be complete before tensor memory is released
        if (lane == 0) {
            mma_commit(bar(A_FIN));
            drain_wait(bar(A_FIN), 0, wns, 0x64);
        }
    } else if (warp >= 4) {
        // ---------------------------------------------------------------- epilogue
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;  // tile row == TMEM lane
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        uint32_t no = 0;
        bool ok = true;
        int prev_slot = -1;
        for (long long t = lo; t < hi && ok; ++t) {
            const long long bh = t / prm.tiles;
            const int tile = (int)(t - bh * prm.tiles);
            const int slot = no % C::NSLOT, a = no % C::NACC;
            if (!(ok = warp_wait(bar(A_AF0 + a), (no / C::NACC) & 1, wns, abort_flag, 0x71, (uint32_t)t)))
                break;
            // the O load into this slot has landed (its MMAs have completed); waiting on its
            // barrier too makes the TMA writes visible to this warp's own reads of the slot
            if (!(ok = warp_wait(bar(A_OF0 + slot), (no / C::NSLOT) & 1, wns, abort_flag, 0x72, (uint32_t)t)))
                break;
            tc_fence_after();
            uint32_t acc[D];
            tmem_ld_cols<D>(tacc + a * D + lane_off, acc);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(A_AE0 + a));
            // the slot holds this tile's O (the load completed before the MMAs that read it)
            uint8_t *rowp = smem + C::OFF_O + slot * C::O_BYTES + r * 128;
            const float *off = prm.woff + bh * D;
#pragma unroll
            for (int u = 0; u < D / 8; ++u) {  // 16-byte units of 8 columns
                const int c = u >> 3, pu = (u & 7) ^ (r & 7);
                uint4 *p = reinterpret_cast<uint4 *>(rowp + c * C::O_CHUNK + pu * 16);
                const uint4 ov = *p;
                const float4 f0 = __ldg(reinterpret_cast<const float4 *>(off + u * 8));
                const float4 f1 = __ldg(reinterpret_cast<const float4 *>(off + u * 8 + 4));
                const float fo[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
                const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w};
                uint32_t res[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float x0 = __uint_as_float(ow[e] << 16), x1 = __uint_as_float(ow[e] & 0xFFFF0000u);
                    res[e] = pack_bf16(x0 + (__uint_as_float(acc[u * 8 + 2 * e]) + fo[2 * e]),
                                       x1 + (__uint_as_float(acc[u * 8 + 2 * e + 1]) + fo[2 * e + 1]));
                }
                *p = make_uint4(res[0], res[1], res[2], res[3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                const int row0 = tile * 128 + q4 * 32;
                if (row0 < prm.N) {
#pragma unroll
                    for (int c = 0; c < C::CHUNKS; ++c)
                        tma_store_3d(&tmOst, sO + slot * C::O_BYTES + c * C::O_CHUNK + q4 * 4096, c * 64,
                                     row0, (int)bh);
                }
                bulk_commit_group();
                // the previous tile's store has read its slot: release it to the producer
                bulk_wait_group_read<1>();
                if (prev_slot >= 0) mbar_arrive(bar(A_OE0 + prev_slot));
            }
            __syncwarp();
            prev_slot = slot;
            ++no;
        }
        if (lane == 0) bulk_wait_group<0>();  // every store written before the CTA leaves
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 2) tmem_dealloc(tacc, C::TMEM_COLS);
}

template <int D>
static cudaError_t launch_apply_t(const CUtensorMap &tmO, const CUtensorMap &tmOst,
                                  const CUtensorMap &tmW, const ApplyParams &p, int num_sms,
                                  cudaStream_t st) {
    using C = ApplyCfg<D>;
    cudaError_t e = cudaFuncSetAttribute(apply_correction_tc_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    long long grid = num_sms;
    if (grid > p.total) grid = p.total;
    if (grid <= 0) return cudaSuccess;
    apply_correction_tc_kernel<D><<<(unsigned)grid, 256, C::SMEM, st>>>(tmO, tmOst, tmW, p);
    return cudaGetLastError();
}

// tmO: O with 128-row boxes (loads), tmOst: O with 32-row boxes (stores), tmW: the W parts
// [BH, 2 D, D] with D-row boxes.
cudaError_t sparsepr_apply(const CUtensorMap &tmO, const CUtensorMap &tmOst, const CUtensorMap &tmW,
                           const float *woff, long long BH, int N, int d, unsigned long long wait_ns,
                           int num_sms, cudaStream_t st) {
    ApplyParams p;
    p.woff = woff;
    p.N = N;
    p.tiles = (N + 127) / 128;
    p.total = BH * p.tiles;
    p.wait_ns = wait_ns;
    return d == 128 ? launch_apply_t<128>(tmO, tmOst, tmW, p, num_sms, st)
                    : launch_apply_t<64>(tmO, tmOst, tmW, p, num_sms, st);
}
// Probe-row tables for the variable-length kernel with the keys split S ways: unit (s, u) is
// query tile u (128 probe rows) of "cluster" s, whose key list is the s-th contiguous run of the
// ceil(N / 128) key tiles (the last tile ragged); output rows are the identity.
__global__ void __launch_bounds__(256) probe_tables_kernel(int2 *__restrict__ units,
                                                           int32_t *__restrict__ tiles,
                                                           int32_t *__restrict__ tcnt,
                                                           int32_t *__restrict__ perm,
                                                           long long BH, int N, int m, int U,
                                                           int S, int tstride) {
    const long long bh = blockIdx.x;
    for (int x = threadIdx.x; x < U * S; x += blockDim.x) {
        const int sp = x / U, r0 = (x - sp * U) * 128;
        units[bh * U * S + x] = r0 < m ? make_int2(r0, (min(128, m - r0) << 16) | sp) : make_int2(0, 0);
    }
    const int nt = (N + 127) / 128;
    for (int x = threadIdx.x; x < S * tstride; x += blockDim.x) {
        const int sp = x / tstride, i = x - sp * tstride;
        const int t = (int)((long long)sp * nt / S) + i;
        if (t < (int)((long long)(sp + 1) * nt / S))
            tiles[(bh * S + sp) * tstride + i] = ((t * 128) << 7) | (min(128, N - t * 128) - 1);
    }
    for (int sp = threadIdx.x; sp < S; sp += blockDim.x)
        tcnt[bh * S + sp] = (int)((long long)(sp + 1) * nt / S - (long long)sp * nt / S);
    for (int i = threadIdx.x; i < m; i += blockDim.x) perm[bh * m + i] = i;
}

// Key splits of the probe attention: enough (query tile, key run) units to keep every SM of a
// 148-SM device busy with two CTAs about twice over, at most one per key tile and 64 in all.
int probe_splits(long long BH, int N, int m) {
    const long long units = BH * ((m + 127) / 128);
    long long s = (592 + units - 1) / units;
    const int nt = (N + 127) / 128;
    if (s > nt) s = nt;
    if (s > 64) s = 64;
    return s < 1 ? 1 : (int)s;
}

}  // namespace bsa

namespace {

struct ProbeWorkspace {
    unsigned int *counter;
    void *qpr;
    float *po, *plse;
    int2 *units;
    int32_t *tiles, *tcnt, *perm;
    double *M, *C, *sums;
    __nv_bfloat16 *wparts;
    float *woff;
    int U, S, tstride;
};

size_t probe_workspace(int B, int H, int N, int d, int m, void *base, ProbeWorkspace *w) {
    const size_t BH = (size_t)B * H;
    ProbeWorkspace t;
    t.U = (m + 127) / 128;
    t.S = bsa::probe_splits(BH, N, m);
    t.tstride = ((N + 127) / 128 + t.S - 1) / t.S;
    size_t off = 0;
    uint8_t *p = reinterpret_cast<uint8_t *>(base);
    auto take = [&](size_t bytes) -> void * {
        void *r = p ? p + off : nullptr;
        off += (bytes + 255) & ~(size_t)255;
        return r;
    };
    t.counter = (unsigned int *)take(256);
    t.qpr = take(BH * m * d * 2);
    t.po = (float *)take((size_t)t.S * BH * m * d * 4);
    t.plse = (float *)take((size_t)t.S * BH * m * 4);
    t.units = (int2 *)take(BH * t.U * t.S * 8);
    t.tiles = (int32_t *)take(BH * t.S * t.tstride * 4);
    t.tcnt = (int32_t *)take(BH * t.S * 4);
    t.perm = (int32_t *)take(BH * m * 4);
    t.M = (double *)take(BH * m * 2 * d * 8);
    t.C = (double *)take(m >= d + 1 ? BH * (size_t)d * 2 * d * 8 : 0);
    t.sums = (double *)take(BH * 2 * d * 8);
    t.wparts = (__nv_bfloat16 *)take(BH * (size_t)2 * d * d * 2);
    t.woff = (float *)take(BH * (size_t)d * 4);
    if (w) *w = t;
    return off;
}

}  // namespace

constexpr int kMaxProbes = 8192;  // probe rows per head

extern "C" size_t sa_sparsepr_workspace_bytes(int B, int H, int N, int d, int m) {
    if (B <= 0 || H <= 0 || N <= 0 || (d != 64 && d != 128) || m <= 0 || m > kMaxProbes) return 0;
    return probe_workspace(B, H, N, d, m, nullptr, nullptr);
}

// O = block-sparse attention over (kv_idx, kv_cnt), corrected by the probe fit with the exact
// outputs of the m probe rows of each head (probes [B, H, m] int32 token ids).
extern "C" sa_status sa_sparsepr_attn_fwd(const void *q, const void *k, const void *v,
                                          const int32_t *kv_idx, const int32_t *kv_cnt,
                                          const int32_t *probes, int m, void *o, int B, int H,
                                          int N, int d, int bs, float scale, void *workspace,
                                          size_t workspace_bytes, void *stream) {
    if (!q || !k || !v || !kv_idx || !kv_cnt || !probes || !o || !workspace) return SA_ERR_INVALID_ARG;
    if (!shape_ok(B, H, N) || m < 1 || m > kMaxProbes || m > N || isnan(scale)) return SA_ERR_INVALID_ARG;
    if (!dims_supported(d, bs)) return SA_ERR_UNSUPPORTED;
    if (sa_num_blocks(N, bs) > 1024 || N >= (1 << 24)) return SA_ERR_UNSUPPORTED;
    if (workspace_bytes < sa_sparsepr_workspace_bytes(B, H, N, d, m) || !aligned16(workspace))
        return SA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(probes))
        return SA_ERR_INVALID_ARG;
    int dev;
    if (!select_device(o, &dev)) return SA_ERR_INVALID_ARG;
    const cudaStream_t st = (cudaStream_t)stream;
    const long long BH = (long long)B * H;
    ProbeWorkspace w;
    probe_workspace(B, H, N, d, m, workspace, &w);
    // 1. the sparse output
    sa_status s = run_attention(q, k, v, kv_idx, kv_cnt, o, B, H, N, d, bs, scale, w.counter, stream);
    if (s != SA_OK) return s;
    // 2. exact outputs of the probe rows
    const int sms = num_sms(dev);
    const int vec = d / 8;
    bsa::gather_probe_rows_kernel<<<(unsigned)((BH * m * vec + 255) / 256 < sms * 16 ? (BH * m * vec + 255) / 256 : sms * 16), 256, 0, st>>>(
        reinterpret_cast<const uint4 *>(q), probes, reinterpret_cast<uint4 *>(w.qpr), BH, N, m, vec);
    bsa::probe_tables_kernel<<<(unsigned)BH, 256, 0, st>>>(w.units, w.tiles, w.tcnt, w.perm, BH, N, m,
                                                           w.U, w.S, w.tstride);
    if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;
    CUtensorMap tq, tk, tv;
    if (!make_tmap(&tq, w.qpr, BH, m, d, 128) || !make_tmap(&tk, k, BH, N, d, 128) ||
        !make_tmap(&tv, v, BH, N, d, 128))
        return SA_ERR_CUDA;
    cudaError_t e = bsa::attn_varlen_fwd(tq, tk, tv, w.units, w.U * w.S, w.tiles, w.tcnt, w.tstride,
                                         w.perm, nullptr, BH, N, m, w.S, d, resolve_scale(scale, d),
                                         g_wait_ns, sms, w.counter, st, w.po, w.plse);
    if (e != cudaSuccess) return SA_ERR_CUDA;
    // 3. residuals, the per-head least-squares map, the correction of every row
    const long long nres = BH * m * d;
    bsa::probe_merge_kernel<<<(unsigned)((nres + 255) / 256 < sms * 8 ? (nres + 255) / 256 : sms * 8), 256, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16 *>(o), w.po, w.plse, probes, w.M, BH, N, m, d, w.S);
    if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;
    e = bsa::sparsepr_solve(w.M, w.C, w.sums, w.wparts, w.woff, BH, m, d, st);
    if (e != cudaSuccess) return SA_ERR_CUDA;
    CUtensorMap to, tost, tw;
    if (!make_tmap(&to, o, BH, N, d, 128) || !make_tmap(&tost, o, BH, N, d, 32) ||
        !make_tmap(&tw, w.wparts, BH, 2 * d, d, d))
        return SA_ERR_CUDA;
    return from_cuda(bsa::sparsepr_apply(to, tost, tw, w.woff, BH, N, d, g_wait_ns, sms, st));
}
