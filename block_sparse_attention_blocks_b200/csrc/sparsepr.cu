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
// At the full numerical rank this is the page's fit of the residuals in their observed output
// subspace: the minimum-norm least-squares map of the residuals is already a combination of the
// rows of R.
//
// Steps (one stream, no host synchronisation):
//   1. O_s by the block-sparse attention kernel;
//   2. the probe rows of Q gathered into [BH, m, d]; their exact outputs by the variable-length
//      attention kernel with one query cluster covering the m rows and one key list covering
//      every key (128-key tiles, the last one ragged);
//   3. X and R in fp64; W by one CTA per head in fp64: the normal equations of the smaller side,
//      Cholesky with a ridge of 1e-12 times the mean diagonal (which keeps a rank-deficient X
//      solvable and approximates the pseudo-inverse's minimum-norm choice);
//   4. O += [O, 1] W in place on the bf16 output (W staged in shared memory per head).
#include "bsa_internal.h"
#include "sparse_attn.h"

namespace bsa {

// ------------------------------------------------------------------------------------------
// minimum-norm least squares for one head, by a team of threads (a CTA), fp64
// ------------------------------------------------------------------------------------------
namespace lsq {

// In-place Cholesky of the k x k SPD matrix G (row-major, lower triangle used), G = L L^T.
template <class Sync>
__device__ void cholesky(double *G, int k, int tid, int nt, Sync sync) {
    for (int j = 0; j < k; ++j) {
        if (tid == 0) G[j * k + j] = sqrt(G[j * k + j] > 0.0 ? G[j * k + j] : 1e-300);
        sync();
        const double inv = 1.0 / G[j * k + j];
        for (int i = j + 1 + tid; i < k; i += nt) G[i * k + j] *= inv;
        sync();
        // trailing update of the lower triangle: G[i][c] -= L[i][j] L[c][j], j < c <= i
        const int w = k - j - 1;
        const long long pairs = (long long)w * (w + 1) / 2;
        for (long long p = tid; p < pairs; p += nt) {
            // p -> (ii, cc) with 0 <= cc <= ii < w
            int ii = (int)((sqrt(8.0 * (double)p + 1.0) - 1.0) / 2.0);
            while ((long long)(ii + 1) * (ii + 2) / 2 <= p) ++ii;
            while ((long long)ii * (ii + 1) / 2 > p) --ii;
            const int cc = (int)(p - (long long)ii * (ii + 1) / 2);
            const int i = j + 1 + ii, c = j + 1 + cc;
            G[i * k + c] -= G[i * k + j] * G[c * k + j];
        }
        sync();
    }
}

// Solve L L^T Y = B in place for `ncol` right-hand sides (B row-major k x ncol), one column per
// thread.
template <class Sync>
__device__ void chol_solve(const double *L, int k, double *B, int ncol, int tid, int nt, Sync sync) {
    for (int c = tid; c < ncol; c += nt) {
        for (int i = 0; i < k; ++i) {  // forward: L y = b
            double s = B[i * ncol + c];
            for (int e = 0; e < i; ++e) s -= L[i * k + e] * B[e * ncol + c];
            B[i * ncol + c] = s / L[i * k + i];
        }
        for (int i = k - 1; i >= 0; --i) {  // backward: L^T x = y
            double s = B[i * ncol + c];
            for (int e = i + 1; e < k; ++e) s -= L[e * k + i] * B[e * ncol + c];
            B[i * ncol + c] = s / L[i * k + i];
        }
    }
    sync();
}

// X [m x n] (n = d + 1, last column ones), R [m x d] -> W [n x d].
// Scratch: G [min(m, n)^2], Z [min(m, n) * d].
template <class Sync>
__device__ void min_norm_lstsq(const double *X, const double *R, int m, int d, double *W, double *G,
                          double *Z, double eps, int tid, int nt, Sync sync) {
    const int n = d + 1;
    if (m >= n) {
        for (int p = tid; p < n * n; p += nt) {  // G = X^T X
            const int i = p / n, c = p % n;
            double s = 0.0;
            for (int r = 0; r < m; ++r) s += X[r * n + i] * X[r * n + c];
            G[p] = s;
        }
        for (int p = tid; p < n * d; p += nt) {  // Z = X^T R
            const int i = p / d, c = p % d;
            double s = 0.0;
            for (int r = 0; r < m; ++r) s += X[r * n + i] * R[r * d + c];
            Z[p] = s;
        }
        sync();
        if (tid == 0) {
            double tr = 0.0;
            for (int i = 0; i < n; ++i) tr += G[i * n + i];
            for (int i = 0; i < n; ++i) G[i * n + i] += eps * tr / n;
        }
        sync();
        cholesky(G, n, tid, nt, sync);
        chol_solve(G, n, Z, d, tid, nt, sync);
        for (int p = tid; p < n * d; p += nt) W[p] = Z[p];
        sync();
    } else {
        for (int p = tid; p < m * m; p += nt) {  // G = X X^T
            const int i = p / m, c = p % m;
            double s = 0.0;
            for (int e = 0; e < n; ++e) s += X[i * n + e] * X[c * n + e];
            G[p] = s;
        }
        for (int p = tid; p < m * d; p += nt) Z[p] = R[p];
        sync();
        if (tid == 0) {
            double tr = 0.0;
            for (int i = 0; i < m; ++i) tr += G[i * m + i];
            for (int i = 0; i < m; ++i) G[i * m + i] += eps * tr / m;
        }
        sync();
        cholesky(G, m, tid, nt, sync);
        chol_solve(G, m, Z, d, tid, nt, sync);
        for (int p = tid; p < n * d; p += nt) {  // W = X^T Z
            const int i = p / d, c = p % d;
            double s = 0.0;
            for (int r = 0; r < m; ++r) s += X[r * n + i] * Z[r * d + c];
            W[p] = s;
        }
        sync();
    }
}

}  // namespace lsq

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

// X [BH, m, d + 1] and R [BH, m, d] in fp64 from O_s (bf16 [BH, N, d]) and E (bf16 [BH, m, d]).
__global__ void __launch_bounds__(256) probe_residual_kernel(
    const __nv_bfloat16 *__restrict__ os, const __nv_bfloat16 *__restrict__ e,
    const int32_t *__restrict__ probes, double *__restrict__ X, double *__restrict__ R,
    long long BH, int N, int m, int d) {
    const long long total = BH * m * (d + 1);
    for (long long x = (long long)blockIdx.x * blockDim.x + threadIdx.x; x < total;
         x += (long long)gridDim.x * blockDim.x) {
        const long long row = x / (d + 1);  // bh * m + i
        const int c = (int)(x - row * (d + 1));
        if (c == d) {
            X[x] = 1.0;
            continue;
        }
        const long long bh = row / m;
        const int t = min(max(probes[row], 0), N - 1);
        const double o = (double)__bfloat162float(os[(bh * N + t) * d + c]);
        X[x] = o;
        R[row * d + c] = (double)__bfloat162float(e[row * d + c]) - o;
    }
}

// One CTA per head: W [BH, d + 1, d] (fp32) = X^+ R.  Scratch per head: G [k^2], Z [k d],
// k = min(m, d + 1) (the normal equations of the smaller side), fp64.
__global__ void __launch_bounds__(256) probe_solve_kernel(const double *__restrict__ X,
                                                          const double *__restrict__ R,
                                                          double *__restrict__ G,
                                                          double *__restrict__ Z,
                                                          double *__restrict__ Wd,
                                                          float *__restrict__ W, int m, int d,
                                                          double eps) {
    const long long bh = blockIdx.x;
    const int n = d + 1, k = m < n ? m : n;
    auto sync = []() { __syncthreads(); };
    double *w64 = Wd + bh * n * d;
    lsq::min_norm_lstsq(X + bh * m * n, R + bh * m * d, m, d, w64, G + bh * k * k,
                                Z + bh * (long long)k * d, eps, threadIdx.x, blockDim.x, sync);
    for (int p = threadIdx.x; p < n * d; p += blockDim.x) W[bh * n * d + p] = (float)w64[p];
}

// O[bh, t, :] += [O[bh, t, :], 1] W[bh]   in place on the bf16 output; CTA = 64 rows of one
// head, thread = (row, 32-column block); W of the head staged in shared memory.
template <int D>
__global__ void __launch_bounds__(256) apply_correction_kernel(__nv_bfloat16 *__restrict__ o,
                                                               const float *__restrict__ W,
                                                               int N) {
    constexpr int ROWS = 64, CB = D / 32;  // rows per CTA, column blocks per row
    constexpr int TPR = 256 / ROWS;        // threads per row (4)
    static_assert(CB % TPR == 0 || TPR % CB == 0, "layout");
    extern __shared__ float sm_apply[];
    float *ws = sm_apply;                  // [(D + 1) * D]
    float *os = sm_apply + (D + 1) * D;    // [ROWS][D + 1]
    const long long bh = blockIdx.y;
    const int r0 = blockIdx.x * ROWS;
    for (int p = threadIdx.x; p < (D + 1) * D; p += 256) ws[p] = W[bh * (D + 1) * D + p];
    for (int p = threadIdx.x; p < ROWS * D; p += 256) {
        const int rr = p / D, c = p % D;
        const int t = r0 + rr;
        os[rr * (D + 1) + c] = t < N ? __bfloat162float(o[(bh * N + t) * D + c]) : 0.f;
    }
    __syncthreads();
    const int rr = threadIdx.x / TPR, part = threadIdx.x % TPR;
    const int t = r0 + rr;
    for (int cb = part; cb < CB; cb += TPR) {
        float acc[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[j] = ws[D * D + cb * 32 + j];  // the offset row
        for (int e = 0; e < D; ++e) {
            const float a = os[rr * (D + 1) + e];
#pragma unroll
            for (int j = 0; j < 32; ++j) acc[j] = fmaf(a, ws[e * D + cb * 32 + j], acc[j]);
        }
        if (t < N) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int c = cb * 32 + j;
                o[(bh * N + t) * D + c] = __float2bfloat16(os[rr * (D + 1) + c] + acc[j]);
            }
        }
    }
}


cudaError_t sparsepr_apply(void *o, const float *W, long long BH, int N, int d, cudaStream_t st) {
    const dim3 g((unsigned)((N + 63) / 64), (unsigned)BH);
    auto *ob = reinterpret_cast<__nv_bfloat16 *>(o);
    if (d == 128) {
        const size_t smem = ((size_t)129 * 128 + 64 * 129) * 4;
        cudaFuncSetAttribute(apply_correction_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        apply_correction_kernel<128><<<g, 256, smem, st>>>(ob, W, N);
    } else {
        const size_t smem = ((size_t)65 * 64 + 64 * 65) * 4;
        apply_correction_kernel<64><<<g, 256, smem, st>>>(ob, W, N);
    }
    return cudaGetLastError();
}
cudaError_t sparsepr_solve(const double *X, const double *R, double *G, double *Z, double *Wd,
                           float *W, long long BH, int m, int d, cudaStream_t st) {
    probe_solve_kernel<<<(unsigned)BH, 256, 0, st>>>(X, R, G, Z, Wd, W, m, d, 1e-12);
    return cudaGetLastError();
}

// Probe-row tables for the varlen kernel: per head ceil(m/128) query tiles of cluster 0, one
// key list covering [0, N) in 128-key tiles, identity output rows.
__global__ void __launch_bounds__(256) probe_tables_kernel(int2 *__restrict__ units,
                                                           int32_t *__restrict__ tiles,
                                                           int32_t *__restrict__ tcnt,
                                                           int32_t *__restrict__ perm,
                                                           long long BH, int N, int m, int U,
                                                           int tstride) {
    const long long bh = blockIdx.x;
    for (int u = threadIdx.x; u < U; u += blockDim.x) {
        const int r0 = u * 128;
        units[bh * U + u] = r0 < m ? make_int2(r0, min(128, m - r0) << 16) : make_int2(0, 0);
    }
    const int nt = (N + 127) / 128;
    for (int t = threadIdx.x; t < tstride; t += blockDim.x)
        if (t < nt) tiles[bh * tstride + t] = ((t * 128) << 7) | (min(128, N - t * 128) - 1);
    if (threadIdx.x == 0) tcnt[bh] = nt;
    for (int i = threadIdx.x; i < m; i += blockDim.x) perm[bh * m + i] = i;
}

}  // namespace bsa

namespace {

struct ProbeWorkspace {
    unsigned int *counter;
    void *qpr, *e;
    int2 *units;
    int32_t *tiles, *tcnt, *perm;
    double *X, *R, *G, *Z, *Wd;
    float *W;
    int U, tstride, k;
};

size_t probe_workspace(int B, int H, int N, int d, int m, void *base, ProbeWorkspace *w) {
    const size_t BH = (size_t)B * H;
    ProbeWorkspace t;
    t.U = (m + 127) / 128;
    t.tstride = (N + 127) / 128;
    t.k = m < d + 1 ? m : d + 1;
    size_t off = 0;
    uint8_t *p = reinterpret_cast<uint8_t *>(base);
    auto take = [&](size_t bytes) -> void * {
        void *r = p ? p + off : nullptr;
        off += (bytes + 255) & ~(size_t)255;
        return r;
    };
    t.counter = (unsigned int *)take(256);
    t.qpr = take(BH * m * d * 2);
    t.e = take(BH * m * d * 2);
    t.units = (int2 *)take(BH * t.U * 8);
    t.tiles = (int32_t *)take(BH * t.tstride * 4);
    t.tcnt = (int32_t *)take(BH * 4);
    t.perm = (int32_t *)take(BH * m * 4);
    t.X = (double *)take(BH * m * (d + 1) * 8);
    t.R = (double *)take(BH * m * d * 8);
    t.G = (double *)take(BH * (size_t)t.k * t.k * 8);
    t.Z = (double *)take(BH * (size_t)t.k * d * 8);
    t.Wd = (double *)take(BH * (size_t)(d + 1) * d * 8);
    t.W = (float *)take(BH * (size_t)(d + 1) * d * 4);
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
                                                           w.U, w.tstride);
    if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;
    CUtensorMap tq, tk, tv;
    if (!make_tmap(&tq, w.qpr, BH, m, d, 128) || !make_tmap(&tk, k, BH, N, d, 128) ||
        !make_tmap(&tv, v, BH, N, d, 128))
        return SA_ERR_CUDA;
    cudaError_t e = bsa::attn_varlen_fwd(tq, tk, tv, w.units, w.U, w.tiles, w.tcnt, w.tstride, w.perm,
                                         w.e, BH, N, m, 1, d, resolve_scale(scale, d), g_wait_ns,
                                         sms, w.counter, st);
    if (e != cudaSuccess) return SA_ERR_CUDA;
    // 3. residuals, the per-head least-squares map, the correction of every row
    const long long nres = BH * m * (d + 1);
    bsa::probe_residual_kernel<<<(unsigned)((nres + 255) / 256 < sms * 16 ? (nres + 255) / 256 : sms * 16), 256, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16 *>(o), reinterpret_cast<const __nv_bfloat16 *>(w.e),
        probes, w.X, w.R, BH, N, m, d);
    if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;
    e = bsa::sparsepr_solve(w.X, w.R, w.G, w.Z, w.Wd, w.W, BH, m, d, st);
    if (e == cudaSuccess) e = bsa::sparsepr_apply(o, w.W, BH, N, d, st);
    return from_cuda(e);
}
