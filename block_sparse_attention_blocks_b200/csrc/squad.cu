// SQuad attention (page "SQuad: Sub-Quadratic Attention Distillation for Efficient Video
// Generation", method section 1, the SQuad attention operator) on the library's kernels.  With
// n = W w tokens per (b, h), token t = a w + r (window a, position r):
//   local pass   Y[a w + r] = softmax over the w tokens of window a            (values v)
//   global pass  O[a w + r] = softmax over the W tokens at position r, one per window
//                                                                            (values Y)
// The local pass is one dense attention call over B*H*W "heads" of w tokens (a reshape of the
// [B, H, n, d] tensors, no copy).  Q, K and Y are then regrouped by position, [W, w] -> [w, W]
// within each (b, h); the global pass attends within each of the B*H*w sequences of W tokens
// (for W <= 64 packed 128 / W sequences to a 128-row tile with a block-diagonal mask, else one
// dense call over B*H*w heads), and its output is regrouped back into O.  For video with w = the tokens of one latent frame,
// the local pass is spatial attention within a frame and the global pass temporal attention
// across frames at each spatial position.
#include "bsa_internal.h"
#include "sparse_attn.h"

namespace bsa {

// dst[g, r, a, :] = src[g, a, r, :] for a < A, r < R: token rows of d bf16 moved as 16-byte
// vectors; consecutive threads read consecutive vectors of src.
__global__ void __launch_bounds__(256) permute_tokens_kernel(const uint4 *__restrict__ src,
                                                             uint4 *__restrict__ dst, long long G,
                                                             long long A, long long R, int vec) {
    const long long n = G * A * R * vec;
    for (long long x = (long long)blockIdx.x * blockDim.x + threadIdx.x; x < n;
         x += (long long)gridDim.x * blockDim.x) {
        const long long tok = x / vec;
        const int c = (int)(x - tok * vec);
        const long long r = tok % R;
        const long long ga = tok / R;
        const long long a = ga % A;
        const long long g = ga / A;
        dst[((g * R + r) * A + a) * vec + c] = src[x];
    }
}

cudaError_t permute_tokens(const void *src, void *dst, long long G, long long A, long long R,
                           int d, int num_sms, cudaStream_t st) {
    const int vec = d / 8;  // 16-byte vectors per token row
    const long long n = G * A * R * vec;
    if (n == 0) return cudaSuccess;
    long long grid = (n + 255) / 256;
    const long long cap = (long long)num_sms * 16;
    if (grid > cap) grid = cap;
    permute_tokens_kernel<<<(unsigned)grid, 256, 0, st>>>(reinterpret_cast<const uint4 *>(src),
                                                          reinterpret_cast<uint4 *>(dst), G, A, R,
                                                          vec);
    return cudaGetLastError();
}

}  // namespace bsa

namespace {

size_t squad_tensor_bytes(int B, int H, int N, int d) {
    return ((size_t)B * H * N * d * 2 + 255) & ~(size_t)255;
}

}  // namespace

extern "C" size_t sa_squad_workspace_bytes(int B, int H, int N, int d) {
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return 0;
    return kAttnWorkspaceBytes + 4 * squad_tensor_bytes(B, H, N, d);
}

extern "C" sa_status sa_squad_attn_fwd(const void *q, const void *k, const void *v, void *o, int B,
                                       int H, int N, int d, int w, float scale, void *workspace,
                                       size_t workspace_bytes, void *stream) {
    if (!q || !k || !v || !o || !workspace || !shape_ok(B, H, N)) return SA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return SA_ERR_UNSUPPORTED;
    if (w <= 0 || N % w != 0 || isnan(scale)) return SA_ERR_INVALID_ARG;
    const int W = N / w;
    const long long heads_local = (long long)B * H * W, heads_global = (long long)B * H * w;
    if (heads_local > 0x7FFFFFFF || heads_global > 0x7FFFFFFF) return SA_ERR_UNSUPPORTED;
    if (sa_num_blocks(w, 128) > 1024 || sa_num_blocks(W, 128) > 1024) return SA_ERR_UNSUPPORTED;
    if (workspace_bytes < sa_squad_workspace_bytes(B, H, N, d) || !aligned16(workspace))
        return SA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return SA_ERR_INVALID_ARG;
    int dev;
    if (!select_device(o, &dev)) return SA_ERR_INVALID_ARG;
    const cudaStream_t st = (cudaStream_t)stream;
    uint8_t *ws = reinterpret_cast<uint8_t *>(workspace);
    const size_t T = squad_tensor_bytes(B, H, N, d);
    void *counter = ws;
    void *qg = ws + kAttnWorkspaceBytes, *kg = ws + kAttnWorkspaceBytes + T;
    void *yg = ws + kAttnWorkspaceBytes + 2 * T, *og = ws + kAttnWorkspaceBytes + 3 * T;
    const long long G = (long long)B * H;
    const int sms = num_sms(dev);
    // local pass into o (as Y): B*H*W heads of w tokens
    sa_status s = run_attention(q, k, v, nullptr, nullptr, o, 1, (int)heads_local, w, d, 128,
                                scale, counter, stream);
    if (s != SA_OK) return s;
    // regroup Q, K and Y by position within the window
    cudaError_t e = bsa::permute_tokens(q, qg, G, W, w, d, sms, st);
    if (e == cudaSuccess) e = bsa::permute_tokens(k, kg, G, W, w, d, sms, st);
    if (e == cudaSuccess) e = bsa::permute_tokens(o, yg, G, W, w, d, sms, st);
    if (e != cudaSuccess) return SA_ERR_CUDA;
    // global pass: B*H*w sequences of W tokens, values Y.  Short sequences are packed 128 / W to
    // a tile with a block-diagonal mask; longer ones run as B*H*w heads of the dense kernel.
    const long long Ntot = heads_global * W;
    if (W <= 64 && Ntot <= 0x7FFFFFFFLL) {
        CUtensorMap tq, tk, tv;
        if (!make_tmap(&tq, qg, 1, (int)Ntot, d, 128) || !make_tmap(&tk, kg, 1, (int)Ntot, d, 128) ||
            !make_tmap(&tv, yg, 1, (int)Ntot, d, 128))
            return SA_ERR_CUDA;
        e = bsa::attn_group_fwd(tq, tk, tv, og, Ntot, W, d, resolve_scale(scale, d), g_wait_ns, sms,
                                reinterpret_cast<unsigned int *>(counter), st);
        if (e != cudaSuccess) return SA_ERR_CUDA;
    } else {
        s = run_attention(qg, kg, yg, nullptr, nullptr, og, 1, (int)heads_global, W, d, 128, scale,
                          counter, stream);
        if (s != SA_OK) return s;
    }
    // back to token order
    return from_cuda(bsa::permute_tokens(og, o, G, w, W, d, sms, st));
}
