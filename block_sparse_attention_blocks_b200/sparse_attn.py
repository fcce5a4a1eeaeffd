"""Python binding of libbsa (include/sparse_attn.h): argument marshalling only.

Every step of the path runs in the library's sm_100a kernels; this module checks tensor
properties, allocates outputs through PyTorch (which owns device memory and streams here) and
passes raw pointers and the current CUDA stream through ctypes.  For host inputs,
`sparse_attention` also stages the tensors through device memory in chunks of heads, with the
copies on side streams (plumbing only: no arithmetic runs on the host).  There is no fallback:
if the library is missing, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libbsa.so")

if not os.path.exists(_LIB_PATH):
    raise ImportError(
        "libbsa.so is not built; run `python -m block_sparse_attention_blocks_b200.build` "
        "(nvcc for sm_100a) first")

lib = ctypes.CDLL(_LIB_PATH)

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float

lib.sa_pool_blocks.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P]
lib.sa_select_mask_topk_topp.argtypes = [_P, _P, _I, _I, _I, _I, _I, _F, _F, _P, _P, _P, _P]
lib.sa_select_from_logits.argtypes = [_P, _I, _I, _I, _I, _F, _P, _P, _P, _P]
lib.sa_block_scores.argtypes = [_P, _P, _I, _I, _I, _I, _F, _P, _P]
lib.sa_static_mask.argtypes = [_P, _I, _I, _I, _P, _P, _P, _P]
lib.sa_pool_select_topk_topp.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _F, _P, _P,
                                         _P, _P]
_Z = ctypes.c_size_t
lib.sa_squad_workspace_bytes.argtypes = [_I, _I, _I, _I]
lib.sa_squad_workspace_bytes.restype = _Z
lib.sa_squad_attn_fwd.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P, _Z, _P]
lib.sa_kmeans.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _Z, _P]
lib.sa_kmeans_workspace_bytes.argtypes = [_I, _I, _I, _I, _I]
lib.sa_kmeans_workspace_bytes.restype = _Z
lib.sa_cluster_sort.argtypes = [_P, _I, _I, _I, _I, _P, _P, _P, _P, _Z, _P]
lib.sa_cluster_sort_workspace_bytes.argtypes = [_I, _I, _I, _I]
lib.sa_cluster_sort_workspace_bytes.restype = _Z
lib.sa_centroid_topp_workspace_bytes.argtypes = [_I, _I, _I, _I]
lib.sa_centroid_topp_workspace_bytes.restype = _Z
lib.sa_centroid_topp.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _F, _F, _P, _P, _Z, _P]
lib.sa_cluster_attn_workspace_bytes.argtypes = [_I, _I, _I, _I, _I, _I]
lib.sa_cluster_attn_workspace_bytes.restype = _Z
lib.sa_cluster_attn_fwd.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P, _Z,
                                    _P]
lib.sa_svg2_workspace_bytes.argtypes = [_I, _I, _I, _I, _I, _I]
lib.sa_svg2_workspace_bytes.restype = _Z
lib.sa_svg2_attn_fwd.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _F, _P, _P,
                                 _Z, _P]
lib.sa_block_sparse_attn_fwd.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P, _Z, _P]
lib.sa_sparsepr_attn_fwd.argtypes = [_P, _P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _F, _P, _Z,
                                     _P]
lib.sa_sparsepr_workspace_bytes.argtypes = [_I, _I, _I, _I, _I]
lib.sa_sparsepr_workspace_bytes.restype = _Z
lib.sa_dense_attn_fwd.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _F, _P, _Z, _P]
lib.sa_attn_workspace_bytes.argtypes = []
lib.sa_attn_workspace_bytes.restype = _Z
lib.sa_get_error_string.argtypes = [_I]
lib.sa_get_error_string.restype = ctypes.c_char_p
lib.sa_get_device_error.argtypes = [_P]
lib.sa_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
lib.sa_probe_bounded_wait.argtypes = [_P]
lib.sa_num_blocks.argtypes = [_I, _I]
for _f in (lib.sa_pool_blocks, lib.sa_select_mask_topk_topp, lib.sa_select_from_logits,
           lib.sa_pool_select_topk_topp, lib.sa_block_scores, lib.sa_static_mask,
           lib.sa_squad_attn_fwd, lib.sa_kmeans, lib.sa_cluster_sort, lib.sa_centroid_topp,
           lib.sa_cluster_attn_fwd, lib.sa_svg2_attn_fwd,
           lib.sa_block_sparse_attn_fwd, lib.sa_sparsepr_attn_fwd, lib.sa_dense_attn_fwd,
           lib.sa_get_device_error,
           lib.sa_set_wait_limit_ns, lib.sa_probe_bounded_wait, lib.sa_num_blocks):
    _f.restype = _I
lib.sa_get_error_string.restype = ctypes.c_char_p

SA_OK, SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED, SA_ERR_CUDA, SA_ERR_TIMEOUT = range(5)

lib.sa_get_wait_diagnostics.argtypes = [ctypes.c_void_p]
lib.sa_get_wait_diagnostics.restype = _I

# BSA_WAIT_LIMIT_NS bounds every device-side wait of this process (default 2 s)
if os.environ.get("BSA_WAIT_LIMIT_NS"):
    lib.sa_set_wait_limit_ns(int(os.environ["BSA_WAIT_LIMIT_NS"]))


class SAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lib.sa_get_error_string(status).decode()}")


def _check(status: int, where: str):
    if status != SA_OK:
        raise SAError(status, where)


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _ptr(t: torch.Tensor) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype, ndim: int):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dim() != ndim or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {ndim}-d tensor, got shape {tuple(t.shape)}")


def _shape(t: torch.Tensor, name: str, shape):
    """Buffers are passed to the library as bare pointers, so their sizes are checked here."""
    if tuple(t.shape) != tuple(int(s) for s in shape):
        raise ValueError(f"{name} must have shape {tuple(int(s) for s in shape)}, "
                         f"got {tuple(t.shape)}")


def _cuda_device(device) -> torch.device:
    """A CUDA device with its index ("cuda" alone means the current device)."""
    dev = torch.device(device) if device is not None else torch.device("cuda")
    if dev.type == "cuda" and dev.index is None:
        dev = torch.device("cuda", torch.cuda.current_device())
    return dev


def _same_device(ref: torch.Tensor, **tensors):
    for name, t in tensors.items():
        if t.device != ref.device:
            raise ValueError(f"{name} is on {t.device}, expected {ref.device}")


_WORKSPACES = {}


def _workspace(device):
    """A small device workspace per (device, current stream): launches on one stream run in
    order, so they can share it; launches on different streams get their own."""
    st = torch.cuda.current_stream(device)
    key = (device.index, st.cuda_stream)
    ws = _WORKSPACES.get(key)
    if ws is None:
        n = int(lib.sa_attn_workspace_bytes())
        ws = torch.empty(n, dtype=torch.uint8, device=device)
        _WORKSPACES[key] = ws
    return ws


def num_blocks(N: int, bs: int) -> int:
    return (N + bs - 1) // bs


def pool_blocks(q: torch.Tensor, k: torch.Tensor, bs: int, qp=None, kp=None):
    """Mean of Q and K over each block of bs tokens -> (qp, kp) [B, H, nb, d] fp32."""
    _need(q, "q", torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, 4)
    if q.shape != k.shape:
        raise ValueError("q and k must have the same shape")
    B, H, N, d = q.shape
    nb = num_blocks(N, bs)
    qp = qp if qp is not None else torch.empty(B, H, nb, d, device=q.device, dtype=torch.float32)
    kp = kp if kp is not None else torch.empty(B, H, nb, d, device=q.device, dtype=torch.float32)
    _need(qp, "qp", torch.float32, 4)
    _need(kp, "kp", torch.float32, 4)
    _shape(qp, "qp", (B, H, nb, d))
    _shape(kp, "kp", (B, H, nb, d))
    _same_device(q, k=k, qp=qp, kp=kp)
    _check(lib.sa_pool_blocks(_ptr(q), _ptr(k), _ptr(qp), _ptr(kp), B, H, N, d, bs,
                              _stream(q.device)), "sa_pool_blocks")
    return qp, kp


def _sel_outputs(B, H, nb, device, mask, kv_idx, kv_cnt):
    mask = mask if mask is not None else torch.empty(B, H, nb, nb, device=device, dtype=torch.uint8)
    kv_idx = kv_idx if kv_idx is not None else torch.empty(B, H, nb, nb, device=device,
                                                           dtype=torch.int32)
    kv_cnt = kv_cnt if kv_cnt is not None else torch.empty(B, H, nb, device=device,
                                                           dtype=torch.int32)
    _need(mask, "mask", torch.uint8, 4)
    _need(kv_idx, "kv_idx", torch.int32, 4)
    _need(kv_cnt, "kv_cnt", torch.int32, 3)
    _shape(mask, "mask", (B, H, nb, nb))
    _shape(kv_idx, "kv_idx", (B, H, nb, nb))
    _shape(kv_cnt, "kv_cnt", (B, H, nb))
    dev = _cuda_device(device)
    for n, t in (("mask", mask), ("kv_idx", kv_idx), ("kv_cnt", kv_cnt)):
        if t.device != dev:
            raise ValueError(f"{n} is on {t.device}, expected {dev}")
    return mask, kv_idx, kv_cnt


def select_mask_topk_topp(qp, kp, topk: int, topp: float, scale: float | None = None, mask=None,
                          kv_idx=None, kv_cnt=None):
    """Hybrid top-k union top-p block selection -> (mask, kv_idx, kv_cnt)."""
    _need(qp, "qp", torch.float32, 4)
    _need(kp, "kp", torch.float32, 4)
    B, H, nb, d = qp.shape
    _shape(kp, "kp", qp.shape)
    _same_device(qp, kp=kp)
    mask, kv_idx, kv_cnt = _sel_outputs(B, H, nb, qp.device, mask, kv_idx, kv_cnt)
    _check(lib.sa_select_mask_topk_topp(_ptr(qp), _ptr(kp), B, H, nb, d, int(topk), float(topp),
                                        float(scale or 0.0), _ptr(mask), _ptr(kv_idx),
                                        _ptr(kv_cnt), _stream(qp.device)),
           "sa_select_mask_topk_topp")
    return mask, kv_idx, kv_cnt


def pool_select_topk_topp(q, k, bs: int, topk: int, topp: float, scale: float | None = None,
                          qp=None, kp=None, mask=None, kv_idx=None, kv_cnt=None):
    """Pooling and selection in one call -> (qp, kp, mask, kv_idx, kv_cnt), the same values
    pool_blocks + select_mask_topk_topp give."""
    for n, t in (("q", q), ("k", k)):
        _need(t, n, torch.bfloat16, 4)
    B, H, N, d = q.shape
    nb = num_blocks(N, bs)
    qp = qp if qp is not None else torch.empty(B, H, nb, d, dtype=torch.float32, device=q.device)
    kp = kp if kp is not None else torch.empty(B, H, nb, d, dtype=torch.float32, device=q.device)
    _need(qp, "qp", torch.float32, 4)
    _need(kp, "kp", torch.float32, 4)
    _shape(k, "k", q.shape)
    _shape(qp, "qp", (B, H, nb, d))
    _shape(kp, "kp", (B, H, nb, d))
    _same_device(q, k=k, qp=qp, kp=kp)
    mask, kv_idx, kv_cnt = _sel_outputs(B, H, nb, q.device, mask, kv_idx, kv_cnt)
    _check(lib.sa_pool_select_topk_topp(_ptr(q), _ptr(k), _ptr(qp), _ptr(kp), B, H, N, d, bs,
                                        int(topk), float(topp), float(scale or 0.0), _ptr(mask),
                                        _ptr(kv_idx), _ptr(kv_cnt), _stream(q.device)),
           "sa_pool_select_topk_topp")
    return qp, kp, mask, kv_idx, kv_cnt


def block_scores(qp, kp, scale: float | None = None, logits=None):
    """The pooled block scores scale * Qp Kp^T -> [B, H, nb, nb] fp32."""
    _need(qp, "qp", torch.float32, 4)
    _need(kp, "kp", torch.float32, 4)
    B, H, nb, d = qp.shape
    logits = logits if logits is not None else torch.empty(B, H, nb, nb, dtype=torch.float32,
                                                           device=qp.device)
    _need(logits, "logits", torch.float32, 4)
    _shape(kp, "kp", qp.shape)
    _shape(logits, "logits", (B, H, nb, nb))
    _same_device(qp, kp=kp, logits=logits)
    _check(lib.sa_block_scores(_ptr(qp), _ptr(kp), B, H, nb, d, float(scale or 0.0), _ptr(logits),
                               _stream(qp.device)), "sa_block_scores")
    return logits


def static_mask(patterns, B: int, nb: int, device=None, mask=None, kv_idx=None, kv_cnt=None):
    """Static block patterns -> (mask, kv_idx, kv_cnt) for block_sparse_attn_fwd.
    patterns: H descriptors (flags, w, p, s): flags 1 = diagonal band |i - j| <= w, 2 = diagonals
    every p blocks (half-width w), 4 = the first s key blocks; 0 = skipped head."""
    dev = _cuda_device(device)
    pat = torch.as_tensor(patterns, dtype=torch.int32).reshape(-1, 4).to(dev)
    H = pat.shape[0]
    mask, kv_idx, kv_cnt = _sel_outputs(B, H, nb, dev, mask, kv_idx, kv_cnt)
    _check(lib.sa_static_mask(_ptr(pat), B, H, nb, _ptr(mask), _ptr(kv_idx), _ptr(kv_cnt),
                              _stream(dev)), "sa_static_mask")
    return mask, kv_idx, kv_cnt


def select_from_logits(logits, topk: int, topp: float, mask=None, kv_idx=None, kv_cnt=None):
    """Selection from given block scores [B, H, nb, nb] fp32 -> (mask, kv_idx, kv_cnt)."""
    _need(logits, "logits", torch.float32, 4)
    B, H, nb, _ = logits.shape
    _shape(logits, "logits", (B, H, nb, nb))
    mask, kv_idx, kv_cnt = _sel_outputs(B, H, nb, logits.device, mask, kv_idx, kv_cnt)
    _check(lib.sa_select_from_logits(_ptr(logits), B, H, nb, int(topk), float(topp), _ptr(mask),
                                     _ptr(kv_idx), _ptr(kv_cnt), _stream(logits.device)),
           "sa_select_from_logits")
    return mask, kv_idx, kv_cnt


def block_sparse_attn_fwd(q, k, v, kv_idx, kv_cnt, bs: int, scale: float | None = None, o=None):
    """Attention over the kept key blocks listed in (kv_idx, kv_cnt) -> O [B, H, N, d] bf16."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, n, torch.bfloat16, 4)
    _need(kv_idx, "kv_idx", torch.int32, 4)
    _need(kv_cnt, "kv_cnt", torch.int32, 3)
    B, H, N, d = q.shape
    nb = num_blocks(N, bs)
    o = o if o is not None else torch.empty_like(q)
    _need(o, "o", torch.bfloat16, 4)
    for n, t in (("k", k), ("v", v), ("o", o)):
        _shape(t, n, q.shape)
    _shape(kv_idx, "kv_idx", (B, H, nb, nb))
    _shape(kv_cnt, "kv_cnt", (B, H, nb))
    _same_device(q, k=k, v=v, o=o, kv_idx=kv_idx, kv_cnt=kv_cnt)
    ws = _workspace(q.device)
    _check(lib.sa_block_sparse_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(kv_idx), _ptr(kv_cnt),
                                        _ptr(o), B, H, N, d, bs, float(scale or 0.0), _ptr(ws),
                                        ws.numel(), _stream(q.device)), "sa_block_sparse_attn_fwd")
    return o


def sparsepr_attn_fwd(q, k, v, kv_idx, kv_cnt, probes, bs: int, scale: float | None = None,
                      o=None, workspace=None):
    """Block-sparse attention over (kv_idx, kv_cnt) corrected by the probe fit of SparsePR with the
    exact outputs of the probe rows probes [B, H, m] int32 -> O [B, H, N, d] bf16."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, n, torch.bfloat16, 4)
    _need(kv_idx, "kv_idx", torch.int32, 4)
    _need(kv_cnt, "kv_cnt", torch.int32, 3)
    _need(probes, "probes", torch.int32, 3)
    B, H, N, d = q.shape
    nb = num_blocks(N, bs)
    m = probes.shape[2]
    o = o if o is not None else torch.empty_like(q)
    _need(o, "o", torch.bfloat16, 4)
    for n, t in (("k", k), ("v", v), ("o", o)):
        _shape(t, n, q.shape)
    _shape(kv_idx, "kv_idx", (B, H, nb, nb))
    _shape(kv_cnt, "kv_cnt", (B, H, nb))
    _shape(probes, "probes", (B, H, m))
    nbytes = int(lib.sa_sparsepr_workspace_bytes(B, H, N, d, m))
    if nbytes == 0:
        raise SAError(SA_ERR_INVALID_ARG, "sa_sparsepr_workspace_bytes")
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    _need(workspace, "workspace", torch.uint8, 1)
    if workspace.numel() < nbytes:
        raise ValueError(f"workspace must hold {nbytes} bytes, got {workspace.numel()}")
    _same_device(q, k=k, v=v, o=o, kv_idx=kv_idx, kv_cnt=kv_cnt, probes=probes,
                 workspace=workspace)
    _check(lib.sa_sparsepr_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(kv_idx), _ptr(kv_cnt),
                                    _ptr(probes), m, _ptr(o), B, H, N, d, bs,
                                    float(scale or 0.0), _ptr(workspace), workspace.numel(),
                                    _stream(q.device)), "sa_sparsepr_attn_fwd")
    return o


def dense_attn_fwd(q, k, v, scale: float | None = None, o=None):
    """Dense softmax attention (the 0 %-sparsity control) -> O [B, H, N, d] bf16."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, n, torch.bfloat16, 4)
    B, H, N, d = q.shape
    o = o if o is not None else torch.empty_like(q)
    _need(o, "o", torch.bfloat16, 4)
    for n, t in (("k", k), ("v", v), ("o", o)):
        _shape(t, n, q.shape)
    _same_device(q, k=k, v=v, o=o)
    ws = _workspace(q.device)
    _check(lib.sa_dense_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, N, d,
                                 float(scale or 0.0), _ptr(ws), ws.numel(), _stream(q.device)),
           "sa_dense_attn_fwd")
    return o


def squad_attn_fwd(q, k, v, w: int, scale: float | None = None, o=None):
    """SQuad attention: softmax attention within windows of w tokens, then across windows at
    each position with the local outputs as values -> O [B, H, N, d] bf16 (N a multiple of w)."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, n, torch.bfloat16, 4)
    B, H, N, d = q.shape
    o = o if o is not None else torch.empty_like(q)
    _need(o, "o", torch.bfloat16, 4)
    for n, t in (("k", k), ("v", v), ("o", o)):
        _shape(t, n, q.shape)
    _same_device(q, k=k, v=v, o=o)
    nbytes = int(lib.sa_squad_workspace_bytes(B, H, N, d))
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    _check(lib.sa_squad_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, N, d, int(w),
                                 float(scale or 0.0), _ptr(ws), ws.numel(), _stream(q.device)),
           "sa_squad_attn_fwd")
    return o


def kmeans(x, cent, iters: int):
    """Lloyd k-means of the token rows of every head, from the centroids `cent` [B, H, C, d]
    fp32, which are overwritten with the result (SVG2 section A, warm-started from a cache as in
    section C).  x: [B, H, N, d] bf16.  Returns (assign [B, H, N], perm [B, H, N], cstart
    [B, H, C], csize [B, H, C]) int32: the final assignment, and the stable order of the tokens
    by cluster (cluster c is perm[cstart[c] : cstart[c] + csize[c]])."""
    _need(x, "x", torch.bfloat16, 4)
    _need(cent, "cent", torch.float32, 4)
    B, H, N, d = x.shape
    C = cent.shape[2]
    _shape(cent, "cent", (B, H, C, d))
    _same_device(x, cent=cent)
    assign = torch.empty(B, H, N, device=x.device, dtype=torch.int32)
    perm = torch.empty_like(assign)
    cstart = torch.empty(B, H, C, device=x.device, dtype=torch.int32)
    csize = torch.empty_like(cstart)
    nbytes = int(lib.sa_kmeans_workspace_bytes(B, H, N, C, d))
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=x.device)
    _check(lib.sa_kmeans(_ptr(x), _ptr(cent), _ptr(assign), _ptr(perm), _ptr(cstart), _ptr(csize),
                         B, H, N, d, C, int(iters), _ptr(ws), ws.numel(), _stream(x.device)),
           "sa_kmeans")
    return assign, perm, cstart, csize


def cluster_sort(assign, C: int):
    """Stable order of the tokens by cluster id: (perm [B, H, N], cstart [B, H, C], csize
    [B, H, C]) int32 from assign [B, H, N] int32 ids in [0, C)."""
    _need(assign, "assign", torch.int32, 3)
    B, H, N = assign.shape
    perm = torch.empty_like(assign)
    cstart = torch.empty(B, H, C, device=assign.device, dtype=torch.int32)
    csize = torch.empty_like(cstart)
    nbytes = int(lib.sa_cluster_sort_workspace_bytes(B, H, N, int(C)))
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=assign.device)
    _check(lib.sa_cluster_sort(_ptr(assign), B, H, N, int(C), _ptr(perm), _ptr(cstart),
                               _ptr(csize), _ptr(ws), ws.numel(), _stream(assign.device)),
           "sa_cluster_sort")
    return perm, cstart, csize


def centroid_topp(cq, ck, size_k, topp: float, scale: float | None = None):
    """Centroid top-p (SVG2 section B): sel [B, H, Cq, Ck] uint8, the key clusters each query
    cluster takes.  cq [B, H, Cq, d], ck [B, H, Ck, d] fp32 centroids; size_k [B, H, Ck] int32
    key cluster sizes."""
    _need(cq, "cq", torch.float32, 4)
    _need(ck, "ck", torch.float32, 4)
    _need(size_k, "size_k", torch.int32, 3)
    B, H, Cq, d = cq.shape
    Ck = ck.shape[2]
    _shape(ck, "ck", (B, H, Ck, d))
    _shape(size_k, "size_k", (B, H, Ck))
    _same_device(cq, ck=ck, size_k=size_k)
    sel = torch.empty(B, H, Cq, Ck, device=cq.device, dtype=torch.uint8)
    nbytes = int(lib.sa_centroid_topp_workspace_bytes(B, H, Cq, Ck))
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=cq.device)
    _check(lib.sa_centroid_topp(_ptr(cq), _ptr(ck), _ptr(size_k), B, H, Cq, Ck, d, float(topp),
                                float(scale or 0.0), _ptr(sel), _ptr(ws), ws.numel(),
                                _stream(cq.device)), "sa_centroid_topp")
    return sel


def cluster_attn_fwd(q, k, v, assign_q, assign_k, sel, scale: float | None = None, o=None):
    """Attention of each query token over the keys of the key clusters its query cluster
    selected -> O [B, H, N, d] bf16.  assign_q, assign_k [B, H, N] int32 cluster ids; sel
    [B, H, Cq, Ck] uint8."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, n, torch.bfloat16, 4)
    _need(assign_q, "assign_q", torch.int32, 3)
    _need(assign_k, "assign_k", torch.int32, 3)
    _need(sel, "sel", torch.uint8, 4)
    B, H, N, d = q.shape
    Cq, Ck = sel.shape[2], sel.shape[3]
    o = o if o is not None else torch.empty_like(q)
    _need(o, "o", torch.bfloat16, 4)
    for n, t in (("k", k), ("v", v), ("o", o)):
        _shape(t, n, q.shape)
    _shape(assign_q, "assign_q", (B, H, N))
    _shape(assign_k, "assign_k", (B, H, N))
    _shape(sel, "sel", (B, H, Cq, Ck))
    _same_device(q, k=k, v=v, o=o, assign_q=assign_q, assign_k=assign_k, sel=sel)
    nbytes = int(lib.sa_cluster_attn_workspace_bytes(B, H, N, d, Cq, Ck))
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    _check(lib.sa_cluster_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(assign_q),
                                   _ptr(assign_k), _ptr(sel), B, H, N, d, Cq, Ck,
                                   float(scale or 0.0), _ptr(ws), ws.numel(), _stream(q.device)),
           "sa_cluster_attn_fwd")
    return o


def svg2_attn_fwd(q, k, v, cent_q, cent_k, iters: int, topp: float, scale: float | None = None,
                  o=None, sel=None, workspace=None):
    """The semantic-aware permutation path of SVG2: k-means of Q and of K from the centroid
    cache cent_q [B, H, Cq, d] / cent_k [B, H, Ck, d] fp32 (updated in place), centroid top-p,
    attention over the selected clusters.  Returns (O [B, H, N, d] bf16, sel [B, H, Cq, Ck])."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, n, torch.bfloat16, 4)
    _need(cent_q, "cent_q", torch.float32, 4)
    _need(cent_k, "cent_k", torch.float32, 4)
    B, H, N, d = q.shape
    Cq, Ck = cent_q.shape[2], cent_k.shape[2]
    o = o if o is not None else torch.empty_like(q)
    sel = sel if sel is not None else torch.empty(B, H, Cq, Ck, device=q.device, dtype=torch.uint8)
    _need(o, "o", torch.bfloat16, 4)
    _need(sel, "sel", torch.uint8, 4)
    for n, t in (("k", k), ("v", v), ("o", o)):
        _shape(t, n, q.shape)
    _shape(cent_q, "cent_q", (B, H, Cq, d))
    _shape(cent_k, "cent_k", (B, H, Ck, d))
    _shape(sel, "sel", (B, H, Cq, Ck))
    _same_device(q, k=k, v=v, o=o, cent_q=cent_q, cent_k=cent_k, sel=sel)
    nbytes = int(lib.sa_svg2_workspace_bytes(B, H, N, d, Cq, Ck))
    if (workspace is None or workspace.numel() < nbytes or workspace.dtype != torch.uint8
            or workspace.device != q.device):
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    _check(lib.sa_svg2_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(cent_q), _ptr(cent_k),
                                B, H, N, d, Cq, Ck, int(iters), float(topp), float(scale or 0.0),
                                _ptr(sel), _ptr(workspace), workspace.numel(), _stream(q.device)),
           "sa_svg2_attn_fwd")
    return o, sel


def _host_pipeline(q, k, v, bs, topk, topp, scale, dev, out, chunks):
    """Host inputs: the heads go through in chunks so that copies and kernels overlap.  Chunk c
    is copied in on one stream, pooled, selected and attended on the current stream, and copied
    out on a third; the next chunk's copy in and the previous chunk's copy out run meanwhile."""
    B, H, N, d = q.shape
    BH = B * H
    nb = num_blocks(N, bs)
    qf, kf, vf = (t.reshape(BH, N, d) for t in (q, k, v))
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=q.is_pinned())
    of = out.reshape(BH, N, d)
    qd, kd, vd = (torch.empty((BH, N, d), dtype=torch.bfloat16, device=dev) for _ in range(3))
    od = torch.empty((BH, N, d), dtype=torch.bfloat16, device=dev)
    qp = torch.empty((1, BH, nb, d), dtype=torch.float32, device=dev)
    kp = torch.empty_like(qp)
    mask = torch.empty((1, BH, nb, nb), dtype=torch.uint8, device=dev)
    kv_idx = torch.empty((1, BH, nb, nb), dtype=torch.int32, device=dev)
    kv_cnt = torch.empty((1, BH, nb), dtype=torch.int32, device=dev)
    main = torch.cuda.current_stream(dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    s_in.wait_stream(main)
    s_out.wait_stream(main)
    per = -(-BH // chunks)
    for h0 in range(0, BH, per):
        h1 = min(BH, h0 + per)
        with torch.cuda.stream(s_in):
            for dst, src in ((qd, qf), (kd, kf), (vd, vf)):
                dst[h0:h1].copy_(src[h0:h1], non_blocking=True)
            ev_in = torch.cuda.Event()
            ev_in.record(s_in)
        main.wait_event(ev_in)
        sl = lambda t: t[:, h0:h1] if t.dim() == 4 else t[h0:h1].unsqueeze(0)
        pool_select_topk_topp(sl(qd), sl(kd), bs, topk, topp, scale, qp=sl(qp), kp=sl(kp),
                              mask=sl(mask), kv_idx=sl(kv_idx), kv_cnt=kv_cnt[:, h0:h1])
        block_sparse_attn_fwd(sl(qd), sl(kd), sl(vd), sl(kv_idx), kv_cnt[:, h0:h1], bs, scale,
                              o=sl(od))
        ev_done = torch.cuda.Event()
        ev_done.record(main)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done)
            of[h0:h1].copy_(od[h0:h1], non_blocking=True)
    main.wait_stream(s_out)
    # the device buffers stay in use by the side streams until their copies end
    for t in (qd, kd, vd, od):
        t.record_stream(s_in)
        t.record_stream(s_out)
    main.synchronize()  # O is on the host when the call returns
    sel = (mask.reshape(B, H, nb, nb), kv_idx.reshape(B, H, nb, nb), kv_cnt.reshape(B, H, nb))
    return out, sel


def sparse_attention(q, k, v, bs: int, topk: int, topp: float, scale: float | None = None,
                     device=None, return_selection: bool = False, out=None, chunks: int = 8):
    """The whole path: pool -> select -> block-sparse attention.

    q, k, v may live on the host (ideally pinned) or on a CUDA device.  Device inputs return a
    device O.  Host inputs are processed in `chunks` groups of heads on `device` (default: the
    current CUDA device), with the copies of one group overlapping the kernels of another; O is
    written to `out` (a host tensor of q's shape, ideally pinned) or to a new host tensor, and is
    complete when the call returns.
    """
    if not q.is_cuda:
        for n, t in (("q", q), ("k", k), ("v", v)):
            if t.dtype != torch.bfloat16 or t.dim() != 4 or not t.is_contiguous():
                raise TypeError(f"{n}: expected a contiguous 4-D bfloat16 tensor")
            if t.shape != q.shape or t.is_cuda:
                raise ValueError(f"{n}: expected a host tensor of shape {tuple(q.shape)}")
        if out is not None and (out.shape != q.shape or out.dtype != torch.bfloat16
                                or out.is_cuda or not out.is_contiguous()):
            raise ValueError(f"out: expected a contiguous host bfloat16 tensor of shape "
                             f"{tuple(q.shape)}")
        dev = _cuda_device(device)
        o, sel = _host_pipeline(q, k, v, bs, topk, topp, scale, dev, out, max(1, int(chunks)))
        return (o, sel) if return_selection else o
    _, _, mask, kv_idx, kv_cnt = pool_select_topk_topp(q, k, bs, topk, topp, scale)
    o = block_sparse_attn_fwd(q, k, v, kv_idx, kv_cnt, bs, scale, o=out)
    if return_selection:
        return o, (mask, kv_idx, kv_cnt)
    return o


def device_error(stream=None) -> int:
    """Synchronise and read/clear the library's device error word (an sa_status code)."""
    s = ctypes.c_void_p(stream) if stream is not None else _stream(None)
    return int(lib.sa_get_device_error(s))


def wait_diagnostics() -> dict:
    """Where the first device-side wait that ran out gave up (then cleared); {} if none did."""
    rec = ctypes.c_uint64(0)
    _check(lib.sa_get_wait_diagnostics(ctypes.byref(rec)), "sa_get_wait_diagnostics")
    r = rec.value
    if r == 0:
        return {}
    return {"site": r >> 56, "cta": (r >> 32) & 0xFFFFFF, "step": (r >> 16) & 0xFFFF,
            "unit": r & 0xFFFF}


def exp2_poly(x: torch.Tensor) -> torch.Tensor:
    """The softmax's FMA-pipe 2^x evaluated on a CUDA fp32 tensor (test hook)."""
    _need(x, "x", torch.float32, x.dim())
    y = torch.empty_like(x)
    lib.sa_test_exp2_poly.argtypes = [_P, _P, _I, _P]
    lib.sa_test_exp2_poly.restype = _I
    _check(lib.sa_test_exp2_poly(_ptr(x), _ptr(y), x.numel(), _stream(x.device)),
           "sa_test_exp2_poly")
    return y


def set_wait_limit_ns(ns: int):
    _check(lib.sa_set_wait_limit_ns(int(ns)), "sa_set_wait_limit_ns")


def probe_bounded_wait():
    _check(lib.sa_probe_bounded_wait(_stream(None)), "sa_probe_bounded_wait")
