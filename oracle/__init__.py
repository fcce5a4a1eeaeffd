"""fp64 CPU oracle for block-sparse attention with hybrid top-k + top-p block masks.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and the benchmark's
CPU-baseline leg may import this module.  The CUDA path never imports it, and it never imports
the CUDA path: the two share nothing but the seeded input generator.

The arithmetic lives in ``oracle.c`` (plain fp64 loops, OpenMP over rows).  This module only
compiles it, loads it with ctypes and marshals numpy arrays; each of those functions cites the
passage it follows in its C definition.  The one exception is the probe-fitted correction at the
end of this file, whose steps are numpy library calls (SVD, least squares) written out here.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (plain -O2, no fast-math, portable ISA)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB)
    P = ctypes.c_void_p
    I = ctypes.c_int64
    D = ctypes.c_double
    lib.or_num_threads.restype = ctypes.c_int
    lib.or_pool_blocks.argtypes = [P, I, I, I, I, P]
    lib.or_block_probs.argtypes = [P, P, I, I, I, I, D, P]
    lib.or_block_logits.argtypes = [P, P, I, I, I, I, D, P]
    lib.or_softmax_rows.argtypes = [P, I, I, P]
    lib.or_select_rows.argtypes = [P, I, I, I, D, P, P, P, P, P, P, P, P]
    lib.or_masked_attention.argtypes = [P, P, P, I, I, I, P, D, P, P, I, P]
    lib.or_dense_attention.argtypes = [P, P, P, I, I, D, P, P, I, P]
    lib.or_static_mask.argtypes = [P, I, I, P]
    lib.or_squad_attention.argtypes = [P, P, P, I, I, I, I, D, P]
    lib.or_kmeans.argtypes = [P, I, I, I, I, P, P]
    lib.or_centroid_topp.argtypes = [P, P, P, I, I, I, D, D, P]
    lib.or_cluster_attention.argtypes = [P, P, P, I, I, P, P, P, I, D, P]
    for f in (lib.or_pool_blocks, lib.or_block_probs, lib.or_block_logits, lib.or_softmax_rows,
              lib.or_select_rows,
              lib.or_masked_attention, lib.or_dense_attention, lib.or_static_mask,
              lib.or_squad_attention, lib.or_kmeans, lib.or_centroid_topp,
              lib.or_cluster_attention):
        f.restype = None
    _lib = lib
    return lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _bits(x: np.ndarray) -> np.ndarray:
    """bf16 tensors travel as their uint16 bit patterns."""
    x = np.ascontiguousarray(x)
    if x.dtype != np.uint16:
        raise TypeError("bf16 inputs must be given as uint16 bit patterns, got %s" % x.dtype)
    return x


def num_threads() -> int:
    return int(_load().or_num_threads())


def pool_blocks(x_bits: np.ndarray, bs: int) -> np.ndarray:
    """Mean of each block of bs tokens (tail block: mean of its valid tokens).

    x_bits: [..., N, d] uint16 (bf16 bits).  Returns [..., nb, d] float64.
    """
    x = _bits(x_bits)
    *lead, N, d = x.shape
    BH = int(np.prod(lead)) if lead else 1
    nb = (N + bs - 1) // bs
    out = np.empty((BH, nb, d), np.float64)
    _load().or_pool_blocks(_ptr(x), BH, N, d, bs, _ptr(out))
    return out.reshape(*lead, nb, d)


def block_probs(qp: np.ndarray, kp: np.ndarray, scale: float) -> np.ndarray:
    """Row softmax of the pooled block scores Qp Kp^T * scale.  qp: [..., nbq, d]."""
    qp = np.ascontiguousarray(qp, np.float64)
    kp = np.ascontiguousarray(kp, np.float64)
    *lead, nbq, d = qp.shape
    nbk = kp.shape[-2]
    BH = int(np.prod(lead)) if lead else 1
    out = np.empty((BH, nbq, nbk), np.float64)
    _load().or_block_probs(_ptr(qp), _ptr(kp), BH, nbq, nbk, d, float(scale), _ptr(out))
    return out.reshape(*lead, nbq, nbk)


def block_logits(qp: np.ndarray, kp: np.ndarray, scale: float) -> np.ndarray:
    """The pooled block scores Qp Kp^T * scale (the logits of block_probs)."""
    qp = np.ascontiguousarray(qp, np.float64)
    kp = np.ascontiguousarray(kp, np.float64)
    *lead, nbq, d = qp.shape
    nbk = kp.shape[-2]
    BH = int(np.prod(lead)) if lead else 1
    out = np.empty((BH, nbq, nbk), np.float64)
    _load().or_block_logits(_ptr(qp), _ptr(kp), BH, nbq, nbk, d, float(scale), _ptr(out))
    return out.reshape(*lead, nbq, nbk)


def softmax_rows(logits: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(logits, np.float64)
    n = x.shape[-1]
    rows = x.size // n if n else 0
    out = np.empty_like(x)
    _load().or_softmax_rows(_ptr(x), rows, n, _ptr(out))
    return out


class Selection:
    """Per-row result of the hybrid selection, with the diagnostics the parity rule needs."""

    def __init__(self, mask, cnt, tau_k, tau_p, m_p, cum_lo, cum_hi, rank, prob, topk, topp):
        self.mask, self.cnt = mask, cnt
        self.tau_k, self.tau_p, self.m_p = tau_k, tau_p, m_p
        self.cum_lo, self.cum_hi, self.rank = cum_lo, cum_hi, rank
        self.prob, self.topk, self.topp = prob, topk, topp
        self.logit = None  # block scores, when the selection was made from scores


def select_from_probs(prob: np.ndarray, topk: int, topp: float) -> Selection:
    """Hybrid top-k union top-p selection applied row by row to block probabilities."""
    P = np.ascontiguousarray(prob, np.float64)
    *lead, nb = P.shape
    rows = int(np.prod(lead)) if lead else 1
    mask = np.empty((rows, nb), np.uint8)
    cnt = np.empty(rows, np.int32)
    tau_k = np.empty(rows, np.float64)
    tau_p = np.empty(rows, np.float64)
    m_p = np.empty(rows, np.int32)
    lo = np.empty(rows, np.float64)
    hi = np.empty(rows, np.float64)
    rank = np.empty((rows, nb), np.int32)
    _load().or_select_rows(_ptr(P), rows, nb, int(topk), float(topp), _ptr(mask), _ptr(cnt),
                           _ptr(tau_k), _ptr(tau_p), _ptr(m_p), _ptr(lo), _ptr(hi), _ptr(rank))
    shp = tuple(lead)
    return Selection(mask.reshape(*shp, nb), cnt.reshape(shp), tau_k.reshape(shp),
                     tau_p.reshape(shp), m_p.reshape(shp), lo.reshape(shp), hi.reshape(shp),
                     rank.reshape(*shp, nb), P, topk, topp)


def select_from_logits(logits: np.ndarray, topk: int, topp: float) -> Selection:
    sel = select_from_probs(softmax_rows(logits), topk, topp)
    sel.logit = np.ascontiguousarray(logits, np.float64)
    return sel


def select(qp: np.ndarray, kp: np.ndarray, topk: int, topp: float, scale: float) -> Selection:
    """Block scores, row softmax and hybrid selection from pooled Q and K."""
    sel = select_from_probs(block_probs(qp, kp, scale), topk, topp)
    sel.logit = block_logits(qp, kp, scale)
    return sel


def static_mask(patterns, B: int, nb: int) -> np.ndarray:
    """Static block pattern mask [B, H, nb, nb] uint8 from per-head descriptors
    patterns[h] = (flags, w, p, s): diagonal band, multi-diagonal, vertical stripe (see oracle.c)."""
    pat = np.ascontiguousarray(np.asarray(patterns, np.int32).reshape(-1, 4))
    H = pat.shape[0]
    out = np.empty((H, nb, nb), np.uint8)
    _load().or_static_mask(_ptr(pat), H, nb, _ptr(out))
    return np.broadcast_to(out, (B, H, nb, nb)).copy()


def squad_attention(q_bits, k_bits, v_bits, w: int, scale: float) -> np.ndarray:
    """SQuad attention (local pass in windows of w tokens, global pass across windows at each
    position with the local outputs as values).  q/k/v_bits: [BH, N, d] uint16, N a multiple of
    w.  Returns [BH, N, d] float64."""
    q, k, v = _bits(q_bits), _bits(k_bits), _bits(v_bits)
    BH, N, d = q.shape
    if N % w:
        raise ValueError("N must be a multiple of w")
    out = np.empty((BH, N, d), np.float64)
    _load().or_squad_attention(_ptr(q), _ptr(k), _ptr(v), BH, N, d, w, float(scale), _ptr(out))
    return out


def _bf16_values(bits) -> np.ndarray:
    """The values of bf16 bit patterns (the top half of an IEEE binary32), as float64."""
    b = np.ascontiguousarray(_bits(bits)).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def kmeans(x: np.ndarray, init: np.ndarray, iters: int):
    """Lloyd k-means of the rows of x [n, d] from the centroids init [C, d] (SVG2 method A/C).
    Returns (centroids [C, d] float64, assignment [n] int32)."""
    x = np.ascontiguousarray(x, np.float64)
    cent = np.ascontiguousarray(init, np.float64).copy()
    n, d = x.shape
    assign = np.empty(n, np.int32)
    _load().or_kmeans(_ptr(x), n, d, cent.shape[0], int(iters), _ptr(cent), _ptr(assign))
    return cent, assign


def centroid_topp(cq: np.ndarray, ck: np.ndarray, size_k: np.ndarray, scale: float,
                  p: float) -> np.ndarray:
    """SVG2 centroid top-p (method B): sel [Cq, Ck] 0/1, key clusters taken by estimated score
    size * exp(scale cq . ck) normalised per query cluster, until the cumulative score reaches p."""
    cq = np.ascontiguousarray(cq, np.float64)
    ck = np.ascontiguousarray(ck, np.float64)
    size = np.ascontiguousarray(size_k, np.int64)
    Cq, d = cq.shape
    Ck = ck.shape[0]
    sel = np.empty((Cq, Ck), np.uint8)
    _load().or_centroid_topp(_ptr(cq), _ptr(ck), _ptr(size), Cq, Ck, d, float(scale), float(p),
                             _ptr(sel))
    return sel


def cluster_attention(q_bits, k_bits, v_bits, assign_q, assign_k, sel, scale: float) -> np.ndarray:
    """Attention of each query token over the keys of the clusters its cluster selected (one
    head; q/k/v_bits [n, d] uint16).  Returns [n, d] float64."""
    q, k, v = _bits(q_bits), _bits(k_bits), _bits(v_bits)
    n, d = q.shape
    aq = np.ascontiguousarray(assign_q, np.int32)
    ak = np.ascontiguousarray(assign_k, np.int32)
    s = np.ascontiguousarray(sel, np.uint8)
    out = np.empty((n, d), np.float64)
    _load().or_cluster_attention(_ptr(q), _ptr(k), _ptr(v), n, d, _ptr(aq), _ptr(ak), _ptr(s),
                                 s.shape[1], float(scale), _ptr(out))
    return out


def svg2_attention(q_bits, k_bits, v_bits, init_q, init_k, iters: int, p: float, scale: float):
    """The SVG2 path for one head: k-means of Q and of K (from the given, e.g. cached,
    centroids), centroid top-p, attention over the selected clusters.  Returns (out [n, d],
    assign_q, assign_k, cent_q, cent_k, sel)."""
    qd, kd = _bf16_values(q_bits), _bf16_values(k_bits)
    cent_q, aq = kmeans(qd, init_q, iters)
    cent_k, ak = kmeans(kd, init_k, iters)
    size_k = np.bincount(ak, minlength=cent_k.shape[0]).astype(np.int64)
    sel = centroid_topp(cent_q, cent_k, size_k, scale, p)
    out = cluster_attention(q_bits, k_bits, v_bits, aq, ak, sel, scale)
    return out, aq, ak, cent_q, cent_k, sel


def masked_attention(q_bits, k_bits, v_bits, mask, bs: int, scale: float, sel=None):
    """Attention restricted to the kept key blocks of each query block.

    q/k/v_bits: [BH, N, d] uint16; mask: [BH, nb, nb] 0/1.
    sel: optional list of (bh, i) query blocks; default all.  Returns [nsel, bs, d] float64
    (rows at or beyond N are zero) and the selection arrays.
    """
    q, k, v = _bits(q_bits), _bits(k_bits), _bits(v_bits)
    BH, N, d = q.shape
    nb = (N + bs - 1) // bs
    m = np.ascontiguousarray(mask, np.uint8).reshape(BH, nb, nb)
    if sel is None:
        sel = [(bh, i) for bh in range(BH) for i in range(nb)]
    sel = np.asarray(sel, np.int64).reshape(-1, 2)
    sb = np.ascontiguousarray(sel[:, 0])
    si = np.ascontiguousarray(sel[:, 1])
    out = np.zeros((len(sel), bs, d), np.float64)
    _load().or_masked_attention(_ptr(q), _ptr(k), _ptr(v), N, d, bs, _ptr(m), float(scale),
                                _ptr(sb), _ptr(si), len(sel), _ptr(out))
    return out


def dense_attention(q_bits, k_bits, v_bits, scale: float, rows=None):
    """Full softmax attention.  rows: optional list of (bh, t); default every row.

    Returns [nrows, d] float64.
    """
    q, k, v = _bits(q_bits), _bits(k_bits), _bits(v_bits)
    BH, N, d = q.shape
    if rows is None:
        rows = [(bh, t) for bh in range(BH) for t in range(N)]
    rows = np.asarray(rows, np.int64).reshape(-1, 2)
    sb = np.ascontiguousarray(rows[:, 0])
    st = np.ascontiguousarray(rows[:, 1])
    out = np.zeros((len(rows), d), np.float64)
    _load().or_dense_attention(_ptr(q), _ptr(k), _ptr(v), N, d, float(scale), _ptr(sb), _ptr(st),
                               len(rows), _ptr(out))
    return out


# ---------------------------------------------------------------------------------------------
# Probe-fitted residual reconstruction (page "Partition the Support, Reconstruct the Residual:
# Training-Free Sparse Attention for Video Generation and World Models", the abstract and the
# summary's section 3).  The page describes this step in a single sentence: per call, a handful
# of rows computed exactly fix an affine correction of the sparse output, limited to the
# directions their residuals occupy.  The steps below are the plainest reading of it; their
# library steps are numpy's SVD and least squares.
# ---------------------------------------------------------------------------------------------
def probe_fit_correction(o_sparse, probes, exact, rtol: float = 1e-9, rank=None):
    """One head of one call.  o_sparse [n, d]: the sparse attention output; probes [m]: probe
    query rows; exact [m, d]: their exact (dense) attention outputs.

      R  = exact - o_sparse[probes]                the probe residuals
      Bs = orthonormal basis [d, r] of the residual subspace: the right singular vectors
           of R whose singular value exceeds rtol times the largest (its numerical row space),
           or only the leading `rank` of them when rank is given
      A  = argmin || [o_sparse[probes], 1] A - R Bs ||   over A [(d + 1), r]; the minimum-norm
           solution when the probes leave it underdetermined
      o  = o_sparse + [o_sparse, 1] A Bs^T         applied to every row

    With the whole numerical row space (rank None) the correction equals the minimum-norm
    least-squares fit of the residuals themselves, [o, 1] X^+ R with X = [o_sparse[probes], 1]:
    that fit is already a combination of the rows of R.  A smaller rank confines it further.

    Returns (o [n, d], Bs [d, r], A [d + 1, r]), float64."""
    Os = np.asarray(o_sparse, np.float64)
    n, d = Os.shape
    P = np.asarray(probes, np.int64).reshape(-1)
    E = np.asarray(exact, np.float64).reshape(len(P), d)
    R = E - Os[P]
    if len(P) == 0 or not np.any(R):
        return Os.copy(), np.zeros((d, 0)), np.zeros((d + 1, 0))
    _, s, vt = np.linalg.svd(R, full_matrices=False)
    r = int(np.count_nonzero(s > rtol * s[0]))
    if rank is not None:
        r = min(r, int(rank))
    Bs = vt[:r].T
    X = np.hstack([Os[P], np.ones((len(P), 1))])
    A = np.linalg.lstsq(X, R @ Bs, rcond=None)[0]
    return Os + np.hstack([Os, np.ones((n, 1))]) @ A @ Bs.T, Bs, A


def sparsepr_attention(q_bits, k_bits, v_bits, mask, bs: int, scale: float, probes):
    """Block-sparse attention of one head (q/k/v_bits [N, d], mask [nb, nb]) followed by the
    probe-fitted correction with the exact outputs of the given probe rows.  Returns
    (o_corrected [N, d], o_sparse [N, d])."""
    q, k, v = _bits(q_bits), _bits(k_bits), _bits(v_bits)
    N, d = q.shape
    nb = (N + bs - 1) // bs
    blocks = masked_attention(q[None], k[None], v[None], np.asarray(mask).reshape(1, nb, nb), bs,
                              scale)
    o_sparse = blocks.reshape(nb * bs, d)[:N]
    P = np.asarray(probes, np.int64).reshape(-1)
    exact = dense_attention(q[None], k[None], v[None], scale, rows=[(0, int(t)) for t in P])
    o, _, _ = probe_fit_correction(o_sparse, P, exact)
    return o, o_sparse
