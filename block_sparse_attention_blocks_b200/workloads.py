"""Seeded synthetic Q/K/V shaped like video-DiT self-attention.

This module only makes inputs.  It holds none of the attention or selection arithmetic, imports
nothing else from this package, and is shared by the CUDA path's tests and benchmark and by the
CPU oracle, which receive exactly the same bf16 bytes.

Tokens of a video latent are laid out in raster order n = t*(Y*X) + y*X + x over a (T, Y, X)
grid.  The generators give Q and K the structure the block-sparse papers describe for video
DiTs: tokens that belong to one semantic region attend to each other (cluster field), some heads
are local along the sequence or repeat across frames (diagonal and multi-diagonal heads, as in
Sparse-vDiT's pattern analysis), and a few keys act as attention sinks (the skewed rows of
SpargeAttention2's failure analysis).  No model activations are involved: every value comes
from a counter-based numpy PCG64 stream keyed by (seed, workload, batch, head).

All tensors are returned as uint16 arrays holding bf16 bit patterns (round-to-nearest-even from
fp32), shape [B, H, N, d].
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace

import numpy as np

__all__ = ["Workload", "WORKLOADS", "get", "make_qkv", "f32_to_bf16_bits", "bf16_bits_to_f32"]


@dataclass(frozen=True)
class Workload:
    """One attention call: shapes, block size and the hybrid selection parameters."""

    name: str
    B: int
    H: int
    N: int
    d: int
    bs: int
    topk: int
    topp: float
    grid: tuple  # latent (T, Y, X); T*Y*X == N
    recipe: str  # "pr1" | "cluster" | "hunyuan" | "mixed"
    centres: int = 0
    amp: float = 0.0  # norm of the structured component added to Q and K (cluster field)
    amp_diag: float = 0.0  # norm of the diagonal locality field
    amp_multi: float = 0.0  # norm of the multi-diagonal locality field
    sink_heads: tuple = ()
    sink_gain: float = 8.0
    wid: int = 0  # stream key
    sweep: tuple = field(default=())  # extra (topk, topp) points timed on this shape

    @property
    def nb(self) -> int:
        return (self.N + self.bs - 1) // self.bs

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def with_selection(self, topk: int, topp: float) -> "Workload":
        return replace(self, topk=int(topk), topp=float(topp))


def _k_for(sparsity: float, nb: int) -> int:
    """k that keeps (1 - sparsity) of the key blocks before top-p adds any."""
    return max(1, int(round((1.0 - sparsity) * nb)))


WORKLOADS = {
    # Small case: 4x16x16 latent, 8 cluster centres of norm 3, one sink key in head 0.
    "pr1_1k": Workload("pr1_1k", B=1, H=2, N=1024, d=64, bs=64, topk=2, topp=0.6,
                       grid=(4, 16, 16), recipe="pr1", centres=8, amp=3.0, sink_heads=(0,),
                       sink_gain=8.0, wid=1),
    # Wan2.1-1.3B at 480p: 21x30x52 latent, 12 heads of 128.
    "wan1.3b_480p": Workload("wan1.3b_480p", B=1, H=12, N=32760, d=128, bs=128,
                             topk=_k_for(0.95, 256), topp=0.9, grid=(21, 30, 52),
                             recipe="cluster", centres=64, amp=36.0, sink_heads=(0, 6),
                             sink_gain=8.0, wid=2),
    # Wan2.1-14B at 720p: 21x45x80 latent, 40 heads of 128; sparsity swept 80/90/95 %.
    "wan14b_720p": Workload("wan14b_720p", B=1, H=40, N=75600, d=128, bs=128,
                            topk=_k_for(0.95, 591), topp=0.9, grid=(21, 45, 80),
                            recipe="cluster", centres=128, amp=38.0, sink_heads=(0, 20),
                            sink_gain=8.0, wid=3,
                            sweep=tuple((_k_for(s, 591), p) for s in (0.80, 0.90, 0.95)
                                        for p in (0.8, 0.9, 0.95))),
    # HunyuanVideo at 720p: 33x45x80 latent, 24 heads; heads 0-11 locality, 12-23 clusters.
    "hunyuan_720p": Workload("hunyuan_720p", B=1, H=24, N=118800, d=128, bs=128,
                             topk=_k_for(0.95, 929), topp=0.9, grid=(33, 45, 80),
                             recipe="hunyuan", centres=128, amp=36.0, amp_diag=12.0,
                             amp_multi=20.0, wid=4),
    # Stress: per head a third of the query blocks each uniform / sink-dominated / local.
    "stress_mixed": Workload("stress_mixed", B=2, H=16, N=49152, d=64, bs=128, topk=4,
                             topp=0.95, grid=(16, 48, 64), recipe="mixed", amp=10.0,
                             sink_gain=12.0, wid=5),
}


def get(name: str) -> Workload:
    return WORKLOADS[name]


# ------------------------------------------------------------------------------------------------
# bf16 bit conversion (round to nearest even; inputs are finite)
# ------------------------------------------------------------------------------------------------
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + r) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(
        np.float32)


# ------------------------------------------------------------------------------------------------
# structured fields
# ------------------------------------------------------------------------------------------------
def _coords(grid):
    T, Y, X = grid
    t, y, x = np.meshgrid(np.arange(T), np.arange(Y), np.arange(X), indexing="ij")
    return t.reshape(-1), y.reshape(-1), x.reshape(-1)


def _unit_rows(rng, n, d, norm):
    c = rng.standard_normal((n, d))
    c /= np.linalg.norm(c, axis=1, keepdims=True)
    return c * norm


def _cluster_field(rng, grid, centres, d, amp):
    """Smooth mixture of `centres` directions: nearest-centre regions blurred by (1, 2, 2) cells."""
    from scipy.ndimage import gaussian_filter

    T, Y, X = grid
    vec = _unit_rows(rng, centres, d, amp)
    pos = rng.random((centres, 3)) * np.array([T, Y, X], np.float64)
    t, y, x = _coords(grid)
    cell = np.stack([t, y, x], 1).astype(np.float64) + 0.5
    # nearest centre of every cell (Voronoi regions of the seeded positions)
    best = np.zeros(cell.shape[0], np.int64)
    bestd = np.full(cell.shape[0], np.inf)
    for c in range(centres):
        dd = ((cell - pos[c]) ** 2).sum(1)
        better = dd < bestd
        best[better] = c
        bestd[better] = dd[better]
    onehot = np.zeros((centres, T, Y, X), np.float32)
    onehot.reshape(centres, -1)[best, np.arange(best.size)] = 1.0
    w = gaussian_filter(onehot, sigma=(0, 1, 2, 2), mode="nearest")
    w = w.reshape(centres, -1)
    w /= w.sum(0, keepdims=True)
    return (w.T.astype(np.float64) @ vec).astype(np.float32)


def _diag_field(rng, N, d, amp, bs):
    """Features of the flat position at 8 log-spaced periods: F(n).F(m) ~ sum cos(w (n - m))."""
    periods = 2.0 * bs * (max(N, 4 * bs) / (2.0 * bs)) ** (np.arange(8) / 7.0)
    w = 2 * np.pi / periods * (1.0 + 0.1 * rng.random(8))
    n = np.arange(N, dtype=np.float64)[:, None]
    phi = np.concatenate([np.cos(n * w), np.sin(n * w)], 1)  # [N, 16], |phi|^2 = 8
    basis, _ = np.linalg.qr(rng.standard_normal((d, 16)))
    return (phi @ basis.T * (amp / math.sqrt(8.0))).astype(np.float32)


def _multidiag_field(rng, grid, d, amp):
    """Features of (y, x) only: every frame repeats the same map (multi-diagonal pattern)."""
    T, Y, X = grid
    _, y, x = _coords(grid)
    py = np.array([3.0, 6.0, 12.0, 2.0 * Y]) * (1.0 + 0.1 * rng.random(4))
    px = np.array([3.0, 6.0, 12.0, 2.0 * X]) * (1.0 + 0.1 * rng.random(4))
    ay = 2 * np.pi * y[:, None] / py
    ax = 2 * np.pi * x[:, None] / px
    phi = np.concatenate([np.cos(ay), np.sin(ay), np.cos(ax), np.sin(ax)], 1)  # |phi|^2 = 8
    basis, _ = np.linalg.qr(rng.standard_normal((d, 16)))
    return (phi @ basis.T * (amp / math.sqrt(8.0))).astype(np.float32)


# ------------------------------------------------------------------------------------------------
# per-head generators
# ------------------------------------------------------------------------------------------------
def _rng(seed, w, b, h):
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(w.wid, b, h))))


def _normal(rng, N, d):
    return rng.standard_normal((N, d), dtype=np.float32)


def _head_pr1(w, rng, h):
    T, Y, X = w.grid
    cells = T * (Y // 8) * (X // 8)
    vec = _unit_rows(rng, w.centres, w.d, w.amp).astype(np.float32)
    perm = rng.permutation(cells)
    t, y, x = _coords(w.grid)
    cell = (t * (Y // 8) + y // 8) * (X // 8) + x // 8
    F = vec[perm[cell] % w.centres]
    q = _normal(rng, w.N, w.d) + F
    k = _normal(rng, w.N, w.d) + F
    v = _normal(rng, w.N, w.d)
    if h in w.sink_heads:
        k[0] *= w.sink_gain
    return q, k, v


def _head_cluster(w, rng, h):
    F = _cluster_field(rng, w.grid, w.centres, w.d, w.amp)
    s = np.float32(1.0 / math.sqrt(2.0))
    q = _normal(rng, w.N, w.d) * s + F
    k = _normal(rng, w.N, w.d) * s + F
    v = _normal(rng, w.N, w.d)
    if h in w.sink_heads:
        k[0] *= w.sink_gain
    return q, k, v


def _head_hunyuan(w, rng, h):
    half = w.H // 2
    if h < half // 2:
        F = _diag_field(rng, w.N, w.d, w.amp_diag, w.bs)
    elif h < half:
        F = _multidiag_field(rng, w.grid, w.d, w.amp_multi)
    else:
        F = _cluster_field(rng, w.grid, w.centres, w.d, w.amp)
    s = np.float32(1.0 / math.sqrt(2.0))
    q = _normal(rng, w.N, w.d) * s + F
    k = _normal(rng, w.N, w.d) * s + F
    v = _normal(rng, w.N, w.d)
    return q, k, v


def _head_mixed(w, rng, h):
    nb = w.nb
    F = _diag_field(rng, w.N, w.d, w.amp, w.bs)
    k = _normal(rng, w.N, w.d) + F
    nsink = int(rng.integers(1, 5))
    sinks = np.sort(rng.choice(w.N, size=nsink, replace=False))
    k[sinks] *= w.sink_gain
    q = _normal(rng, w.N, w.d)
    role = rng.permutation(nb) % 3  # 0 uniform, 1 sink-dominated, 2 local
    for i in range(nb):
        t0, t1 = i * w.bs, min((i + 1) * w.bs, w.N)
        if role[i] == 1:
            s = sinks[i % nsink]
            u = k[s] / np.linalg.norm(k[s])
            q[t0:t1] += np.float32(w.amp * 16.0) * u
        elif role[i] == 2:
            q[t0:t1] += F[t0:t1]
    v = _normal(rng, w.N, w.d)
    return q, k, v


_RECIPES = {"pr1": _head_pr1, "cluster": _head_cluster, "hunyuan": _head_hunyuan,
            "mixed": _head_mixed}


def make_qkv(w: Workload, seed: int = 0, threads: int | None = None, heads=None):
    """Q, K, V for workload `w` as bf16 bit patterns [B, H, N, d] (uint16).

    heads: optional list of flat (batch, head) indices bh = b * H + h; then only those heads are
    generated, as [1, len(heads), N, d] in the given order, each bit-identical to its slice of
    the full tensors (every head has its own seeded stream)."""
    T, Y, X = w.grid
    assert T * Y * X == w.N, (w.name, w.grid, w.N)
    sel = list(range(w.B * w.H)) if heads is None else [int(x) for x in heads]
    shape = (w.B, w.H, w.N, w.d) if heads is None else (1, len(sel), w.N, w.d)
    out = [np.empty(shape, np.uint16) for _ in range(3)]
    flat = [x.reshape(-1, w.N, w.d) for x in out]
    fn = _RECIPES[w.recipe]

    def one(slot):
        b, h = divmod(sel[slot], w.H)
        rng = _rng(seed, w, b, h)
        for dst, x in zip(flat, fn(w, rng, h)):
            dst[slot] = f32_to_bf16_bits(x)

    n = len(sel)
    threads = threads or min(max(n, 1), os.cpu_count() or 1, 16)
    if threads <= 1:
        for slot in range(n):
            one(slot)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(one, range(n)))
    return tuple(out)
