"""Host-side checks of the C ABI that need no GPU: the library loads, exports every entry point
declared in include/*.h, and rejects bad arguments before launching anything."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_blocks_b200 import build

    path = build.build()
    return ctypes.CDLL(path)


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names |= set(re.findall(r"\b(sa_[a-z0-9_]+)\s*\(", src))
    return sorted(names)


def test_header_declares_the_path():
    names = _declared()
    for required in ("sa_pool_blocks", "sa_select_mask_topk_topp", "sa_block_sparse_attn_fwd",
                     "sa_pool_select_topk_topp",
                     "sa_dense_attn_fwd", "sa_get_error_string", "sa_get_device_error",
                     "sa_select_from_logits"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in _declared():
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"


def test_error_strings(lib):
    lib.sa_get_error_string.restype = ctypes.c_char_p
    lib.sa_get_error_string.argtypes = [ctypes.c_int]
    assert lib.sa_get_error_string(0) == b"SA_OK"
    assert b"TIMEOUT" in lib.sa_get_error_string(4)
    assert b"unknown" in lib.sa_get_error_string(99)


def test_num_blocks(lib):
    lib.sa_num_blocks.argtypes = [ctypes.c_int, ctypes.c_int]
    assert lib.sa_num_blocks(32760, 128) == 256
    assert lib.sa_num_blocks(75600, 128) == 591
    assert lib.sa_num_blocks(118800, 128) == 929
    assert lib.sa_num_blocks(1024, 64) == 16
    assert lib.sa_num_blocks(0, 128) == 0


# Fake, 16-byte aligned, non-null addresses: every call below must be rejected by the host-side
# checks before the library touches CUDA.
A = ctypes.c_void_p(0x10000)
A2 = ctypes.c_void_p(0x20000)
MIS = ctypes.c_void_p(0x10008)
MIS4 = ctypes.c_void_p(0x10002)  # not even 4-byte aligned (int32 / fp32 element buffers)
NUL = ctypes.c_void_p(0)
S = ctypes.c_void_p(0)


def test_pool_argument_checks(lib):
    f = lib.sa_pool_blocks
    f.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 5 + [ctypes.c_void_p]
    assert f(NUL, A, A, A, 1, 1, 128, 128, 128, S) == 1
    assert f(A, A, A, A, 0, 1, 128, 128, 128, S) == 1
    assert f(A, A, A, A, 1, 1, 0, 128, 128, S) == 1
    assert f(A, A, A, A, 300, 300, 128, 128, 128, S) == 1  # B*H > 65535
    assert f(A, A, A, A, 1, 1, 128, 96, 128, S) == 2
    assert f(A, A, A, A, 1, 1, 128, 128, 32, S) == 2
    assert f(MIS, A, A, A, 1, 1, 128, 128, 128, S) == 1


def test_select_argument_checks(lib):
    f = lib.sa_select_mask_topk_topp
    f.argtypes = [ctypes.c_void_p] * 2 + [ctypes.c_int] * 5 + [ctypes.c_float] * 2 + \
        [ctypes.c_void_p] * 4
    ok = dict(B=1, H=1, nb=16, d=64, k=2, p=0.5, s=0.0)

    def call(qp=A, mask=A2, idx=A, cnt=A2, **kw):
        a = {**ok, **kw}
        return f(qp, A, a["B"], a["H"], a["nb"], a["d"], a["k"], a["p"], a["s"], mask, idx, cnt, S)

    assert call(qp=NUL) == 1
    assert call(k=-1) == 1
    assert call(p=1.5) == 1
    assert call(p=-0.1) == 1
    assert call(p=float("nan")) == 1
    assert call(s=float("nan")) == 1
    assert call(d=80) == 2
    assert call(nb=1025) == 2
    assert call(idx=MIS4) == 1
    g = lib.sa_select_from_logits
    g.argtypes = [ctypes.c_void_p] + [ctypes.c_int] * 4 + [ctypes.c_float] + [ctypes.c_void_p] * 4
    assert g(NUL, 1, 1, 16, 2, 0.5, A, A, A, S) == 1
    assert g(A, 1, 1, 2000, 2, 0.5, A, A, A, S) == 2
    assert g(A, 1, 1, 16, 2, 2.0, A, A, A, S) == 1


def test_pool_select_argument_checks(lib):
    f = lib.sa_pool_select_topk_topp
    f.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 6 + [ctypes.c_float] * 2 + \
        [ctypes.c_void_p] * 4
    ok = dict(B=1, H=1, N=256, d=128, bs=128, k=2, p=0.5, s=0.0)

    def call(q=A, qp=A2, idx=A, **kw):
        a = {**ok, **kw}
        return f(q, A, qp, A2, a["B"], a["H"], a["N"], a["d"], a["bs"], a["k"], a["p"], a["s"],
                 A, idx, A2, S)

    assert call(q=NUL) == 1
    assert call(k=-1) == 1
    assert call(p=1.5) == 1
    assert call(s=float("nan")) == 1
    assert call(d=96) == 2
    assert call(bs=32) == 2
    assert call(N=128 * 1025) == 2
    assert call(qp=MIS) == 1
    assert call(idx=MIS4) == 1


def test_attention_argument_checks(lib):
    lib.sa_attn_workspace_bytes.restype = ctypes.c_size_t
    W = lib.sa_attn_workspace_bytes()
    assert 8 <= W <= 4096
    f = lib.sa_block_sparse_attn_fwd
    f.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_int] * 5 + [ctypes.c_float, ctypes.c_void_p,
                                                                ctypes.c_size_t, ctypes.c_void_p]
    assert f(A, A, A, NUL, A, A, 1, 1, 256, 128, 128, 0.0, A2, W, S) == 1
    assert f(A, A, A, A, A, A, 1, 1, 256, 256, 128, 0.0, A2, W, S) == 2
    assert f(A, A, A, A, A, A, 1, 1, 256, 128, 256, 0.0, A2, W, S) == 2
    assert f(A, A, A, A, A, A, 1, 1, 128 * 1025, 128, 128, 0.0, A2, W, S) == 2
    assert f(A, A, A, A, A, MIS, 1, 1, 256, 128, 128, 0.0, A2, W, S) == 1
    assert f(A, A, A, A, A, A, 1, 1, 256, 128, 128, float("nan"), A2, W, S) == 1
    assert f(A, A, A, A, A, A, 1, 1, 256, 128, 128, 0.0, NUL, W, S) == 1
    assert f(A, A, A, A, A, A, 1, 1, 256, 128, 128, 0.0, A2, W - 1, S) == 1
    g = lib.sa_dense_attn_fwd
    g.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 4 + [ctypes.c_float, ctypes.c_void_p,
                                                                ctypes.c_size_t, ctypes.c_void_p]
    assert g(A, A, NUL, A, 1, 1, 256, 128, 0.0, A2, W, S) == 1
    assert g(A, A, A, A, 1, 1, 256, 32, 0.0, A2, W, S) == 2
    assert g(A, A, A, A, 1, 1, 256, 128, 0.0, NUL, W, S) == 1


def test_noalloc_attention_argument_checks(lib):
    # the allocation-free entry point rejects what the workspace entry point rejects, on the host
    # and before it resolves its scratch array: null pointers, unsupported sizes, a NaN scale,
    # misaligned buffers, and an output that is not device memory
    f = lib.sa_block_sparse_attn_fwd_noalloc
    f.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_int] * 5 + [ctypes.c_float, ctypes.c_void_p]
    assert f(A, A, A, A, A, NUL, 1, 1, 256, 128, 128, 0.0, S) == 1   # null o
    assert f(NUL, A, A, A, A, A, 1, 1, 256, 128, 128, 0.0, S) == 1   # null q
    assert f(A, A, A, A, NUL, A, 1, 1, 256, 128, 128, 0.0, S) == 1   # null kv_cnt
    assert f(A, A, A, A, A, A, 1, 1, 256, 96, 128, 0.0, S) == 2      # unsupported d
    assert f(A, A, A, A, A, A, 1, 1, 256, 128, 32, 0.0, S) == 2      # unsupported bs
    assert f(A, A, A, A, A, A, 1, 1, 128 * 1025, 128, 128, 0.0, S) == 2
    assert f(A, A, A, A, A, A, 1, 1, 256, 128, 128, float("nan"), S) == 1
    assert f(A, A, A, A, A, MIS, 1, 1, 256, 128, 128, 0.0, S) == 1
    assert f(A, A, A, A, A, A, 0, 1, 256, 128, 128, 0.0, S) == 1
    host = ctypes.create_string_buffer(256 * 128 * 2 + 16)
    o_host = ctypes.c_void_p((ctypes.addressof(host) + 15) // 16 * 16)
    assert f(A, A, A, A, A, o_host, 1, 1, 256, 128, 128, 0.0, S) == 1  # o not device memory


def test_sparsepr_argument_checks(lib):
    lib.sa_sparsepr_workspace_bytes.restype = ctypes.c_size_t
    lib.sa_sparsepr_workspace_bytes.argtypes = [ctypes.c_int] * 5
    W = lib.sa_sparsepr_workspace_bytes(1, 2, 1000, 128, 40)
    assert W > 2 * 40 * 128 * 2  # at least the gathered probe rows
    assert lib.sa_sparsepr_workspace_bytes(1, 2, 1000, 96, 40) == 0      # unsupported d
    assert lib.sa_sparsepr_workspace_bytes(1, 2, 1000, 128, 0) == 0      # no probes
    assert lib.sa_sparsepr_workspace_bytes(1, 2, 1000, 128, 9000) == 0   # too many probes
    f = lib.sa_sparsepr_attn_fwd
    f.argtypes = ([ctypes.c_void_p] * 6 + [ctypes.c_int, ctypes.c_void_p] + [ctypes.c_int] * 5
                  + [ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p])
    ok = lambda **kw: f(kw.get("q", A), A, A, A, A, kw.get("pr", A), kw.get("m", 40),
                        kw.get("o", A), 1, 2, kw.get("N", 1000), kw.get("d", 128),
                        kw.get("bs", 128), kw.get("s", 0.0), kw.get("ws", A2), kw.get("wb", W), S)
    assert ok(q=NUL) == 1
    assert ok(pr=NUL) == 1
    assert ok(o=NUL) == 1
    assert ok(ws=NUL) == 1
    assert ok(wb=W - 1) == 1
    assert ok(m=0) == 1
    assert ok(m=1001) == 1           # more probes than tokens
    assert ok(d=96) == 2
    assert ok(bs=32) == 2
    assert ok(s=float("nan")) == 1
    assert ok(pr=MIS4) == 1
    assert ok(o=MIS) == 1


def test_python_binding_imports():
    import block_sparse_attention_blocks_b200 as pkg

    assert callable(pkg.sparse_attention)
    assert pkg.num_blocks(75600, 128) == 591


def test_block_scores_argument_checks(lib):
    f = lib.sa_block_scores
    f.argtypes = [ctypes.c_void_p] * 2 + [ctypes.c_int] * 4 + [ctypes.c_float] + [ctypes.c_void_p] * 2
    assert f(NUL, A, 1, 1, 16, 128, 0.0, A2, S) == 1
    assert f(A, A, 1, 1, 16, 96, 0.0, A2, S) == 2
    assert f(A, A, 1, 1, 16, 128, float("nan"), A2, S) == 1
    assert f(A, A, 1, 1, 16, 128, 0.0, MIS4, S) == 1
    assert f(MIS, A, 1, 1, 16, 128, 0.0, A2, S) == 1
    assert f(A, A, 0, 1, 16, 128, 0.0, A2, S) == 1


def test_bf16_three_way_split_is_exact():
    # The tensor-core block scores split every fp32 operand x into bf16 parts by masking: h = x
    # with the low 16 bits cleared, m the same of x - h, l = x - h - m.  The split must be exact
    # (h + m + l == x) with l representable in bf16 (low 16 bits zero), for any sign and scale.
    import numpy as np

    rng = np.random.default_rng(3)
    x = (rng.standard_normal(200000) * np.exp2(rng.integers(-60, 60, 200000))).astype(np.float32)
    x = np.concatenate([x, np.float32([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38, 1.0e-30])])
    mask = np.uint32(0xFFFF0000)
    h = (x.view(np.uint32) & mask).view(np.float32)
    rm = (x - h).astype(np.float32)
    m = (rm.view(np.uint32) & mask).view(np.float32)
    low = (rm - m).astype(np.float32)
    assert np.all((low.view(np.uint32) & np.uint32(0xFFFF)) == 0)
    assert np.array_equal(h.astype(np.float64) + m.astype(np.float64) + low.astype(np.float64),
                          x.astype(np.float64))
    # the dropped products m*l, l*m, l*l are below 2^-15 of |x|^2 each (|m| < 2^-7 |x|,
    # |l| < 2^-14 |x| for normal x)
    nz = np.abs(x) > 1e-30
    assert np.all(np.abs(m[nz]) <= np.abs(x[nz]) * 2.0 ** -7)
    assert np.all(np.abs(low[nz]) <= np.abs(x[nz]) * 2.0 ** -14)


def test_static_mask_argument_checks(lib):
    f = lib.sa_static_mask
    f.argtypes = [ctypes.c_void_p] + [ctypes.c_int] * 3 + [ctypes.c_void_p] * 4
    assert f(NUL, 1, 1, 16, A, A2, A, S) == 1
    assert f(A, 1, 1, 16, A, MIS4, A, S) == 1
    assert f(A, 0, 1, 16, A, A2, A, S) == 1
    assert f(A, 1, 1, 16, NUL, A2, A, S) == 1


def test_squad_argument_checks(lib):
    lib.sa_squad_workspace_bytes.restype = ctypes.c_size_t
    lib.sa_squad_workspace_bytes.argtypes = [ctypes.c_int] * 4
    W = lib.sa_squad_workspace_bytes(1, 2, 512, 64)
    assert W >= 4 * 2 * 512 * 64 * 2
    f = lib.sa_squad_attn_fwd
    f.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 5 + [ctypes.c_float, ctypes.c_void_p,
                                                                ctypes.c_size_t, ctypes.c_void_p]
    assert f(NUL, A, A, A, 1, 2, 512, 64, 64, 0.0, A2, W, S) == 1
    assert f(A, A, A, A, 1, 2, 512, 96, 64, 0.0, A2, W, S) == 2
    assert f(A, A, A, A, 1, 2, 512, 64, 100, 0.0, A2, W, S) == 1   # N not a multiple of w
    assert f(A, A, A, A, 1, 2, 512, 64, 0, 0.0, A2, W, S) == 1
    assert f(A, A, A, A, 1, 2, 512, 64, 64, 0.0, A2, W - 1, S) == 1
    assert f(A, A, A, A, 1, 2, 512, 64, 64, float("nan"), A2, W, S) == 1


def test_cluster_entry_point_argument_checks(lib):
    I, P, F, Z = ctypes.c_int, ctypes.c_void_p, ctypes.c_float, ctypes.c_size_t
    lib.sa_kmeans_workspace_bytes.restype = Z
    lib.sa_kmeans_workspace_bytes.argtypes = [I] * 5
    Wk = lib.sa_kmeans_workspace_bytes(1, 2, 100, 8, 64)
    assert Wk >= 2 * 3 * 8 * 64 * 2 + 2 * 8 * 4       # centroid parts (bf16) and norms
    assert lib.sa_kmeans_workspace_bytes(0, 2, 100, 8, 64) == 0
    assert lib.sa_kmeans_workspace_bytes(1, 2, 0, 8, 64) == 0
    # above 128 centroids, each 128-centroid tile's candidate per token (8 bytes) is kept too
    assert (lib.sa_kmeans_workspace_bytes(1, 2, 100, 300, 64)
            >= 2 * 3 * 300 * 64 * 2 + 2 * 300 * 4 + 3 * 2 * 100 * 8)
    km = lib.sa_kmeans
    km.argtypes = [P] * 6 + [I] * 6 + [P, Z, P]
    assert km(NUL, A, A, A, A, A, 1, 2, 100, 64, 8, 2, A2, Wk, S) == 1
    assert km(A, A, A, A, A, A, 1, 2, 100, 96, 8, 2, A2, Wk, S) == 2          # d
    assert km(A, A, A, A, A, A, 1, 2, 100, 64, 0, 2, A2, Wk, S) == 1          # C < 1
    assert km(A, A, A, A, A, A, 1, 2, 100, 64, 1025, 2, A2, Wk, S) == 1       # C > 1024
    assert km(A, A, A, A, A, A, 1, 2, 100, 64, 8, -1, A2, Wk, S) == 1         # iters
    assert km(A, MIS, A, A, A, A, 1, 2, 100, 64, 8, 2, A2, Wk, S) == 1        # centroids need 16 B
    assert km(A, A, A, A, A, A, 1, 2, 100, 64, 8, 2, NUL, Wk, S) == 1         # no workspace
    assert km(A, A, A, A, A, A, 1, 2, 100, 64, 8, 2, A2, Wk - 1, S) == 1      # workspace too small
    lib.sa_cluster_sort_workspace_bytes.restype = Z
    lib.sa_cluster_sort_workspace_bytes.argtypes = [I] * 4
    Ws = lib.sa_cluster_sort_workspace_bytes(1, 2, 10000, 40)
    assert Ws >= 2 * 3 * 40 * 4                         # counts of every 4096-token chunk
    assert lib.sa_cluster_sort_workspace_bytes(1, 2, 0, 40) == 0
    cs = lib.sa_cluster_sort
    cs.argtypes = [P] + [I] * 4 + [P] * 4 + [Z, P]
    assert cs(NUL, 1, 1, 10, 4, A, A, A, A2, Ws, S) == 1
    assert cs(A, 1, 1, 10, 4, MIS4, A, A, A2, Ws, S) == 1
    assert cs(A, 1, 2, 10000, 40, A, A, A, NUL, Ws, S) == 1       # no workspace
    assert cs(A, 1, 2, 10000, 40, A, A, A, A2, Ws - 1, S) == 1    # workspace too small

    lib.sa_centroid_topp_workspace_bytes.restype = Z
    lib.sa_centroid_topp_workspace_bytes.argtypes = [I] * 4
    Wt = lib.sa_centroid_topp_workspace_bytes(1, 2, 16, 40)
    assert Wt >= 2 * 16 * 40 * 4 + 2 * 16 * 4
    assert lib.sa_centroid_topp_workspace_bytes(0, 2, 16, 40) == 0
    ct = lib.sa_centroid_topp
    ct.argtypes = [P] * 3 + [I] * 5 + [F, F, P, P, Z, P]
    assert ct(NUL, A, A, 1, 2, 16, 40, 64, 0.9, 0.0, A2, A, Wt, S) == 1
    assert ct(A, A, A, 1, 2, 16, 40, 80, 0.9, 0.0, A2, A, Wt, S) == 2
    assert ct(A, A, A, 1, 2, 16, 40, 64, 1.5, 0.0, A2, A, Wt, S) == 1
    assert ct(A, A, A, 1, 2, 16, 40, 64, 0.9, float("nan"), A2, A, Wt, S) == 1
    assert ct(A, A, A, 1, 2, 16, 40, 64, 0.9, 0.0, A2, A, Wt - 1, S) == 1
    assert ct(A, A, A, 1, 2, 16, 2000, 64, 0.9, 0.0, A2, A, Wt, S) == 1

    for name in ("sa_cluster_attn_workspace_bytes", "sa_svg2_workspace_bytes"):
        getattr(lib, name).restype = Z
        getattr(lib, name).argtypes = [I] * 6
    Wc = lib.sa_cluster_attn_workspace_bytes(1, 2, 1000, 64, 16, 40)
    Ws = lib.sa_svg2_workspace_bytes(1, 2, 1000, 64, 16, 40)
    # three permuted tensors, two permutations, tile tables; the full path adds the assignments
    # and the centroid scores
    assert Wc >= 3 * 2 * 1000 * 64 * 2 + 2 * 2 * 1000 * 4 + 2 * 16 * (8 + 40) * 4
    assert Ws >= Wc + 2 * 2 * 1000 * 4 + 2 * 16 * 40 * 4
    ca = lib.sa_cluster_attn_fwd
    ca.argtypes = [P] * 7 + [I] * 6 + [F, P, Z, P]
    assert ca(NUL, A, A, A, A, A, A, 1, 2, 1000, 64, 16, 40, 0.0, A2, Wc, S) == 1
    assert ca(A, A, A, A, A, A, A, 1, 2, 1000, 96, 16, 40, 0.0, A2, Wc, S) == 2
    assert ca(A, A, A, A, A, A, A, 1, 2, 1 << 24, 64, 16, 40, 0.0, A2, Wc, S) == 2  # N limit
    assert ca(A, A, A, A, A, A, A, 1, 2, 1000, 64, 0, 40, 0.0, A2, Wc, S) == 1
    assert ca(A, A, A, A, A, A, A, 1, 2, 1000, 64, 16, 40, 0.0, A2, Wc - 1, S) == 1
    assert ca(A, A, A, A, MIS4, A, A, 1, 2, 1000, 64, 16, 40, 0.0, A2, Wc, S) == 1
    assert ca(MIS, A, A, A, A, A, A, 1, 2, 1000, 64, 16, 40, 0.0, A2, Wc, S) == 1
    sv = lib.sa_svg2_attn_fwd
    sv.argtypes = [P] * 6 + [I] * 7 + [F, F, P, P, Z, P]
    assert sv(A, A, A, A, A, NUL, 1, 2, 1000, 64, 16, 40, 2, 0.9, 0.0, A, A2, Ws, S) == 1
    assert sv(A, A, A, A, A, A, 1, 2, 1000, 128, 16, 40, -1, 0.9, 0.0, A, A2, Ws, S) == 1
    assert sv(A, A, A, A, A, A, 1, 2, 1000, 64, 16, 40, 2, -0.1, 0.0, A, A2, Ws, S) == 1
    assert sv(A, A, A, A, A, A, 1, 2, 1000, 64, 16, 40, 2, 0.9, 0.0, A, A2, Wc, S) == 1
    assert sv(A, A, A, A, MIS, A, 1, 2, 1000, 64, 16, 40, 2, 0.9, 0.0, A, A2, Ws, S) == 1
    assert sv(A, A, A, A, A, A, 1, 2, 1000, 32, 16, 40, 2, 0.9, 0.0, A, A2, Ws, S) == 2


def test_host_inputs_are_checked_before_any_device_work():
    import torch

    from block_sparse_attention_blocks_b200 import sparse_attn as s

    q = torch.empty(1, 2, 100, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        s.sparse_attention(q, q[:, :1].contiguous(), q, 64, 2, 0.9)       # k of another shape
    with pytest.raises(TypeError):
        s.sparse_attention(q, q.float(), q, 64, 2, 0.9)                   # v not bf16
    with pytest.raises(ValueError):
        s.sparse_attention(q, q, q, 64, 2, 0.9, out=torch.empty(1, 2, 99, 64,
                                                                 dtype=torch.bfloat16))
    with pytest.raises(TypeError):
        s.sparse_attention(q, q, q.transpose(2, 3), 64, 2, 0.9)           # not contiguous
