"""The allocation-free attention entry point against the workspace entry point.

sa_block_sparse_attn_fwd_noalloc serves callers that cannot lend the library device memory (no
spare buffer in a foreign allocator, or no cudaMalloc allowed where attention runs); it keeps
its work counter in a fixed array inside the library.  This test calls it through the C ABI
twice in a row, since every call shares that array and must leave it reusable, and compares each
result with sa_block_sparse_attn_fwd under the attention tolerance of the other GPU tests.  The
file name makes pytest collect it last.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import block_sparse_attention_blocks_b200 as bsa  # noqa: E402
from block_sparse_attention_blocks_b200 import sparse_attn as sa  # noqa: E402
from tests.parity import ATOL_MAX, ATOL_MEAN  # noqa: E402


def _noalloc(q, k, v, kv_idx, kv_cnt, o, bs):
    f = sa.lib.sa_block_sparse_attn_fwd_noalloc
    f.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_int] * 5 + [ctypes.c_float, ctypes.c_void_p]
    f.restype = ctypes.c_int
    B, H, N, d = q.shape
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return f(p(q), p(k), p(v), p(kv_idx), p(kv_cnt), p(o), B, H, N, d, bs, 0.0,
             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_workspace_entry_point_twice():
    dev = torch.device("cuda", 0)
    torch.manual_seed(0)
    B, H, N, d, bs = 1, 3, 2000, 128, 128
    q, k, v = (torch.randn(B, H, N, d, device=dev).to(torch.bfloat16) for _ in range(3))
    nb = (N + bs - 1) // bs
    g = torch.Generator().manual_seed(1)
    mask = torch.rand(B, H, nb, nb, generator=g) < 0.35
    mask[..., 0] = True
    mask[0, 1, 2, :] = False  # an empty query block
    cnt = mask.sum(-1).to(torch.int32)
    idx = torch.zeros(B, H, nb, nb, dtype=torch.int32)
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                ids = torch.nonzero(mask[b, h, i]).flatten()
                idx[b, h, i, :ids.numel()] = ids.to(torch.int32)
    idx, cnt = idx.to(dev), cnt.to(dev)

    ref = bsa.block_sparse_attn_fwd(q, k, v, idx, cnt, bs)
    for _ in range(2):
        o = torch.full_like(q, float("nan"))
        assert _noalloc(q, k, v, idx, cnt, o, bs) == 0
        torch.cuda.synchronize()
        assert bsa.device_error() == 0
        err = (o.float() - ref.float()).abs()
        assert torch.isfinite(o.float()).all()
        assert err.max().item() <= ATOL_MAX and err.mean().item() <= ATOL_MEAN
