"""The allocation-free attention entry point against the workspace entry point and the oracle.

sa_block_sparse_attn_fwd_noalloc serves callers that cannot lend the library device memory (no
spare buffer in a foreign allocator, or no cudaMalloc allowed where attention runs); it keeps
its work counter in a fixed array inside the library that every call shares.  This test calls it
through the C ABI several times in a row, on shapes that claim different numbers of query blocks
(a larger call, then smaller ones with other head and block sizes, then the larger one again),
because a counter left over from the previous call would skip or repeat work.  Each result must
be bit-identical to sa_block_sparse_attn_fwd's on the same inputs (both run the same kernel, and
a query block's arithmetic does not depend on which CTA claims it), and within the attention
tolerance of the fp64 oracle on sampled query blocks.  The file name makes pytest collect it
last.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import block_sparse_attention_blocks_b200 as bsa  # noqa: E402
from block_sparse_attention_blocks_b200 import sparse_attn as sa  # noqa: E402
from block_sparse_attention_blocks_b200.workloads import bf16_bits_to_f32  # noqa: E402
from tests.parity import compare_attention, list_from_mask  # noqa: E402

DEV = torch.device("cuda", 0)


def _noalloc(q, k, v, kv_idx, kv_cnt, o, bs):
    f = sa.lib.sa_block_sparse_attn_fwd_noalloc
    f.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_int] * 5 + [ctypes.c_float, ctypes.c_void_p]
    f.restype = ctypes.c_int
    B, H, N, d = q.shape
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return f(p(q), p(k), p(v), p(kv_idx), p(kv_cnt), p(o), B, H, N, d, bs, 0.0,
             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _case(seed, B, H, N, d, bs):
    g = torch.Generator().manual_seed(seed)
    q, k, v = (torch.randn(B, H, N, d, generator=g).to(torch.bfloat16) for _ in range(3))
    nb = (N + bs - 1) // bs
    mask = (torch.rand(B, H, nb, nb, generator=g) < 0.35).numpy().astype(np.uint8)
    mask[..., 0] = 1
    mask[0, H - 1, min(2, nb - 1), :] = 0  # an empty query block
    idx, cnt = list_from_mask(mask)
    return q, k, v, mask, idx, cnt


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def test_noalloc_bit_identical_and_oracle_across_shapes(orc):
    cases = [  # (seed, B, H, N, d, bs): query-block counts 48, 10, 34, 48
        (1, 1, 3, 2000, 128, 128),
        (2, 1, 2, 300, 64, 64),
        (3, 2, 1, 2100, 64, 128),
        (1, 1, 3, 2000, 128, 128),
    ]
    rng = np.random.default_rng(5)
    for seed, B, H, N, d, bs in cases:
        q, k, v, mask, idx, cnt = _case(seed, B, H, N, d, bs)
        qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
        idd, cnd = torch.from_numpy(idx).to(DEV), torch.from_numpy(cnt).to(DEV)
        ref = bsa.block_sparse_attn_fwd(qd, kd, vd, idd, cnd, bs)
        for _ in range(2):  # two calls in a row on the shared array
            o = torch.full_like(qd, float("nan"))
            assert _noalloc(qd, kd, vd, idd, cnd, o, bs) == 0
            torch.cuda.synchronize()
            assert bsa.device_error() == 0
            assert torch.equal(o.view(torch.int16), ref.view(torch.int16)), (seed, B, H, N, d, bs)
        # against the fp64 oracle on sampled query blocks (incl. the ragged last and the empty one)
        BH, nb = B * H, mask.shape[-1]
        picks = sorted({(0, 0), (BH - 1, nb - 1), (H - 1, min(2, nb - 1)),
                        (int(rng.integers(BH)), int(rng.integers(nb)))})
        refo = orc.masked_attention(_bits(q).reshape(BH, N, d), _bits(k).reshape(BH, N, d),
                                    _bits(v).reshape(BH, N, d), mask.reshape(BH, nb, nb), bs,
                                    1 / math.sqrt(d), picks)
        of = bf16_bits_to_f32(_bits(o.cpu())).reshape(BH, N, d)
        got = np.zeros_like(refo)
        for s, (bh, i) in enumerate(picks):
            r1 = min(bs, N - i * bs)
            got[s, :r1] = of[bh, i * bs:i * bs + r1]
        compare_attention(got, refo)
