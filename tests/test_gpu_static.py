"""GPU parity of the static block patterns (Sparse-vDiT section 3: diagonal, multi-diagonal,
vertical-stripe and skipped heads) against the oracle, and of attention over them.  All calls go
through the C ABI via the Python binding."""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_blocks_b200.workloads import bf16_bits_to_f32, f32_to_bf16_bits
from tests.parity import compare_attention

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import block_sparse_attention_blocks_b200 as bsa  # noqa: E402  (loads libbsa.so, fails loudly)

DEV = torch.device("cuda", 0)


def _patterns(rng, H):
    return [(int(rng.integers(0, 8)), int(rng.integers(0, 12)), int(rng.integers(0, 40)),
             int(rng.integers(0, 20))) for _ in range(H)]


@pytest.mark.parametrize("nb", [1, 31, 32, 33, 100, 591, 1024])
def test_static_mask_bit_exact(orc, nb):
    rng = np.random.default_rng(nb)
    B, H = 2, 6
    pats = _patterns(rng, H)
    pats[0] = (0, 5, 3, 2)      # skipped head
    pats[1] = (5, 7, 0, 16)     # band + leading stripe
    mask, idx, cnt = bsa.static_mask(pats, B, nb)
    torch.cuda.synchronize()
    ref = orc.static_mask(pats, B, nb)
    got = mask.cpu().numpy()
    assert np.array_equal(got, ref)
    c = cnt.cpu().numpy().reshape(-1)
    assert np.array_equal(c, ref.reshape(-1, nb).sum(1))
    ids = idx.cpu().numpy().reshape(-1, nb)
    for r, row in enumerate(ref.reshape(-1, nb)):
        assert np.array_equal(ids[r, :c[r]], np.flatnonzero(row))


@pytest.mark.parametrize("d,bs,N", [(128, 128, 1000), (64, 64, 777)])
def test_attention_over_static_patterns(orc, d, bs, N):
    rng = np.random.default_rng(N)
    B, H = 1, 4
    nb = (N + bs - 1) // bs
    pats = [(1, 1, 0, 0), (2, 0, 3, 0), (4, 0, 0, 2), (0, 0, 0, 0)]
    q, k, v = (f32_to_bf16_bits(rng.standard_normal((B, H, N, d)).astype(np.float32))
               for _ in range(3))
    mask, idx, cnt = bsa.static_mask(pats, B, nb)
    to_dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).view(torch.bfloat16).to(DEV)
    o = bsa.block_sparse_attn_fwd(to_dev(q), to_dev(k), to_dev(v), idx, cnt, bs)
    torch.cuda.synchronize()
    og = bf16_bits_to_f32(o.contiguous().view(torch.int16).cpu().numpy().view(np.uint16))
    og = og.reshape(B * H, N, d)
    gm = orc.static_mask(pats, B, nb).reshape(B * H, nb, nb)
    ref = orc.masked_attention(q.reshape(B * H, N, d), k.reshape(B * H, N, d),
                               v.reshape(B * H, N, d), gm, bs, 1 / math.sqrt(d))
    got = np.zeros_like(ref)
    for s in range(B * H * nb):
        bh, i = divmod(s, nb)
        r1 = min(bs, N - i * bs)
        got[s, :r1] = og[bh, i * bs:i * bs + r1]
    compare_attention(got, ref)
    # the skipped head writes zeros
    assert not og[3].any()
