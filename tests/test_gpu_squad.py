"""GPU parity of SQuad attention (local pass within windows, global pass across windows with the
local outputs as values) against the fp64 oracle, through the C ABI via the Python binding."""
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


@pytest.mark.parametrize("B,H,N,d,w", [(1, 2, 512, 64, 64),     # 8 windows of one tile
                                       (1, 2, 900, 128, 300),   # windows with a ragged tile
                                       (2, 1, 384, 128, 128),   # 3 windows
                                       (1, 1, 256, 64, 256),    # one window: dense attention
                                       # global pass packed 6 sequences of 21 to a tile, the
                                       # last tile holding 2
                                       (1, 2, 2100, 128, 100),
                                       (1, 1, 1024, 64, 16),    # 64-token sequences, 2 per tile
                                       (1, 1, 1400, 64, 20)])   # 70-token sequences: unpacked
def test_squad_parity(orc, B, H, N, d, w):
    rng = np.random.default_rng(N + w)
    q, k, v = (f32_to_bf16_bits(rng.standard_normal((B, H, N, d)).astype(np.float32))
               for _ in range(3))
    to_dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).view(torch.bfloat16).to(DEV)
    o = bsa.squad_attn_fwd(to_dev(q), to_dev(k), to_dev(v), w)
    torch.cuda.synchronize()
    got = bf16_bits_to_f32(o.contiguous().view(torch.int16).cpu().numpy().view(np.uint16))
    ref = orc.squad_attention(q.reshape(B * H, N, d), k.reshape(B * H, N, d),
                              v.reshape(B * H, N, d), w, 1 / math.sqrt(d))
    compare_attention(got.reshape(B * H, N, d).astype(np.float64), ref)
