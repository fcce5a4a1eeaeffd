"""GPU parity of SparsePR's probe-fitted residual correction (page "Partition the Support,
Reconstruct the Residual", abstract and summary section 3) against the oracle, through the C ABI.

The GPU fits on the bf16 sparse output and fp32 exact probe outputs (fp64 solve) and writes
bf16; the oracle works in fp64 throughout.  The comparison is the attention tolerance on every row of every head,
for probe counts well below and well above d + 1 (where the fit is well conditioned: with about
d + 1 probes the square system amplifies the bf16 rounding of its inputs, so that case is
checked through the properties that hold at any precision instead: the probe rows come out at
their exact values and a full mask leaves the output unchanged)."""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_blocks_b200.workloads import bf16_bits_to_f32, f32_to_bf16_bits
from tests.parity import compare_attention, list_from_mask

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import block_sparse_attention_blocks_b200 as bsa  # noqa: E402

DEV = torch.device("cuda", 0)


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16).to(DEV)


def _host(t):
    return bf16_bits_to_f32(t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16))


def _case(rng, B, H, N, d, bs, m, density=0.3):
    q, k, v = (f32_to_bf16_bits(rng.standard_normal((B * H, N, d)).astype(np.float32))
               for _ in range(3))
    nb = (N + bs - 1) // bs
    mask = (rng.random((B, H, nb, nb)) < density).astype(np.uint8)
    mask[..., 0] = 1
    idx, cnt = list_from_mask(mask)
    probes = np.stack([np.sort(rng.choice(N, m, replace=False)) for _ in range(B * H)]).astype(np.int32)
    return q, k, v, mask, idx, cnt, probes


def _run(q, k, v, idx, cnt, probes, B, H, N, d, bs):
    o = bsa.sparsepr_attn_fwd(_dev(q.reshape(B, H, N, d)), _dev(k.reshape(B, H, N, d)),
                              _dev(v.reshape(B, H, N, d)), torch.from_numpy(idx).to(DEV),
                              torch.from_numpy(cnt).to(DEV),
                              torch.from_numpy(probes.reshape(B, H, -1)).to(DEV), bs)
    torch.cuda.synchronize()
    assert bsa.device_error() == 0
    return _host(o).reshape(B * H, N, d)


@pytest.mark.parametrize("d,N,m,bs", [(64, 1000, 8, 128), (128, 1500, 40, 128),
                                      (128, 2100, 400, 128), (64, 777, 300, 64),
                                      (128, 300, 1, 64)])
def test_sparsepr_matches_oracle(orc, d, N, m, bs):
    rng = np.random.default_rng(N + m)
    B, H = 1, 2
    q, k, v, mask, idx, cnt, probes = _case(rng, B, H, N, d, bs, m)
    got = _run(q, k, v, idx, cnt, probes, B, H, N, d, bs)
    nb = mask.shape[-1]
    scale = 1 / math.sqrt(d)
    for h in range(B * H):
        ref, ref_sparse = orc.sparsepr_attention(q[h], k[h], v[h], mask.reshape(B * H, nb, nb)[h],
                                                 bs, scale, probes[h])
        compare_attention(got[h], ref)
        # the correction does act: the output differs from the uncorrected sparse attention
        assert np.abs(ref - ref_sparse).max() > 1e-3


@pytest.mark.parametrize("d,m", [(64, 65), (128, 16)])
def test_sparsepr_probe_rows_exact(orc, d, m):
    # with at most d + 1 probes the fit interpolates: each probe row comes out at its exact
    # (dense) attention output, whatever the conditioning
    rng = np.random.default_rng(d * 7 + m)
    B, H, N, bs = 1, 2, 1200, 128
    q, k, v, mask, idx, cnt, probes = _case(rng, B, H, N, d, bs, m)
    got = _run(q, k, v, idx, cnt, probes, B, H, N, d, bs)
    scale = 1 / math.sqrt(d)
    for h in range(B * H):
        dense = orc.dense_attention(q[h][None], k[h][None], v[h][None], scale,
                                    rows=[(0, int(t)) for t in probes[h]])
        assert np.abs(got[h][probes[h]] - dense).max() < 2e-2


def test_sparsepr_full_mask_is_dense(orc):
    # every key block kept: the sparse output is exact, the residuals vanish (up to bf16), and
    # the corrected output is dense attention
    rng = np.random.default_rng(5)
    B, H, N, d, bs, m = 1, 2, 900, 128, 128, 50
    q, k, v, mask, idx, cnt, probes = _case(rng, B, H, N, d, bs, m, density=1.1)
    got = _run(q, k, v, idx, cnt, probes, B, H, N, d, bs)
    for h in range(B * H):
        dense = orc.dense_attention(q[h][None], k[h][None], v[h][None], 1 / math.sqrt(d))
        compare_attention(got[h], dense.reshape(N, d))


@pytest.mark.slow
def test_sparsepr_full_shape_sampled_rows(orc):
    # the bench's SparsePR configuration on two heads of the Wan2.1-14B-720p workload (N = 75600,
    # d = 128, block 128, k = 30, p = 0.9, 256 seeded probes per head, keys split into runs): the
    # oracle fits W in fp64 from the sparse (GPU selection) and dense outputs of the probe rows,
    # computed row by row, and corrects a seeded sample of rows (first, last, random)
    from block_sparse_attention_blocks_b200 import workloads as W
    from dataclasses import replace
    w = W.get("wan14b_720p")
    heads = [0, 1]
    qb, kb, vb = W.make_qkv(w, heads=heads)
    wh = replace(w, B=1, H=len(heads))
    BH, N, d, bs, nb = len(heads), w.N, w.d, w.bs, w.nb
    q, k, v = _dev(qb), _dev(kb), _dev(vb)
    _, _, mask, idx, cnt = bsa.pool_select_topk_topp(q, k, bs, w.topk, w.topp)
    rng = np.random.default_rng(11)
    m = 256
    probes = np.stack([np.sort(rng.choice(N, m, replace=False)) for _ in range(BH)]).astype(np.int32)
    o = bsa.sparsepr_attn_fwd(q, k, v, idx, cnt, torch.from_numpy(probes.reshape(1, BH, m)).to(DEV), bs)
    torch.cuda.synchronize()
    assert bsa.device_error() == 0
    got = _host(o).reshape(BH, N, d)
    gmask = mask.cpu().numpy().reshape(BH, nb, nb)
    scale = 1 / math.sqrt(d)
    for h in range(BH):
        samples = np.unique(np.concatenate([[0, N - 1], rng.choice(N, 30, replace=False)]))
        rows = np.concatenate([probes[h], samples])
        blocks = sorted({int(t) // bs for t in rows})
        ob = orc.masked_attention(qb[0, h][None], kb[0, h][None], vb[0, h][None],
                                  gmask[h][None], bs, scale, [(0, i) for i in blocks])
        pos = {i: s for s, i in enumerate(blocks)}
        o_rows = np.stack([ob[pos[int(t) // bs], int(t) % bs] for t in rows])
        exact = orc.dense_attention(qb[0, h][None], kb[0, h][None], vb[0, h][None], scale,
                                    rows=[(0, int(t)) for t in probes[h]])
        corrected, _, _ = orc.probe_fit_correction(o_rows, np.arange(m), exact)
        compare_attention(got[h][samples], corrected[m:])
