"""GPU parity of each kernel against the fp64 oracle on small cases (several tiles, ragged tails,
edge cases).  All calls go through the C ABI via the Python binding."""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_blocks_b200.workloads import bf16_bits_to_f32, f32_to_bf16_bits
from tests.parity import (compare_attention, compare_masks, list_from_mask, pool_error_bound,
                          score_error_bound)

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import block_sparse_attention_blocks_b200 as bsa  # noqa: E402  (loads libbsa.so, fails loudly)

DEV = torch.device("cuda", 0)


def to_dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16).to(DEV)


def dev_bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def rand_bits(rng, shape, scale=1.0):
    return f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32) * np.float32(scale))


# ------------------------------------------------------------------------------------------------
# pooling
# ------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("d,bs,N", [(128, 128, 1000), (64, 128, 384), (128, 64, 777), (64, 64, 65)])
def test_pool_parity(orc, d, bs, N):
    rng = np.random.default_rng(d + bs + N)
    B, H = 2, 3
    q = rand_bits(rng, (B, H, N, d), 2.0)
    k = rand_bits(rng, (B, H, N, d), 0.5)
    qp, kp = bsa.pool_blocks(to_dev_bf16(q), to_dev_bf16(k), bs)
    torch.cuda.synchronize()
    for x, got in ((q, qp), (k, kp)):
        ref = orc.pool_blocks(x.reshape(B * H, N, d), bs).reshape(B, H, -1, d)
        g = got.cpu().numpy().astype(np.float64)
        # fp32 accumulation of n terms: |err| <= n * 2^-24 * max|x| (plus the final division)
        xf = bf16_bits_to_f32(x).astype(np.float64)
        nb = ref.shape[2]
        for i in range(nb):
            blk = np.abs(xf[:, :, i * bs:(i + 1) * bs]).max()
            n = min(bs, N - i * bs)
            tol = (n + 1) * 2.0 ** -24 * blk
            assert np.abs(g[:, :, i] - ref[:, :, i]).max() <= tol


# ------------------------------------------------------------------------------------------------
# selection
# ------------------------------------------------------------------------------------------------
def _gpu_select_logits(logits32, topk, topp):
    t = torch.from_numpy(np.ascontiguousarray(logits32, np.float32)).to(DEV)
    mask, idx, cnt = bsa.select_from_logits(t, topk, topp)
    torch.cuda.synchronize()
    return mask.cpu().numpy(), idx.cpu().numpy(), cnt.cpu().numpy()


@pytest.mark.parametrize("nb,d", [(591, 128), (130, 64), (7, 128), (256, 64)])
def test_block_scores_against_oracle(orc, nb, d):
    # tensor-core scores (bf16 x3 parts, fp32 accumulation) vs the fp64 definition; the bound is
    # fp32 accumulation of the 6 x d part products plus the three dropped ones (< 2^-24 |q k|
    # each), relative to the sum of |terms| of each dot product
    rng = np.random.default_rng(nb + d)
    B, H = 1, 2
    qp = (rng.standard_normal((B, H, nb, d)) * 2.0).astype(np.float32)
    kp = (rng.standard_normal((B, H, nb, d)) * 2.0).astype(np.float32)
    scale = 1.0 / math.sqrt(d)
    got = bsa.block_scores(torch.from_numpy(qp).to(DEV), torch.from_numpy(kp).to(DEV), scale)
    torch.cuda.synchronize()
    got = got.cpu().numpy().astype(np.float64)
    ref = orc.block_logits(qp.astype(np.float64), kp.astype(np.float64), scale)
    absum = np.einsum("bhic,bhjc->bhij", np.abs(qp.astype(np.float64)),
                      np.abs(kp.astype(np.float64))) * scale
    err = np.abs(got - ref)
    assert np.all(err <= 64 * 2.0 ** -24 * absum + 1e-30), float((err / absum).max())
    # a transposed operand or a misplaced tile would be off by O(1)
    assert float((err / absum).max()) < 1e-6


def test_select_handmade_rows(orc):
    nb = 24
    rows = []
    rows.append(np.log(np.r_[[0.5, 0.3, 0.15, 0.05], np.full(nb - 4, 1e-30)]))  # worked example
    rows.append(np.zeros(nb))  # uniform row
    sink = np.zeros(nb)
    sink[9] = 20.0
    rows.append(sink)  # single sink
    rows.append(np.arange(nb, dtype=np.float64) * -0.3)  # geometric
    rows.append(np.r_[np.full(12, 2.0), np.zeros(12)])  # ties
    L = np.array(rows, np.float32)[None, None]  # [1, 1, rows, nb] read as one head of 5 rows
    L = np.concatenate([L, np.zeros((1, 1, nb - L.shape[2], nb), np.float32)], 2)
    for k, p in [(1, 0.7), (3, 0.7), (0, 0.96), (4, 0.9), (0, 0.6), (12, 0.6), (2, 0.0),
                 (0, 1.0), (30, 0.5)]:
        m, idx, cnt = _gpu_select_logits(L, k, p)
        sel = orc.select_from_logits(L.astype(np.float64), k, p)
        compare_masks(m, idx, cnt, sel)
    # the pages' two failure modes, asserted directly on the GPU result
    m, idx, cnt = _gpu_select_logits(L, 0, 0.6)
    assert cnt[0, 0, 1] == math.ceil(0.6 * nb)  # uniform row: top-p keeps ceil(p nb)
    m, idx, cnt = _gpu_select_logits(L, 4, 0.9)
    assert set(idx[0, 0, 2, :cnt[0, 0, 2]].tolist()) == {0, 1, 2, 9}  # sink row: top-k rescues


@pytest.mark.parametrize("nb", [7, 32, 33, 100, 256, 591, 1024])
def test_select_parity_random(orc, nb):
    rng = np.random.default_rng(nb)
    B, H, d = 1, 3, 64
    qp = (rng.standard_normal((B, H, nb, d)) * rng.uniform(0.2, 1.5)).astype(np.float32)
    kp = (rng.standard_normal((B, H, nb, d)) * 1.0).astype(np.float32)
    scale = 1 / math.sqrt(d)
    for k, p in [(max(1, nb // 20), 0.9), (0, 0.5), (nb, 0.1), (3, 0.99)]:
        mask, idx, cnt = bsa.select_mask_topk_topp(torch.from_numpy(qp).to(DEV),
                                                   torch.from_numpy(kp).to(DEV), k, p)
        torch.cuda.synchronize()
        sel = orc.select(qp.astype(np.float64), kp.astype(np.float64), k, p, scale)
        err = score_error_bound(qp.reshape(B * H, nb, d), kp.reshape(B * H, nb, d), scale)
        st = compare_masks(mask.cpu().numpy(), idx.cpu().numpy(), cnt.cpu().numpy(), sel, err)
        for a in st["allowed"]:
            print(f"nb={nb} k={k} p={p}: allowed mismatch {a}")
        assert st["mismatch"] <= max(2, st["rows"] // 50), st


# ------------------------------------------------------------------------------------------------
# attention with an injected mask
# ------------------------------------------------------------------------------------------------
def _run_sparse(q, k, v, mask, bs, scale=0.0):
    idx, cnt = list_from_mask(mask)
    o = bsa.block_sparse_attn_fwd(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v),
                                  torch.from_numpy(idx).to(DEV), torch.from_numpy(cnt).to(DEV),
                                  bs, scale)
    torch.cuda.synchronize()
    assert bsa.device_error() == 0
    return bf16_bits_to_f32(dev_bits(o))


@pytest.mark.parametrize("d,bs,N", [(128, 128, 1000), (64, 128, 700), (128, 64, 515),
                                    (64, 64, 1024), (128, 128, 128), (64, 128, 1)])
def test_attention_parity_random_masks(orc, d, bs, N):
    rng = np.random.default_rng(N * 7 + d)
    B, H = 1, 2
    q = rand_bits(rng, (B, H, N, d), 1.5)
    k = rand_bits(rng, (B, H, N, d), 1.5)
    v = rand_bits(rng, (B, H, N, d))
    nb = (N + bs - 1) // bs
    mask = (rng.random((B, H, nb, nb)) < 0.4).astype(np.uint8)
    mask[0, 0, 0, :] = 1                       # a full row
    if nb > 1:
        mask[0, 1, 1, :] = 0                   # an empty row -> zeros
        mask[0, 0, nb - 1, :] = 0
        mask[0, 0, nb - 1, nb - 1] = 1         # only the ragged tail block
    o = _run_sparse(q, k, v, mask, bs).reshape(B * H, N, d)
    ref = orc.masked_attention(q.reshape(B * H, N, d), k.reshape(B * H, N, d),
                               v.reshape(B * H, N, d), mask.reshape(B * H, nb, nb), bs,
                               1 / math.sqrt(d))
    got = np.zeros_like(ref)
    for s in range(B * H * nb):
        bh, i = divmod(s, nb)
        r1 = min(bs, N - i * bs)
        got[s, :r1] = o[bh, i * bs:i * bs + r1]
    compare_attention(got, ref)
    if nb > 1:
        assert (o[1, bs:2 * bs] == 0).all()   # the empty row


def test_attention_all_blocks_equals_dense_oracle(orc):
    rng = np.random.default_rng(11)
    B, H, N, d, bs = 1, 2, 900, 128, 128
    q, k, v = (rand_bits(rng, (B, H, N, d), 1.2) for _ in range(3))
    nb = (N + bs - 1) // bs
    o_sparse = _run_sparse(q, k, v, np.ones((B, H, nb, nb), np.uint8), bs)
    od = bsa.dense_attn_fwd(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v))
    torch.cuda.synchronize()
    o_dense = bf16_bits_to_f32(dev_bits(od))
    rows = [(bh, t) for bh in range(B * H) for t in range(0, N, 7)]
    ref = orc.dense_attention(q.reshape(B * H, N, d), k.reshape(B * H, N, d),
                              v.reshape(B * H, N, d), 1 / math.sqrt(d), rows)
    for o in (o_sparse, o_dense):
        o = o.reshape(B * H, N, d)
        compare_attention(np.stack([o[bh, t] for bh, t in rows]), ref)


def test_attention_large_logits_and_constant_v(orc):
    # sharp rows (logits of order 50) exercise the online max / lazy rescale; a constant-V block
    # returns that constant up to the bf16 rounding of P (P V uses bf16 P, l sums fp32 P)
    rng = np.random.default_rng(12)
    B, H, N, d, bs = 1, 1, 512, 64, 128
    q = rand_bits(rng, (B, H, N, d), 4.0)
    k = rand_bits(rng, (B, H, N, d), 4.0)
    v = rand_bits(rng, (B, H, N, d))
    nb = 4
    mask = np.ones((B, H, nb, nb), np.uint8)
    o = _run_sparse(q, k, v, mask, bs).reshape(N, d)
    ref = orc.masked_attention(q[0], k[0], v[0], mask[0], bs, 1 / 8.0).reshape(N, d)
    compare_attention(o, ref)
    vc = f32_to_bf16_bits(np.full((B, H, N, d), 1.75, np.float32))
    mask2 = np.zeros_like(mask)
    mask2[..., 2] = 1
    o2 = _run_sparse(q, k, vc, mask2, bs)
    assert np.abs(o2 - 1.75).max() <= 1.75 * 2.0 ** -8 + 2.0 ** -7


def test_out_of_range_ids_are_clamped_and_flagged():
    B, H, N, d, bs = 1, 1, 256, 64, 128
    z = torch.zeros(B, H, N, d, device=DEV, dtype=torch.bfloat16)
    idx = torch.tensor([[[[0, 5], [1, 0]]]], dtype=torch.int32, device=DEV)
    cnt = torch.tensor([[[2, 1]]], dtype=torch.int32, device=DEV)
    bsa.block_sparse_attn_fwd(z, z, z, idx, cnt, bs)
    assert bsa.device_error() == bsa.sparse_attn.SA_ERR_INVALID_ARG
    assert bsa.device_error() == 0  # cleared


def test_bounded_wait_reports_timeout():
    bsa.set_wait_limit_ns(2_000_000)  # 2 ms
    try:
        bsa.probe_bounded_wait()
        assert bsa.device_error() == bsa.sparse_attn.SA_ERR_TIMEOUT
    finally:
        bsa.set_wait_limit_ns(0)
    assert bsa.device_error() == 0
    # the context is still usable
    x = torch.ones(4, device=DEV)
    assert float(x.sum()) == 4.0


def test_full_path_small(orc):
    rng = np.random.default_rng(13)
    B, H, N, d, bs, topk, topp = 1, 2, 1500, 128, 128, 2, 0.8
    q = rand_bits(rng, (B, H, N, d), 1.0)
    k = rand_bits(rng, (B, H, N, d), 1.0)
    v = rand_bits(rng, (B, H, N, d))
    o, (mask, idx, cnt) = bsa.sparse_attention(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v),
                                               bs, topk, topp, return_selection=True)
    torch.cuda.synchronize()
    qp = orc.pool_blocks(q.reshape(B * H, N, d), bs)
    kp = orc.pool_blocks(k.reshape(B * H, N, d), bs)
    sel = orc.select(qp, kp, topk, topp, 1 / math.sqrt(d))
    err = score_error_bound(qp, kp, 1 / math.sqrt(d), pool_error_bound(orc, q.reshape(B * H, N, d), bs),
                            pool_error_bound(orc, k.reshape(B * H, N, d), bs))
    st = compare_masks(mask.cpu().numpy(), idx.cpu().numpy(), cnt.cpu().numpy(), sel, err)
    for a in st["allowed"]:
        print(f"allowed mismatch {a}")
    gm = mask.cpu().numpy().reshape(B * H, -1, sel.mask.shape[-1])
    ref = orc.masked_attention(q.reshape(B * H, N, d), k.reshape(B * H, N, d),
                               v.reshape(B * H, N, d), gm, bs, 1 / math.sqrt(d))
    og = bf16_bits_to_f32(dev_bits(o)).reshape(B * H, N, d)
    nb = gm.shape[1]
    got = np.zeros_like(ref)
    for s in range(B * H * nb):
        bh, i = divmod(s, nb)
        r1 = min(bs, N - i * bs)
        got[s, :r1] = og[bh, i * bs:i * bs + r1]
    compare_attention(got, ref)


@pytest.mark.parametrize("B,H,N,d,bs", [(1, 3, 1500, 128, 128), (2, 11, 777, 64, 64),
                                          (1, 1, 200, 128, 128)])
def test_pool_select_fused_equals_separate_calls(B, H, N, d, bs):
    # the one-call path must give the separate calls' results bit for bit
    rng = np.random.default_rng(15)
    q = to_dev_bf16(rand_bits(rng, (B, H, N, d), 1.0))
    k = to_dev_bf16(rand_bits(rng, (B, H, N, d), 1.0))
    topk, topp = 3, 0.7
    qp, kp = bsa.pool_blocks(q, k, bs)
    mask, idx, cnt = bsa.select_mask_topk_topp(qp, kp, topk, topp)
    qp2, kp2, mask2, idx2, cnt2 = bsa.pool_select_topk_topp(q, k, bs, topk, topp)
    torch.cuda.synchronize()
    assert torch.equal(qp, qp2) and torch.equal(kp, kp2)
    assert torch.equal(mask, mask2) and torch.equal(cnt, cnt2)
    nb = cnt.shape[-1]
    c = cnt.reshape(-1).cpu().numpy()
    a1 = idx.reshape(-1, nb).cpu().numpy()
    a2 = idx2.reshape(-1, nb).cpu().numpy()
    for r in range(a1.shape[0]):
        assert np.array_equal(a1[r, :c[r]], a2[r, :c[r]])


def test_host_inputs_roundtrip(orc):
    rng = np.random.default_rng(14)
    B, H, N, d, bs = 1, 1, 600, 64, 128
    q, k, v = (rand_bits(rng, (B, H, N, d)) for _ in range(3))
    qh, kh, vh = (torch.from_numpy(x).view(torch.bfloat16).pin_memory() for x in (q, k, v))
    o = bsa.sparse_attention(qh, kh, vh, bs, 5, 1.0)
    assert not o.is_cuda
    ref = orc.dense_attention(q[0], k[0], v[0], 1 / 8.0).reshape(N, d)
    compare_attention(bf16_bits_to_f32(o.view(torch.int16).numpy().view(np.uint16))[0, 0], ref)


def test_exp2_polynomial_against_cuda_exp2():
    # the FMA-pipe 2^x of the softmax against CUDA's exp2f, over the range the softmax feeds it
    # normal results (the exponent-field add does not model subnormals, which bf16 P flushes)
    x = torch.cat([torch.linspace(-120.0, 8.0, 1_000_001, device=DEV),
                   torch.rand(1_000_000, device=DEV) * -30.0,
                   torch.tensor([0.0, -0.5, 0.5, -1.0, 8.0, -119.5], device=DEV)])
    y = bsa.sparse_attn.exp2_poly(x)
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref).abs() / ref).max().item()
    assert rel < 1e-4, rel
    tiny = bsa.sparse_attn.exp2_poly(torch.tensor([-float("inf"), -300.0, -125.7], device=DEV))
    assert (tiny >= 0).all() and tiny.max() < 2e-38


def test_host_pipeline_matches_device_path():
    # host inputs go through in head chunks with overlapped copies; the result must be the
    # device path's, bit for bit (the same kernels per head).  nb = 5: a chunk's kv_idx slice
    # starts 4 bytes off a 16-byte boundary for odd first heads.
    rng = np.random.default_rng(16)
    B, H, N, d, bs = 2, 3, 600, 128, 128
    q, k, v = (rand_bits(rng, (B, H, N, d)) for _ in range(3))
    qh, kh, vh = (torch.from_numpy(x).view(torch.bfloat16).pin_memory() for x in (q, k, v))
    out = torch.empty(qh.shape, dtype=torch.bfloat16).pin_memory()
    oh, (mh, ih, ch) = bsa.sparse_attention(qh, kh, vh, bs, 2, 0.7, out=out, chunks=4,
                                            return_selection=True)
    assert oh.data_ptr() == out.data_ptr() and not oh.is_cuda
    od, (md, idd, cd) = bsa.sparse_attention(qh.to(DEV), kh.to(DEV), vh.to(DEV), bs, 2, 0.7,
                                             return_selection=True)
    torch.cuda.synchronize()
    assert torch.equal(oh.view(torch.int16), od.cpu().view(torch.int16))
    assert torch.equal(mh.cpu(), md.cpu()) and torch.equal(ch.cpu(), cd.cpu())
