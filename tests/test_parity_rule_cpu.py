"""CPU checks of the mask parity rule itself (tests/parity.py): a mismatch far from the row's
threshold is rejected, a swap the fp32 error bound allows is accepted and reported, and the
pooling bound really bounds an fp32 sum taken in the pooling kernel's order."""
import math

import numpy as np
import pytest

from block_sparse_attention_blocks_b200.workloads import bf16_bits_to_f32, f32_to_bf16_bits
from tests.parity import compare_masks, list_from_mask, pool_error_bound, score_error_bound


def _sel(orc, rng, nb=40, d=64, k=3, p=0.8):
    qp = rng.standard_normal((1, nb, d)) * 1.5
    kp = rng.standard_normal((1, nb, d))
    return orc.select(qp, kp, k, p, 1 / math.sqrt(d)), qp, kp


def test_identical_masks_pass(orc):
    sel, qp, kp = _sel(orc, np.random.default_rng(0))
    idx, cnt = list_from_mask(sel.mask)
    st = compare_masks(sel.mask, idx, cnt, sel, score_error_bound(qp, kp, 1 / 8))
    assert st["mismatch"] == 0 and st["allowed"] == []


def test_far_mismatch_rejected(orc):
    sel, qp, kp = _sel(orc, np.random.default_rng(1))
    m = sel.mask.copy()
    r = 5
    top = int(np.nonzero(sel.rank[0, r] == 0)[0][0])  # the row's best block: far from any cut
    m[0, r, top] = 0
    idx, cnt = list_from_mask(m)
    with pytest.raises(AssertionError):
        compare_masks(m, idx, cnt, sel, score_error_bound(qp, kp, 1 / 8))


def test_swap_within_bound_allowed_and_reported(orc):
    # row of logits where the top-k threshold block and the next one differ by 1e-6: an fp32
    # path may order them either way (E covers it), and P differs by 1e-6 relative (rule a)
    nb = 12
    L = np.linspace(2.0, -2.0, nb)
    L[3] = L[2] - 1e-6
    sel = orc.select_from_logits(L[None, None], 3, 0.0)
    m = sel.mask.copy()
    assert m[0, 0, 2] == 1 and m[0, 0, 3] == 0
    m[0, 0, 2], m[0, 0, 3] = 0, 1
    idx, cnt = list_from_mask(m)
    st = compare_masks(m, idx, cnt, sel)
    assert st["near_tau"] == 2 and len(st["allowed"]) == 2
    # the same swap 1e-3 apart is outside rule (a); with a score bound of 1e-4 per block it is
    # also outside rule (b), with 1e-3 it is inside
    L[3] = L[2] - 1e-3
    sel = orc.select_from_logits(L[None, None], 3, 0.0)
    with pytest.raises(AssertionError):
        compare_masks(m, idx, cnt, sel)
    with pytest.raises(AssertionError):
        compare_masks(m, idx, cnt, sel, np.full((1, nb), 1e-4))
    st = compare_masks(m, idx, cnt, sel, np.full((1, nb), 1e-3))
    assert st["near_tau"] == 2


def _kernel_order_mean(x32, bs, d):
    """fp32 block mean in the pooling kernel's order (per-thread rows r0, r0+RPP, ..., then the
    RPP partial sums in order, then the division), emulated with numpy float32."""
    rpp = 256 // (d // 8)
    N = x32.shape[0]
    nb = (N + bs - 1) // bs
    out = np.zeros((nb, d), np.float32)
    for i in range(nb):
        blk = np.zeros((bs, d), np.float32)
        n = min(bs, N - i * bs)
        blk[:n] = x32[i * bs:i * bs + n]
        part = np.zeros((rpp, d), np.float32)
        for r0 in range(rpp):
            a = np.zeros(d, np.float32)
            for pp in range(bs // rpp):
                a = a + blk[r0 + pp * rpp]
            part[r0] = a
        s = np.zeros(d, np.float32)
        for g in range(rpp):
            s = s + part[g]
        out[i] = s / np.float32(n)
    return out


@pytest.mark.parametrize("d,bs,N", [(128, 128, 300), (64, 128, 256), (128, 64, 130), (64, 64, 64)])
def test_pool_bound_covers_kernel_order(orc, d, bs, N):
    rng = np.random.default_rng(d + bs + N)
    # wide dynamic range (magnitudes over 2^-12 .. 2^8) so that fp32 sums really round
    x = rng.standard_normal((N, d)) * np.exp2(rng.uniform(-12, 8, (N, d)))
    bits = f32_to_bf16_bits(x.astype(np.float32))
    x32 = bf16_bits_to_f32(bits).astype(np.float32)
    got = _kernel_order_mean(x32, bs, d).astype(np.float64)
    ref = orc.pool_blocks(bits[None], bs)[0]
    bound = pool_error_bound(orc, bits[None], bs)[0]
    err = np.abs(got - ref)
    assert np.all(err <= bound)
    assert err.max() > 0  # the case does exercise rounding


def test_score_bound_covers_fp32_dot(orc):
    rng = np.random.default_rng(7)
    qp = (rng.standard_normal((2, 30, 128)) * 20).astype(np.float32)
    kp = (rng.standard_normal((2, 40, 128)) * 20).astype(np.float32)
    scale = 1 / math.sqrt(128)
    ref = orc.block_logits(qp.astype(np.float64), kp.astype(np.float64), scale)
    got = np.einsum("bic,bjc->bij", qp, kp).astype(np.float32) * np.float32(scale)
    assert np.all(np.abs(got - ref) <= score_error_bound(qp, kp, scale))
