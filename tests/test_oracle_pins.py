"""Pins for the fp64 oracle against facts that do not come from the oracle itself.

Each test checks one oracle function against a closed form, an invariant the pages state, a
brute-force enumeration, or an independent library routine (numpy / scipy / torch in float64).
The set is chosen so that a plausible slip in the oracle (a dropped term, a wrong sign or index,
a transposed operand, an off-by-one at the top-p cut, the wrong tie order) fails at least one of
them; tests/test_oracle_mutants.py compiles such slips into the C source and checks that they do.
"""
import itertools
import math

import numpy as np
import pytest

from block_sparse_attention_blocks_b200.workloads import f32_to_bf16_bits, bf16_bits_to_f32


def bits(x):
    return f32_to_bf16_bits(np.asarray(x, np.float32))


def widen(b):
    return bf16_bits_to_f32(b).astype(np.float64)


# ------------------------------------------------------------------------------------------------
# pooling: mean over the valid tokens of each block
# ------------------------------------------------------------------------------------------------
def test_pool_constant_blocks(orc):
    bs, nb, d = 16, 5, 8
    vals = np.array([1.5, -2.0, 0.25, 7.0, -0.125], np.float32)
    x = np.repeat(vals, bs)[:, None] * np.ones((1, d), np.float32)
    xp = orc.pool_blocks(bits(x)[None], bs)[0]
    assert np.array_equal(xp, np.repeat(vals.astype(np.float64)[:, None], d, 1))


def test_pool_ramp_midpoint_and_tail(orc):
    # x_t = t within the block (exact in bf16); the mean of 0..n-1 is (n-1)/2, also for the tail
    bs, N, d = 64, 64 * 3 + 10, 4
    t = np.arange(N) % bs
    x = np.repeat(t[:, None], d, 1).astype(np.float32)
    xp = orc.pool_blocks(bits(x)[None], bs)[0]
    want = np.array([31.5, 31.5, 31.5, 4.5])
    assert np.array_equal(xp[:, 0], want)
    assert xp.shape == (4, d)


def test_pool_matches_numpy_mean(orc):
    rng = np.random.default_rng(1)
    BH, N, d, bs = 3, 300, 16, 64
    xb = bits(rng.standard_normal((BH, N, d)))
    xp = orc.pool_blocks(xb, bs)
    xf = widen(xb)
    for i in range(xp.shape[1]):
        ref = xf[:, i * bs:min((i + 1) * bs, N)].mean(axis=1)
        np.testing.assert_allclose(xp[:, i], ref, rtol=0, atol=1e-14)


# ------------------------------------------------------------------------------------------------
# block probabilities: softmax(Qp Kp^T * scale) per query-block row
# ------------------------------------------------------------------------------------------------
def test_block_probs_match_scipy(orc):
    from scipy.special import softmax

    rng = np.random.default_rng(2)
    qp = rng.standard_normal((2, 7, 16))
    kp = rng.standard_normal((2, 9, 16))
    scale = 0.37
    P = orc.block_probs(qp, kp, scale)
    ref = softmax(np.einsum("bic,bjc->bij", qp, kp) * scale, axis=-1)
    np.testing.assert_allclose(P, ref, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(P.sum(-1), 1.0, rtol=0, atol=1e-12)


def test_block_logits_match_einsum_and_feed_the_probs(orc):
    from scipy.special import softmax

    rng = np.random.default_rng(22)
    qp = rng.standard_normal((3, 5, 8))
    kp = rng.standard_normal((3, 6, 8))
    L = orc.block_logits(qp, kp, 0.7)
    np.testing.assert_allclose(L, np.einsum("bic,bjc->bij", qp, kp) * 0.7, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(orc.block_probs(qp, kp, 0.7), softmax(L, axis=-1), rtol=1e-13,
                               atol=1e-15)
    np.testing.assert_allclose(orc.softmax_rows(L), softmax(L, axis=-1), rtol=1e-13, atol=1e-15)
    # asymmetric: Qp_i . Kp_j, not Kp_i . Qp_j
    L2 = orc.block_logits(np.array([[[1.0, 0.0], [0.0, 1.0]]]), np.array([[[3.0, 0.0], [0.0, 0.0]]]), 1.0)
    assert L2[0, 0, 0] == 3.0 and L2[0, 1, 0] == 0.0 and L2[0, 0, 1] == 0.0


def test_block_probs_uniform_and_two_blocks(orc):
    P = orc.block_probs(np.zeros((1, 3, 4)), np.ones((1, 5, 4)), 1.0)
    assert np.allclose(P, 0.2, rtol=0, atol=1e-15)
    # two key blocks with logits a, b: P0 = 1 / (1 + exp(b - a))
    qp = np.array([[[1.0, 0.0]]])
    kp = np.array([[[2.0, 0.0], [-1.0, 5.0]]])
    P = orc.block_probs(qp, kp, 0.5)[0, 0]
    assert abs(P[0] - 1.0 / (1.0 + math.exp(-0.5 - 1.0))) < 1e-15
    # the score uses Qp_i . Kp_j, not Kp_i . Qp_j: an asymmetric case tells them apart
    qp2 = np.array([[[1.0, 0.0], [0.0, 1.0]]])
    kp2 = np.array([[[3.0, 0.0], [0.0, 0.0]]])
    P2 = orc.block_probs(qp2, kp2, 1.0)[0]
    assert abs(P2[0, 0] - 1.0 / (1.0 + math.exp(-3.0))) < 1e-15
    assert abs(P2[1, 0] - 0.5) < 1e-15


# ------------------------------------------------------------------------------------------------
# hybrid selection: top-k union top-p (SpargeAttention2), top-p reaching p (SVG2 2.B)
# ------------------------------------------------------------------------------------------------
def _set(mask_row):
    return set(np.nonzero(mask_row)[0].tolist())


def test_select_worked_example(orc):
    # P = (0.5, 0.3, 0.15, 0.05), fed as probabilities (exact) and as logits ln P
    P = np.array([[0.5, 0.3, 0.15, 0.05]])
    s = orc.select_from_probs(P, 1, 0.7)
    assert _set(s.mask[0]) == {0, 1}
    s = orc.select_from_probs(P, 3, 0.7)
    assert _set(s.mask[0]) == {0, 1, 2}
    s = orc.select_from_probs(P, 0, 0.96)
    assert _set(s.mask[0]) == {0, 1, 2, 3}
    # cumulative mass equals p exactly: "reaches p" keeps one block
    s = orc.select_from_probs(P, 0, 0.5)
    assert _set(s.mask[0]) == {0} and s.m_p[0] == 1 and s.cum_hi[0] == 0.5
    # via logits the cut at exactly p is decided by rounding: the oracle reports the masses
    s = orc.select_from_logits(np.log(P), 0, 0.5)
    assert s.m_p[0] in (1, 2) and abs(s.cum_hi[0] - 0.5) < 1e-12 or abs(s.cum_lo[0] - 0.5) < 1e-12


def test_select_uniform_row_keeps_ceil_p_nb(orc):
    # uniform row (SpargeAttention2 Fig. 2 situation): top-p keeps ceil(p * nb), top-k keeps k
    nb = 16
    L = np.zeros((1, nb))
    s = orc.select_from_logits(L, 0, 0.6)
    assert s.cnt[0] == 10 and _set(s.mask[0]) == set(range(10))
    s = orc.select_from_logits(L, 12, 0.6)
    assert s.cnt[0] == 12 and _set(s.mask[0]) == set(range(12))
    for p in (0.05, 0.3, 0.55, 0.81, 0.99):
        s = orc.select_from_logits(np.zeros((1, 40)), 2, p)
        assert s.m_p[0] == math.ceil(p * 40 - 1e-9)


def test_select_sink_row_top_k_rescues(orc):
    # one sink block (SpargeAttention2 Fig. 3): top-p stops at the sink, top-k still keeps k
    nb = 24
    L = np.zeros((1, nb))
    L[0, 9] = 20.0
    s = orc.select_from_logits(L, 0, 0.9)
    assert _set(s.mask[0]) == {9}
    s = orc.select_from_logits(L, 4, 0.9)
    # ties among the rest resolve to the lower block ids
    assert _set(s.mask[0]) == {9, 0, 1, 2} and s.cnt[0] == 4


def test_select_k_all_or_p_one_keeps_everything(orc):
    rng = np.random.default_rng(3)
    L = rng.standard_normal((5, 13)) * 3
    for s in (orc.select_from_logits(L, 13, 0.1), orc.select_from_logits(L, 40, 0.0),
              orc.select_from_logits(L, 0, 1.0)):
        assert (s.mask == 1).all() and (s.cnt == 13).all()
    s = orc.select_from_logits(L, 0, 0.0)
    assert (s.mask == 0).all() and (s.cnt == 0).all()


def _brute_min_count(P, p):
    """Least |S| over all subsets S with sum_S P >= p (enumeration)."""
    n = len(P)
    for size in range(0, n + 1):
        for S in itertools.combinations(range(n), size):
            if P[list(S)].sum() >= p:
                return size
    return n


@pytest.mark.parametrize("seed", range(12))
def test_select_brute_force_small(orc, seed):
    rng = np.random.default_rng(100 + seed)
    nb = int(rng.integers(2, 11))
    L = rng.standard_normal(nb) * rng.choice([0.3, 1.0, 3.0])
    if seed % 3 == 0:
        L[rng.integers(nb)] += 6.0  # sink-like row
    P = orc.softmax_rows(L[None])[0]
    k = int(rng.integers(0, nb + 1))
    p = float(rng.choice([0.2, 0.5, 0.8, 0.9, 0.95]))
    s = orc.select_from_probs(P[None], k, p)
    kept = _set(s.mask[0])
    # top-p part: minimum cardinality over ALL subsets, realised by the top-ranked blocks
    m = _brute_min_count(P, p)
    assert s.m_p[0] == m
    order = sorted(range(nb), key=lambda j: (-P[j], j))
    assert set(order[:m]) <= kept
    # top-k part: the k largest probabilities
    assert set(order[:min(k, nb)]) <= kept
    # nothing else
    assert kept == set(order[:min(k, nb)]) | set(order[:m])
    # invariants: kept mass >= p; dropping the last top-p block goes below p
    assert P[list(kept)].sum() >= p - 1e-15
    if m > 0:
        assert P[order[:m - 1]].sum() < p


def test_select_random_rows_invariants(orc):
    rng = np.random.default_rng(4)
    rows, nb = 64, 97
    L = rng.standard_normal((rows, nb)) * rng.uniform(0.1, 5.0, (rows, 1))
    k, p = 7, 0.8
    s = orc.select_from_logits(L, k, p)
    P = orc.softmax_rows(L)
    for r in range(rows):
        order = np.lexsort((np.arange(nb), -P[r]))
        kept = _set(s.mask[r])
        assert set(order[:k].tolist()) <= kept
        assert P[r, list(kept)].sum() >= p
        m = s.m_p[r]
        assert np.cumsum(P[r, order])[m - 1] >= p and (m == 1 or np.cumsum(P[r, order])[m - 2] < p)
        assert s.cnt[r] == max(k, m) == len(kept)
        assert s.tau_k[r] == P[r, order[k - 1]] and s.tau_p[r] == P[r, order[m - 1]]


# ------------------------------------------------------------------------------------------------
# attention: masked softmax attention and the dense control
# ------------------------------------------------------------------------------------------------
def _rand_qkv(rng, BH, N, d, sc=1.0):
    return [bits(rng.standard_normal((BH, N, d)) * sc) for _ in range(3)]


def test_dense_matches_torch_sdpa(orc):
    import torch

    rng = np.random.default_rng(5)
    BH, N, d = 2, 150, 32
    q, k, v = _rand_qkv(rng, BH, N, d, 1.5)
    out = orc.dense_attention(q, k, v, 1 / math.sqrt(d)).reshape(BH, N, d)
    Q, K, V = (torch.from_numpy(widen(x)) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V).numpy()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_masked_all_ones_equals_dense(orc):
    rng = np.random.default_rng(6)
    BH, N, d, bs = 2, 200, 16, 64
    q, k, v = _rand_qkv(rng, BH, N, d)
    nb = (N + bs - 1) // bs
    mask = np.ones((BH, nb, nb), np.uint8)
    o = orc.masked_attention(q, k, v, mask, bs, 0.25)
    dense = orc.dense_attention(q, k, v, 0.25).reshape(BH, N, d)
    for bh in range(BH):
        for i in range(nb):
            rows = range(i * bs, min((i + 1) * bs, N))
            np.testing.assert_allclose(o[bh * nb + i, :len(rows)], dense[bh, rows.start:rows.stop],
                                       rtol=0, atol=1e-12)
            assert (o[bh * nb + i, len(rows):] == 0).all()


def test_masked_matches_torch_with_block_mask(orc):
    import torch

    rng = np.random.default_rng(7)
    BH, N, d, bs = 1, 250, 16, 64
    q, k, v = _rand_qkv(rng, BH, N, d)
    nb = 4
    mask = (rng.random((BH, nb, nb)) < 0.5).astype(np.uint8)
    mask[:, :, 0] = 1
    o = orc.masked_attention(q, k, v, mask, bs, 0.3)
    tok = np.repeat(np.repeat(mask[0], bs, 0), bs, 1)[:N, :N].astype(bool)
    Q, K, V = (torch.from_numpy(widen(x))[0] for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q[None], K[None], V[None], attn_mask=torch.from_numpy(tok)[None], scale=0.3)[0].numpy()
    for i in range(nb):
        r0, r1 = i * bs, min((i + 1) * bs, N)
        np.testing.assert_allclose(o[i, :r1 - r0], ref[r0:r1], rtol=0, atol=1e-12)


def test_masked_single_block_constant_v_and_tail_token(orc):
    rng = np.random.default_rng(8)
    N, d, bs = 129, 8, 128  # block 1 holds one token
    q, k, _ = _rand_qkv(rng, 1, N, d, 2.0)
    v = np.zeros((1, N, d), np.float32)
    v[0, :128] = 3.25
    v[0, 128] = np.arange(d) - 2.5
    vb = bits(v)
    mask = np.zeros((1, 2, 2), np.uint8)
    mask[0, 0, 0] = 1  # block 0 sees only block 0 (constant V)
    mask[0, 1, 1] = 1  # block 1 sees only the single tail token
    o = orc.masked_attention(q, k, vb, mask, bs, 0.5)
    assert np.allclose(o[0], 3.25, rtol=0, atol=1e-13)
    assert np.array_equal(o[1, 0], np.arange(d) - 2.5) and (o[1, 1:] == 0).all()
    # a block with nothing kept produces zeros
    mask[0, 1, 1] = 0
    o = orc.masked_attention(q, k, vb, mask, bs, 0.5)
    assert (o[1] == 0).all()


def test_masked_two_keys_closed_form(orc):
    N, d, bs = 2, 2, 1  # each key its own block
    q = bits([[[1.0, 2.0], [0.5, -1.0]]])
    k = bits([[[1.0, 0.0], [0.0, 1.0]]])
    v = bits([[[4.0, -2.0], [1.0, 8.0]]])
    mask = np.ones((1, 2, 2), np.uint8)
    o = orc.masked_attention(q, k, v, mask, bs, 1.0)
    for t, (x1, x2) in enumerate([(1.0, 2.0), (0.5, -1.0)]):
        w1 = 1.0 / (1.0 + math.exp(x2 - x1))
        want = w1 * np.array([4.0, -2.0]) + (1 - w1) * np.array([1.0, 8.0])
        np.testing.assert_allclose(o[t, 0], want, rtol=0, atol=1e-14)


def test_masked_key_order_invariance(orc):
    # permuting the tokens inside a kept key block leaves every output unchanged
    rng = np.random.default_rng(9)
    N, d, bs = 256, 16, 64
    q, k, v = _rand_qkv(rng, 1, N, d)
    mask = np.zeros((1, 4, 4), np.uint8)
    mask[0, :, 1] = mask[0, :, 3] = 1
    o1 = orc.masked_attention(q, k, v, mask, bs, 0.25)
    perm = np.arange(N)
    perm[64:128] = 64 + rng.permutation(64)
    o2 = orc.masked_attention(q, k[:, perm], v[:, perm], mask, bs, 0.25)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------------------------
# static block patterns (Sparse-vDiT page, section 3: diagonal, multi-diagonal, vertical stripe)
# ---------------------------------------------------------------------------------------------
def _brute_static(flags, w, p, s, nb):
    """Pure-Python statement of the three patterns on a tiny grid (modular form)."""
    m = np.zeros((nb, nb), np.uint8)
    for i in range(nb):
        for j in range(nb):
            keep = False
            if flags & 1 and abs(i - j) <= w:
                keep = True
            if flags & 2 and p > 0:
                r = (i - j) % p
                if r <= w or p - r <= w:
                    keep = True
            if flags & 4 and j < s:
                keep = True
            m[i, j] = keep
    return m


def test_static_band_row_counts(orc):
    nb, w = 37, 3
    m = orc.static_mask([(1, w, 0, 0)], 1, nb)[0, 0]
    for i in range(nb):
        assert m[i].sum() == min(i + w, nb - 1) - max(i - w, 0) + 1
    assert np.array_equal(m, m.T)


def test_static_multidiagonal_special_cases(orc):
    nb = 29
    # width 0: exactly the diagonals i - j = m p
    m = orc.static_mask([(2, 0, 5, 0)], 1, nb)[0, 0]
    i, j = np.meshgrid(np.arange(nb), np.arange(nb), indexing="ij")
    assert np.array_equal(m, ((i - j) % 5 == 0).astype(np.uint8))
    # a period longer than the grid leaves only the main band; period 1 keeps everything
    assert np.array_equal(orc.static_mask([(2, 2, 4 * nb, 0)], 1, nb),
                          orc.static_mask([(1, 2, 0, 0)], 1, nb))
    assert orc.static_mask([(2, 0, 1, 0)], 1, nb).all()
    mm = orc.static_mask([(2, 1, 7, 0)], 1, nb)[0, 0]
    assert np.array_equal(mm, mm.T)


def test_static_stripe_skip_and_union(orc):
    nb = 23
    st = orc.static_mask([(4, 0, 0, 5)], 1, nb)[0, 0]
    assert st[:, :5].all() and not st[:, 5:].any()
    assert orc.static_mask([(4, 0, 0, 99)], 1, nb).all()
    assert not orc.static_mask([(0, 9, 3, 9)], 1, nb).any()
    both = orc.static_mask([(5, 2, 0, 4)], 1, nb)
    assert np.array_equal(both, orc.static_mask([(1, 2, 0, 0)], 1, nb) |
                          orc.static_mask([(4, 0, 0, 4)], 1, nb))


def test_static_patterns_against_brute_force(orc):
    rng = np.random.default_rng(5)
    pats = [(int(rng.integers(0, 8)), int(rng.integers(0, 4)), int(rng.integers(0, 9)),
             int(rng.integers(0, 6))) for _ in range(40)]
    nb = 17
    got = orc.static_mask(pats, 2, nb)
    for h, (f, w, p, s) in enumerate(pats):
        ref = _brute_static(f, w, p, s, nb)
        assert np.array_equal(got[0, h], ref) and np.array_equal(got[1, h], ref), (f, w, p, s)


# ---------------------------------------------------------------------------------------------
# SQuad local + global attention (SQuad page, method section 1)
# ---------------------------------------------------------------------------------------------
def _squad_inputs(seed, BH=2, N=24, d=8):
    rng = np.random.default_rng(seed)
    return [f32_to_bf16_bits(rng.standard_normal((BH, N, d)).astype(np.float32)) for _ in range(3)]


def test_squad_single_window_and_unit_window_are_dense(orc):
    # one window of all n tokens: the global groups have one member, O = the local (dense)
    # attention; windows of one token: the local pass returns v, the global pass is dense
    q, k, v = _squad_inputs(1)
    dense = orc.dense_attention(q, k, v, 0.35).reshape(q.shape)
    assert np.abs(orc.squad_attention(q, k, v, 24, 0.35) - dense).max() < 1e-12
    assert np.abs(orc.squad_attention(q, k, v, 1, 0.35) - dense).max() < 1e-12


def test_squad_constant_values(orc):
    q, k, _ = _squad_inputs(2)
    v = np.broadcast_to(f32_to_bf16_bits(np.float32([[0.5, -1.25, 2.0, 0.0, 1.0, 3.0, -2.0, 0.25]])),
                        q.shape).copy()
    o = orc.squad_attention(q, k, v, 6, 0.35)
    assert np.abs(o - bf16_bits_to_f32(v[0, 0]).astype(np.float64)).max() < 1e-12


def test_squad_against_torch_reshape(orc):
    # the same operator by reshapes and fp64 softmax attention in torch
    import torch

    q, k, v = _squad_inputs(3, BH=3, N=30, d=8)
    w, scale = 5, 0.3
    BH, N, d = q.shape
    W = N // w
    tq, tk, tv = (torch.from_numpy(bf16_bits_to_f32(x).astype(np.float64)).reshape(BH, W, w, d)
                  for x in (q, k, v))
    y = torch.softmax(tq @ tk.transpose(-1, -2) * scale, dim=-1) @ tv          # within windows
    gq, gk, gy = (x.transpose(1, 2) for x in (tq, tk, y))                    # [BH, w, W, d]
    o = torch.softmax(gq @ gk.transpose(-1, -2) * scale, dim=-1) @ gy        # across windows
    ref = o.transpose(1, 2).reshape(BH, N, d).numpy()
    assert np.abs(orc.squad_attention(q, k, v, w, scale) - ref).max() < 1e-12


# ---------------------------------------------------------------------------------------------
# SVG2 semantic-aware permutation with centroid top-p (SVG2 page, method A, B and C)
# ---------------------------------------------------------------------------------------------
def _lloyd_numpy(x, init, iters):
    """Plain vectorised Lloyd's algorithm (an independent statement of the oracle's k-means)."""
    cent = init.astype(np.float64).copy()
    for it in range(iters + 1):
        dist = ((x[:, None, :] - cent[None, :, :]) ** 2).sum(-1)
        assign = dist.argmin(1)              # the lower index on a tie
        if it == iters:
            break
        for c in range(cent.shape[0]):
            if (assign == c).any():
                cent[c] = x[assign == c].mean(0)
    return cent, assign


def test_kmeans_separated_blobs_and_fixed_points(orc):
    rng = np.random.default_rng(21)
    centres = np.eye(4) * 6.0
    x = np.concatenate([rng.standard_normal((15, 4)) * 0.2 + c for c in centres[:3]])
    cent, assign = orc.kmeans(x, x[[0, 15, 30]], 6)
    assert np.array_equal(assign, np.repeat(np.arange(3), 15))
    for c in range(3):
        assert np.abs(cent[c] - x[assign == c].mean(0)).max() < 1e-12
    # a converged state does not move; one cluster per point keeps every point as its centroid
    cent2, assign2 = orc.kmeans(x, cent, 3)
    assert np.array_equal(assign2, assign) and np.abs(cent2 - cent).max() < 1e-12
    cent3, assign3 = orc.kmeans(x, x, 2)
    assert np.array_equal(assign3, np.arange(len(x))) and np.abs(cent3 - x).max() < 1e-12


def test_kmeans_against_numpy_lloyd(orc):
    rng = np.random.default_rng(22)
    x = rng.standard_normal((60, 5))
    init = x[rng.choice(60, 7, replace=False)]
    cent, assign = orc.kmeans(x, init, 4)
    ref_c, ref_a = _lloyd_numpy(x, init, 4)
    assert np.array_equal(assign, ref_a) and np.abs(cent - ref_c).max() < 1e-12


def test_centroid_topp_worked_example_and_limits(orc):
    # one query centroid at the origin gives equal logits, so the estimate is the cluster size
    # share: sizes (5, 3, 2, 0) -> (0.5, 0.3, 0.2, 0); p = 0.6 takes clusters 0 and 1
    cq = np.zeros((1, 3))
    ck = np.arange(12, dtype=np.float64).reshape(4, 3)
    size = np.array([5, 3, 2, 0])
    assert orc.centroid_topp(cq, ck, size, 1.0, 0.6).tolist() == [[1, 1, 0, 0]]
    assert orc.centroid_topp(cq, ck, size, 1.0, 0.5).tolist() == [[1, 0, 0, 0]]
    assert orc.centroid_topp(cq, ck, size, 1.0, 1.0).tolist() == [[1, 1, 1, 0]]   # not the empty one
    assert orc.centroid_topp(cq, ck, size, 1.0, 0.0).tolist() == [[0, 0, 0, 0]]
    # unit-size clusters: the estimate is the softmax of the query centroid's scores
    rng = np.random.default_rng(23)
    cq = rng.standard_normal((2, 4))
    ck = rng.standard_normal((6, 4))
    for a in range(2):
        w = np.exp(0.5 * ck @ cq[a])
        w /= w.sum()
        order = sorted(range(6), key=lambda j: (-w[j], j))
        cum, take = 0.0, []
        for j in order:
            take.append(j)
            cum += w[j]
            if cum >= 0.7:
                break
        sel = orc.centroid_topp(cq, ck, np.ones(6, np.int64), 0.5, 0.7)[a]
        assert sorted(np.flatnonzero(sel).tolist()) == sorted(take)


def test_cluster_attention_reduces_to_dense_and_block_sparse(orc):
    rng = np.random.default_rng(24)
    n, d, bs = 48, 8, 16
    q, k, v = (f32_to_bf16_bits(rng.standard_normal((n, d)).astype(np.float32)) for _ in range(3))
    dense = orc.dense_attention(q[None], k[None], v[None], 0.3).reshape(n, d)
    one = np.zeros(n, np.int32)
    assert np.abs(orc.cluster_attention(q, k, v, one, one, np.ones((1, 1), np.uint8), 0.3)
                  - dense).max() < 1e-12
    # clusters = contiguous blocks: the selection is a block mask
    blocks = (np.arange(n) // bs).astype(np.int32)
    mask = np.array([[1, 0, 1], [0, 1, 0], [1, 1, 1]], np.uint8)
    got = orc.cluster_attention(q, k, v, blocks, blocks, mask, 0.3)
    ref = orc.masked_attention(q[None], k[None], v[None], mask[None], bs, 0.3).reshape(n, d)
    assert np.abs(got - ref).max() < 1e-12


def test_svg2_one_key_per_cluster_and_full_p_is_dense(orc):
    rng = np.random.default_rng(25)
    n, d = 32, 8
    q, k, v = (f32_to_bf16_bits(rng.standard_normal((n, d)).astype(np.float32)) for _ in range(3))
    kd = bf16_bits_to_f32(k).astype(np.float64)
    qd = bf16_bits_to_f32(q).astype(np.float64)
    out, aq, ak, cq, ck, sel = orc.svg2_attention(q, k, v, qd[:4], kd, 3, 1.0, 0.3)
    assert np.array_equal(ak, np.arange(n)) and sel.all()
    dense = orc.dense_attention(q[None], k[None], v[None], 0.3).reshape(n, d)
    assert np.abs(out - dense).max() < 1e-12


# ---------------------------------------------------------------------------------------------
# SparsePR probe-fitted residual reconstruction (page "Partition the Support, Reconstruct the
# Residual", abstract and summary section 3)
# ---------------------------------------------------------------------------------------------
def test_probe_fit_recovers_a_planted_affine_residual(orc):
    # residual = [o, 1] A0 B0^T exactly, with enough probes: the fit finds the subspace of B0 and
    # the map, and the corrected output is exact on every row, not only on the probes
    rng = np.random.default_rng(31)
    n, d, r0 = 120, 8, 3
    Os = rng.standard_normal((n, d))
    A0 = rng.standard_normal((d + 1, r0))
    B0 = np.linalg.qr(rng.standard_normal((d, r0)))[0]
    exact_all = Os + np.hstack([Os, np.ones((n, 1))]) @ A0 @ B0.T
    P = rng.choice(n, 30, replace=False)
    o, Bs, A = orc.probe_fit_correction(Os, P, exact_all[P])
    assert Bs.shape == (d, r0)
    assert np.abs(Bs @ Bs.T - B0 @ B0.T).max() < 1e-9
    assert np.abs(o - exact_all).max() < 1e-9


def test_probe_fit_interpolates_few_probes_within_the_residual_subspace(orc):
    rng = np.random.default_rng(32)
    n, d = 60, 16
    Os = rng.standard_normal((n, d))
    P = np.array([3, 17, 40, 41, 59])
    E = rng.standard_normal((5, d))
    o, Bs, A = orc.probe_fit_correction(Os, P, E)
    # fewer probes than affine features: the least-squares fit matches every probe
    assert np.abs(o[P] - E).max() < 1e-9
    proj = np.eye(d) - Bs @ Bs.T
    assert np.abs((E - Os[P]) @ proj).max() < 1e-9     # the basis spans the residuals
    assert np.abs((o - Os) @ proj).max() < 1e-9        # and holds the whole correction
    # minimum norm: A lies in the row space of the probe features
    X = np.hstack([Os[P], np.ones((5, 1))])
    row_space = X.T @ np.linalg.solve(X @ X.T, X)
    assert np.abs(A - row_space @ A).max() < 1e-9
    # the order of the probes does not matter
    perm = np.array([4, 2, 0, 1, 3])
    o2, _, _ = orc.probe_fit_correction(Os, P[perm], E[perm])
    assert np.abs(o2 - o).max() < 1e-9


def test_sparsepr_attention_exact_cases(orc):
    rng = np.random.default_rng(33)
    N, d, bs, scale = 40, 8, 16, 0.3
    q, k, v = (f32_to_bf16_bits(rng.standard_normal((N, d)).astype(np.float32)) for _ in range(3))
    dense = orc.dense_attention(q[None], k[None], v[None], scale).reshape(N, d)
    # a full mask: the sparse output is already exact and nothing is corrected
    o, o_sparse = orc.sparsepr_attention(q, k, v, np.ones((3, 3), np.uint8), bs, scale, [0, 7, 39])
    assert np.abs(o_sparse - dense).max() < 1e-12 and np.abs(o - dense).max() < 1e-12
    # a diagonal mask with fewer probes than d + 1: the probe rows come out exact, the sparse
    # output is the block-masked attention
    mask = np.eye(3, dtype=np.uint8)
    P = [2, 20, 33]
    o, o_sparse = orc.sparsepr_attention(q, k, v, mask, bs, scale, P)
    ref_sparse = orc.masked_attention(q[None], k[None], v[None], mask[None], bs, scale)
    assert np.abs(o_sparse - ref_sparse.reshape(3 * bs, d)[:N]).max() < 1e-12
    assert np.abs(o[P] - dense[P]).max() < 1e-9
    assert np.abs(o_sparse[P] - dense[P]).max() > 1e-3   # the mask did drop something


def test_probe_fit_full_subspace_is_the_least_squares_fit_of_the_residuals(orc):
    # at the full numerical rank the subspace step changes nothing: the correction is the
    # minimum-norm least-squares map of the residuals (pseudo-inverse, another numpy route)
    rng = np.random.default_rng(34)
    n, d = 80, 12
    Os = rng.standard_normal((n, d))
    for m in (6, 40):
        P = rng.choice(n, m, replace=False)
        E = Os[P] + rng.standard_normal((m, d))
        o, Bs, _ = orc.probe_fit_correction(Os, P, E)
        X = np.hstack([Os[P], np.ones((m, 1))])
        W = np.linalg.pinv(X) @ (E - Os[P])
        assert np.abs(o - (Os + np.hstack([Os, np.ones((n, 1))]) @ W)).max() < 1e-9
    # a lower rank keeps the leading residual directions only
    P = rng.choice(n, 40, replace=False)
    E = Os[P] + rng.standard_normal((40, d))
    o2, B2, _ = orc.probe_fit_correction(Os, P, E, rank=2)
    _, _, vt = np.linalg.svd(E - Os[P])
    assert B2.shape == (d, 2)
    assert np.abs(B2 @ B2.T - vt[:2].T @ vt[:2]).max() < 1e-9
    proj = np.eye(d) - B2 @ B2.T
    assert np.abs((o2 - Os) @ proj).max() < 1e-9


def test_cluster_attention_against_torch_masked_sdpa(orc):
    # random clusters and selection: the same as fp64 torch attention with the token mask
    # M[t, s] = sel[aq[t], ak[s]] (rows whose mask is empty are zero)
    import torch

    rng = np.random.default_rng(26)
    n, d, Cq, Ck = 70, 8, 5, 6
    q, k, v = (f32_to_bf16_bits(rng.standard_normal((n, d)).astype(np.float32)) for _ in range(3))
    aq = rng.integers(0, Cq, n).astype(np.int32)
    ak = rng.integers(0, Ck, n).astype(np.int32)
    sel = (rng.random((Cq, Ck)) < 0.4).astype(np.uint8)
    sel[0] = 0
    got = orc.cluster_attention(q, k, v, aq, ak, sel, 0.35)
    M = torch.from_numpy(sel[aq][:, ak].astype(bool))
    t = lambda b: torch.from_numpy(widen(b))
    ref = torch.nn.functional.scaled_dot_product_attention(
        t(q)[None], t(k)[None], t(v)[None], attn_mask=M[None], scale=0.35)[0].numpy()
    empty = ~M.numpy().any(1)
    ref[empty] = 0.0
    assert np.abs(got - ref).max() < 1e-12


def test_svg2_composition_against_numpy_and_torch(orc):
    # the whole path written independently: numpy Lloyd for Q and K, the size-weighted centroid
    # shares ranked and cut in plain Python, fp64 torch attention under the token mask
    import torch

    rng = np.random.default_rng(27)
    n, d, Cq, Ck, iters, p, scale = 90, 6, 4, 7, 2, 0.8, 0.4
    q, k, v = (f32_to_bf16_bits(rng.standard_normal((n, d)).astype(np.float32)) for _ in range(3))
    qd, kd = widen(q), widen(k)
    iq = qd[rng.choice(n, Cq, replace=False)]
    ik = kd[rng.choice(n, Ck, replace=False)]
    out, aq, ak, cq, ck, sel = orc.svg2_attention(q, k, v, iq, ik, iters, p, scale)
    ref_cq, ref_aq = _lloyd_numpy(qd, iq, iters)
    ref_ck, ref_ak = _lloyd_numpy(kd, ik, iters)
    assert np.array_equal(aq, ref_aq) and np.array_equal(ak, ref_ak)
    assert np.abs(cq - ref_cq).max() < 1e-12 and np.abs(ck - ref_ck).max() < 1e-12
    size = np.bincount(ref_ak, minlength=Ck)
    ref_sel = np.zeros((Cq, Ck), np.uint8)
    for a in range(Cq):
        lg = scale * (ref_ck @ ref_cq[a])
        w = np.where(size > 0, size * np.exp(lg - lg[size > 0].max()), 0.0)
        w /= w.sum()
        cum = 0.0
        for j in sorted(range(Ck), key=lambda j: (-w[j], j)):
            if w[j] <= 0 or cum >= p:
                break
            ref_sel[a, j] = 1
            cum += w[j]
    assert np.array_equal(sel, ref_sel)
    M = torch.from_numpy(ref_sel[ref_aq][:, ref_ak].astype(bool))
    t = lambda b: torch.from_numpy(widen(b))
    ref = torch.nn.functional.scaled_dot_product_attention(
        t(q)[None], t(k)[None], t(v)[None], attn_mask=M[None], scale=scale)[0].numpy()
    ref[~M.numpy().any(1)] = 0.0
    assert np.abs(out - ref).max() < 1e-12


def test_sparsepr_composition_against_torch_and_pinv(orc):
    # block-masked and exact attention by fp64 torch, the fit by the pseudo-inverse of the
    # probe features: the oracle's SparsePR path must agree (more probes than features here)
    import torch

    rng = np.random.default_rng(35)
    N, d, bs, scale = 96, 4, 16, 0.5
    nb = N // bs
    q, k, v = (f32_to_bf16_bits(rng.standard_normal((N, d)).astype(np.float32)) for _ in range(3))
    mask = (rng.random((nb, nb)) < 0.4).astype(np.uint8)
    mask[:, 0] = 1
    P = np.sort(rng.choice(N, 20, replace=False))
    o, o_sparse = orc.sparsepr_attention(q, k, v, mask, bs, scale, P)
    t = lambda b: torch.from_numpy(widen(b))
    tok = torch.from_numpy(np.kron(mask, np.ones((bs, bs), np.uint8)).astype(bool))
    sp = torch.nn.functional.scaled_dot_product_attention(
        t(q)[None], t(k)[None], t(v)[None], attn_mask=tok[None], scale=scale)[0].numpy()
    ex = torch.nn.functional.scaled_dot_product_attention(
        t(q)[None], t(k)[None], t(v)[None], scale=scale)[0].numpy()
    assert np.abs(o_sparse - sp).max() < 1e-12
    X = np.hstack([sp[P], np.ones((len(P), 1))])
    W = np.linalg.pinv(X) @ (ex[P] - sp[P])
    assert np.abs(o - (sp + np.hstack([sp, np.ones((N, 1))]) @ W)).max() < 1e-9
