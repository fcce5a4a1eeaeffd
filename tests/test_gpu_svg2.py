"""GPU parity of the semantic-aware permutation path (Sparse VideoGen2, method sections A-C)
against the oracle: the stable sort by cluster, k-means, centroid top-p, attention over the
selected clusters, and the whole path.  All calls go through the C ABI via the Python binding.

Decisions the GPU takes in fp32 (nearest centroid, the top-p cut) are compared with the fp64
oracle under the same rule as the block masks: a difference is allowed only where the two
candidates are within 1e-5 relative of each other (or the cumulative share is within 1e-5 of p);
everything else must match exactly."""
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
REL = 1e-5


def _dev_bits(bits):
    return torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16).to(DEV)


def _host_bf16(t):
    return bf16_bits_to_f32(t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16))


def _blobs(rng, BH, N, d, C, norm=10.0, noise=0.3, skew=False):
    """Token rows around C well-separated centres per head; returns (bits [BH, N, d], labels)."""
    centres = rng.standard_normal((BH, C, d))
    centres *= norm / np.linalg.norm(centres, axis=-1, keepdims=True)
    if skew:  # uneven cluster sizes
        w = rng.dirichlet(np.full(C, 0.5), size=BH)
        lab = np.stack([rng.choice(C, N, p=w[b]) for b in range(BH)])
    else:
        lab = rng.integers(0, C, (BH, N))
    x = np.take_along_axis(centres, lab[..., None], 1) + noise * rng.standard_normal((BH, N, d))
    return f32_to_bf16_bits(x.astype(np.float32)), lab, centres


# ---------------------------------------------------------------------------------------------
# the permutation (section A)
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("N,C", [(1, 1), (1000, 7), (5000, 100), (3000, 1024), (777, 1)])
def test_cluster_sort_is_the_stable_order(N, C):
    rng = np.random.default_rng(N + C)
    BH = 3
    a = rng.integers(0, C, (BH, N)).astype(np.int32)
    if C > 4:
        a[1] = np.minimum(a[1], 3)           # most clusters empty in one head
    perm, cs, cz = bsa.cluster_sort(torch.from_numpy(a).reshape(1, BH, N).to(DEV), C)
    perm, cs, cz = (t.cpu().numpy().reshape(BH, -1) for t in (perm, cs, cz))
    for h in range(BH):
        assert np.array_equal(perm[h], np.argsort(a[h], kind="stable"))
        size = np.bincount(a[h], minlength=C)
        assert np.array_equal(cz[h], size)
        assert np.array_equal(cs[h], np.concatenate([[0], np.cumsum(size)[:-1]]))


# ---------------------------------------------------------------------------------------------
# k-means (section A, warm start of section C)
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("d,N,C,iters", [(64, 1000, 8, 3), (128, 3001, 40, 2), (128, 700, 300, 1)])
def test_kmeans_matches_oracle_on_separated_clusters(orc, d, N, C, iters):
    rng = np.random.default_rng(d + N + C)
    BH = 2
    bits, lab, centres = _blobs(rng, BH, N, d, C, skew=True)
    # start near the centres, plus one centroid far from every token (it keeps its place)
    init = (centres + 0.5 * rng.standard_normal(centres.shape)).astype(np.float32)
    init[:, -1] = 100.0
    cent = torch.from_numpy(init.reshape(1, BH, C, d)).to(DEV)
    assign, perm, cs, cz = bsa.kmeans(_dev_bits(bits.reshape(1, BH, N, d)), cent, iters)
    torch.cuda.synchronize()
    assign = assign.cpu().numpy().reshape(BH, N)
    cent = cent.cpu().numpy().reshape(BH, C, d)
    perm = perm.cpu().numpy().reshape(BH, N)
    cz = cz.cpu().numpy().reshape(BH, C)
    xv = bf16_bits_to_f32(bits).astype(np.float64)
    for h in range(BH):
        ref_c, ref_a = orc.kmeans(xv[h], init[h].astype(np.float64), iters)
        assert np.array_equal(assign[h], ref_a)
        assert np.abs(cent[h] - ref_c).max() < 1e-4
        assert np.array_equal(cent[h, -1], init[h, -1])
        assert np.array_equal(perm[h], np.argsort(assign[h], kind="stable"))
        assert np.array_equal(cz[h], np.bincount(assign[h], minlength=C))


@pytest.mark.parametrize("d,C", [(128, 64),
                                 (64, 300),    # three 128-centroid tiles, merged per token
                                 (128, 257)])  # a last tile of one centroid
def test_kmeans_assignment_is_the_nearest_centroid(orc, d, C):
    # overlapping clusters: ties within rounding may go either way; every choice must be
    # nearest within 1e-5 relative, and with no update step the centroids stay as given
    rng = np.random.default_rng(5 + C)
    BH, N = 2, 2000
    bits = f32_to_bf16_bits(rng.standard_normal((BH, N, d)).astype(np.float32))
    init = rng.standard_normal((BH, C, d)).astype(np.float32)
    cent = torch.from_numpy(init.reshape(1, BH, C, d)).to(DEV)
    assign, _, _, _ = bsa.kmeans(_dev_bits(bits.reshape(1, BH, N, d)), cent, 0)
    torch.cuda.synchronize()
    assert np.array_equal(cent.cpu().numpy().reshape(BH, C, d), init)
    assign = assign.cpu().numpy().reshape(BH, N)
    xv = bf16_bits_to_f32(bits).astype(np.float64)
    exact = 0
    for h in range(BH):
        _, ref_a = orc.kmeans(xv[h], init[h].astype(np.float64), 0)
        dist = ((xv[h][:, None, :] - init[h][None].astype(np.float64)) ** 2).sum(-1)
        best = dist.min(1)
        got = dist[np.arange(N), assign[h]]
        assert (got <= best * (1 + REL)).all()
        exact += int((assign[h] == ref_a).sum())
    assert exact >= BH * N - 4


# ---------------------------------------------------------------------------------------------
# centroid top-p (section B)
# ---------------------------------------------------------------------------------------------
def _topp_reference(cq, ck, size, scale, p):
    """Per query cluster: the oracle's shares w (fp64), the ranked order, and the cut m."""
    out = []
    for a in range(cq.shape[0]):
        lg = scale * (ck @ cq[a])
        ok = size > 0
        mx = lg[ok].max()
        w = np.where(ok, size * np.exp(lg - mx), 0.0)
        w /= w.sum()
        order = sorted(range(len(w)), key=lambda j: (-w[j], j))
        cum, m = 0.0, 0
        for j in order:
            if w[j] <= 0 or (p < 1.0 and cum >= p):
                break
            cum += w[j]
            m += 1
        out.append((w, order, m))
    return out


def _compare_sel(got, ref, cq, ck, size, scale, p):
    near = 0
    for a, (w, order, m) in enumerate(_topp_reference(cq, ck, size, scale, p)):
        diff = np.flatnonzero(got[a] != ref[a])
        if diff.size == 0:
            continue
        cut = w[order[m - 1]] if m > 0 else w[order[0]]
        before = sum(w[j] for j in order[:max(m - 1, 0)])
        rank = {j: r for r, j in enumerate(order)}
        for j in diff:
            # near the threshold share, or the cluster next to an ambiguous cut
            ok = abs(w[j] - cut) <= REL * cut or (0.0 < p < 1.0 and (
                (rank[j] == m - 1 and abs(before - p) <= REL) or
                (rank[j] == m and abs(before + cut - p) <= REL)))
            assert ok, f"row {a} cluster {j}: gpu={got[a, j]} oracle={ref[a, j]} w={w[j]:.9g}"
            near += 1
    return near


@pytest.mark.parametrize("d,Cq,Ck,p", [(64, 20, 50, 0.9), (128, 100, 500, 0.5),
                                       (128, 64, 1024, 0.95), (64, 7, 33, 0.0), (64, 7, 33, 1.0)])
def test_centroid_topp_matches_oracle(orc, d, Cq, Ck, p):
    rng = np.random.default_rng(Cq * Ck + d)
    BH = 2
    cq = (rng.standard_normal((BH, Cq, d)) * 0.6).astype(np.float32)
    ck = (rng.standard_normal((BH, Ck, d)) * 0.6).astype(np.float32)
    size = rng.integers(0, 300, (BH, Ck)).astype(np.int32)
    size[:, ::7] = 0                                    # empty key clusters are never taken
    scale = 1 / math.sqrt(d)
    sel = bsa.centroid_topp(torch.from_numpy(cq).reshape(1, BH, Cq, d).to(DEV),
                            torch.from_numpy(ck).reshape(1, BH, Ck, d).to(DEV),
                            torch.from_numpy(size).reshape(1, BH, Ck).to(DEV), p)
    got = sel.cpu().numpy().reshape(BH, Cq, Ck)
    for h in range(BH):
        ref = orc.centroid_topp(cq[h].astype(np.float64), ck[h].astype(np.float64),
                                size[h].astype(np.int64), scale, p)
        assert not got[h][:, size[h] == 0].any()
        if p <= 0.0:
            assert not got[h].any()
        elif p >= 1.0:
            assert np.array_equal(got[h], np.broadcast_to(size[h] > 0, got[h].shape))
        _compare_sel(got[h], ref, cq[h].astype(np.float64), ck[h].astype(np.float64),
                     size[h].astype(np.float64), scale, p)


# ---------------------------------------------------------------------------------------------
# attention over the selected clusters (section C)
# ---------------------------------------------------------------------------------------------
def _cluster_case(rng, BH, N, d, Cq, Ck, density, skew=True):
    q, k, v = (f32_to_bf16_bits(rng.standard_normal((BH, N, d)).astype(np.float32))
               for _ in range(3))

    def labels(C):
        if not skew:
            return rng.integers(0, C, (BH, N)).astype(np.int32)
        w = rng.dirichlet(np.full(C, 0.3), size=BH)
        return np.stack([rng.choice(C, N, p=w[b]) for b in range(BH)]).astype(np.int32)

    aq, ak = labels(Cq), labels(Ck)
    sel = (rng.random((BH, Cq, Ck)) < density).astype(np.uint8)
    sel[:, 0, :] = 0                                    # a query cluster that selects nothing
    if Ck > 2:
        sel[:, 1, :] = 1                                # one that selects every cluster
    return q, k, v, aq, ak, sel


def _run_cluster(q, k, v, aq, ak, sel, BH, N, d):
    o = bsa.cluster_attn_fwd(_dev_bits(q.reshape(1, BH, N, d)), _dev_bits(k.reshape(1, BH, N, d)),
                             _dev_bits(v.reshape(1, BH, N, d)),
                             torch.from_numpy(aq).reshape(1, BH, N).to(DEV),
                             torch.from_numpy(ak).reshape(1, BH, N).to(DEV),
                             torch.from_numpy(sel).reshape(1, BH, *sel.shape[1:]).to(DEV))
    torch.cuda.synchronize()
    assert bsa.device_error() == 0
    return _host_bf16(o).reshape(BH, N, d)


@pytest.mark.parametrize("d,N,Cq,Ck,density", [(64, 1000, 12, 20, 0.3), (128, 1500, 5, 40, 0.2),
                                               (128, 700, 30, 3, 0.5), (64, 257, 1, 1, 1.0)])
def test_cluster_attention_matches_oracle(orc, d, N, Cq, Ck, density):
    rng = np.random.default_rng(N + Cq + Ck)
    BH = 2
    q, k, v, aq, ak, sel = _cluster_case(rng, BH, N, d, Cq, Ck, density)
    if Cq == 1:
        sel[:] = 1
    got = _run_cluster(q, k, v, aq, ak, sel, BH, N, d)
    scale = 1 / math.sqrt(d)
    for h in range(BH):
        ref = orc.cluster_attention(q[h], k[h], v[h], aq[h], ak[h], sel[h], scale)
        compare_attention(got[h], ref)
        empty = sel[h][aq[h]].astype(np.int64) @ np.bincount(ak[h], minlength=Ck) == 0
        assert not got[h][empty].any()


def test_cluster_attention_with_one_cluster_is_dense(orc):
    rng = np.random.default_rng(77)
    BH, N, d = 1, 390, 128
    q, k, v = (f32_to_bf16_bits(rng.standard_normal((BH, N, d)).astype(np.float32))
               for _ in range(3))
    zero = np.zeros((BH, N), np.int32)
    got = _run_cluster(q, k, v, zero, zero, np.ones((BH, 1, 1), np.uint8), BH, N, d)
    ref = orc.dense_attention(q, k, v, 1 / math.sqrt(d)).reshape(BH, N, d)
    compare_attention(got, ref)


# ---------------------------------------------------------------------------------------------
# the whole path
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("d,N,Cq,Ck,p", [(64, 1200, 10, 16, 0.8), (128, 2000, 16, 48, 0.9)])
def test_svg2_path_matches_oracle(orc, d, N, Cq, Ck, p):
    rng = np.random.default_rng(N + d)
    BH, iters = 2, 3
    qb, _, qc = _blobs(rng, BH, N, d, Cq, norm=4.0, noise=0.5, skew=True)
    kb, _, kc = _blobs(rng, BH, N, d, Ck, norm=4.0, noise=0.5, skew=True)
    vb = f32_to_bf16_bits(rng.standard_normal((BH, N, d)).astype(np.float32))
    iq = (qc + 0.3 * rng.standard_normal(qc.shape)).astype(np.float32)
    ik = (kc + 0.3 * rng.standard_normal(kc.shape)).astype(np.float32)
    cq = torch.from_numpy(iq.reshape(1, BH, Cq, d)).to(DEV)
    ck = torch.from_numpy(ik.reshape(1, BH, Ck, d)).to(DEV)
    o, sel = bsa.svg2_attn_fwd(_dev_bits(qb.reshape(1, BH, N, d)), _dev_bits(kb.reshape(1, BH, N, d)),
                               _dev_bits(vb.reshape(1, BH, N, d)), cq, ck, iters, p)
    torch.cuda.synchronize()
    assert bsa.device_error() == 0
    got_o = _host_bf16(o).reshape(BH, N, d)
    got_sel = sel.cpu().numpy().reshape(BH, Cq, Ck)
    got_cq = cq.cpu().numpy().reshape(BH, Cq, d)
    got_ck = ck.cpu().numpy().reshape(BH, Ck, d)
    scale = 1 / math.sqrt(d)
    for h in range(BH):
        out, aq, ak, rcq, rck, rsel = orc.svg2_attention(qb[h], kb[h], vb[h], iq[h], ik[h], iters,
                                                         p, scale)
        assert np.abs(got_cq[h] - rcq).max() < 1e-4
        assert np.abs(got_ck[h] - rck).max() < 1e-4
        size = np.bincount(ak, minlength=Ck).astype(np.float64)
        _compare_sel(got_sel[h], rsel, rcq, rck, size, scale, p)
        # attention with the GPU's selection (identical to the oracle's away from the cut)
        ref = orc.cluster_attention(qb[h], kb[h], vb[h], aq, ak, got_sel[h], scale)
        compare_attention(got_o[h], ref)
