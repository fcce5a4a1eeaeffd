"""Parity rules shared by the GPU tests (test infrastructure, not product code).

Masks.  The problem statement this library implements lets the GPU mask differ from the fp64
oracle's only on blocks whose score is within 1e-5 relative of the row's selection threshold,
the score being the block probability P = softmax(Qp.Kp^T * scale).  The rule here:
  (a) near-threshold by probability: |P_j - P_tau| <= 1e-5 * P_tau (fp64 oracle probabilities),
      P_tau the probability of the row's threshold block (the last block of the top-k set or of
      the top-p set);
  (b) near-threshold within the fp32 path's proven error: the GPU ranks blocks by fp32 scores
      L = Qp.Kp * scale, whose error at |L| ~ 10-20 can exceed the 1e-5 of (a) (an fp32 ulp of
      20 is 1.9e-6, and L sums d products).  A block also counts as near-threshold when its fp64
      score and the threshold block's differ by no more than the sum of the two scores' proven
      error bounds, E_j + E_tau, i.e. exactly when the fp32 path may order the two either way.
      E comes from `score_error_bound` (the tensor-core score kernel's bound, plus the pooling
      kernel's bound when the GPU pooled the blocks itself); E = 0 when the GPU selected from
      the same logits the oracle did;
  (c) an ambiguous top-p cut: the block just before the cut when the mass before it is within
      1e-5 of p, or the block just after it when the mass at the cut is within 1e-5 of p (the
      GPU sums fp32 probabilities in fixed point).
Every other block must match bit for bit, and every allowed mismatch is recorded with its margin
(stats["allowed"]).  kv_idx / kv_cnt must be exactly the ascending list of the GPU mask's kept
blocks.

Attention: with the oracle's mask injected, the bf16 output must be within max-abs 2e-2 and
mean-abs 2e-3 of the fp64 oracle.
"""
import numpy as np

REL_TAU = 1e-5
CUM_EPS = 1e-5
ATOL_MAX = 2e-2
ATOL_MEAN = 2e-3
U32 = 2.0 ** -24          # unit roundoff of fp32
SCORE_ULPS = 64           # the score kernel's bound, in U32 * scale * sum_c |q_c k_c|


def pool_error_bound(orc, x_bits, bs):
    """Per-channel bound [BH, nb, d] on the GPU's fp32 block means of x_bits [BH, N, d] (bf16
    bits).  The pooling kernel sums in fp32 in a fixed order: each thread adds its bs / RPP rows
    (RPP = 256 / (d / 8) rows per pass) one after another, then the RPP partial sums are added in
    order, then the sum is divided by n.  That is (bs / RPP - 1) + (RPP - 1) roundings on
    partial sums bounded by sum |x|, plus the division, so the mean is within
    (bs / RPP + RPP) * 2^-24 * mean_t |x_tc| of the exact one (one unit of margin for the
    second-order terms).  mean |x| is the oracle's block mean of the absolute values (the bf16
    patterns with the sign bit cleared)."""
    x = np.ascontiguousarray(x_bits)
    BH, N, d = x.shape
    rpp = 256 // (d // 8)
    terms = bs // rpp + rpp
    amean = orc.pool_blocks(x & np.uint16(0x7FFF), bs)
    return terms * U32 * amean


def score_error_bound(qp, kp, scale, eq=None, ek=None):
    """Bound [BH, nbq, nbk] on |L_gpu - L| for the scores L = qp . kp * scale (fp64 qp, kp
    [BH, nb, d]).  The tensor-core score kernel computes fp32 dot products of its fp32 inputs to
    within SCORE_ULPS * 2^-24 * scale * sum_c |q_c k_c| (exact bf16 part products, fp32
    accumulation of 6 d of them, three dropped parts).  When the GPU's inputs are its own pooled
    values, within eq / ek of qp / kp per channel (pool_error_bound), the input error adds
    scale * sum_c (eq|k| + |q|ek + eq ek) and the kernel's bound is taken on the perturbed
    magnitudes."""
    aq = np.abs(np.asarray(qp, np.float64))
    ak = np.abs(np.asarray(kp, np.float64))
    if eq is None:
        eq = np.zeros_like(aq)
    if ek is None:
        ek = np.zeros_like(ak)
    mm = lambda a, b: np.einsum("bic,bjc->bij", a, b, optimize=True)
    inp = mm(eq, ak) + mm(aq, ek) + mm(eq, ek)
    kern = SCORE_ULPS * U32 * mm(aq + eq, ak + ek)
    return scale * (inp + kern)


def compare_masks(gpu_mask, gpu_idx, gpu_cnt, sel, score_err=None):
    """Return a dict of counts; raise AssertionError on a mismatch the rule does not allow.

    sel: the oracle's Selection (with its fp64 logits); score_err: the bound E of rule (b),
    [rows, nb] like the logits, or None when the GPU selected from the oracle's own logits."""
    nb = sel.mask.shape[-1]
    gm = np.asarray(gpu_mask).reshape(-1, nb)
    om = sel.mask.reshape(-1, nb)
    P = sel.prob.reshape(-1, nb)
    rank = sel.rank.reshape(-1, nb)
    tk = sel.tau_k.reshape(-1)
    tp = sel.tau_p.reshape(-1)
    mp = sel.m_p.reshape(-1)
    lo = sel.cum_lo.reshape(-1)
    hi = sel.cum_hi.reshape(-1)
    cnt = np.asarray(gpu_cnt).reshape(-1)
    idx = np.asarray(gpu_idx).reshape(-1, nb)
    assert gm.shape == om.shape
    assert set(np.unique(gm).tolist()) <= {0, 1}

    # kv_idx / kv_cnt are the GPU mask's kept ids, ascending
    pop = gm.sum(1)
    assert np.array_equal(cnt, pop), "kv_cnt differs from the mask's popcount"
    for r in range(gm.shape[0]):
        want = np.nonzero(gm[r])[0]
        got = idx[r, :cnt[r]]
        if not np.array_equal(got, want):
            raise AssertionError(f"row {r}: kv_idx {got[:16]} != mask ids {want[:16]}")

    L = None if sel.logit is None else np.asarray(sel.logit).reshape(-1, nb)
    E = None if score_err is None else np.asarray(score_err, np.float64).reshape(-1, nb)
    kk = min(int(sel.topk), nb)
    rows, cols = np.nonzero(gm != om)
    stats = {"rows": gm.shape[0], "blocks": gm.size, "mismatch": int(rows.size), "near_tau": 0,
             "ambiguous_cut": 0, "oracle_kept": int(om.sum()), "gpu_kept": int(gm.sum()),
             "allowed": []}
    p = sel.topp
    for r, j in zip(rows.tolist(), cols.tolist()):
        pj = P[r, j]
        why = None
        thresholds = []
        if kk > 0:
            thresholds.append(("k", kk - 1, tk[r]))
        if mp[r] > 0:
            thresholds.append(("p", mp[r] - 1, tp[r]))
        for name, thr_rank, ptau in thresholds:
            if np.isfinite(ptau) and abs(pj - ptau) <= REL_TAU * ptau:          # rule (a)
                why = (f"P within 1e-5 of tau_{name}", abs(pj - ptau) / ptau)
                break
            if L is not None and E is not None:                                  # rule (b)
                jt = int(np.nonzero(rank[r] == thr_rank)[0][0])
                dl = abs(L[r, j] - L[r, jt])
                if dl <= E[r, j] + E[r, jt]:
                    relp = abs(pj - ptau) / ptau if ptau > 0 else float("inf")
                    why = (f"|L_j - L_tau_{name}| = {dl:.3g} <= fp32 bound "
                           f"{E[r, j] + E[r, jt]:.3g}", relp)
                    break
        if why is not None:
            stats["near_tau"] += 1
            stats["allowed"].append((r, j, *why))
            continue
        rk = rank[r, j]
        if 0.0 < p < 1.0 and ((rk == mp[r] - 1 and p - lo[r] <= CUM_EPS)
                              or (rk == mp[r] and hi[r] - p <= CUM_EPS)):
            stats["ambiguous_cut"] += 1
            margin = p - lo[r] if rk == mp[r] - 1 else hi[r] - p
            stats["allowed"].append((r, j, f"top-p cut mass within {margin:.3g} of p", None))
            continue
        raise AssertionError(
            f"row {r} block {j}: gpu={gm[r, j]} oracle={om[r, j]} P={pj:.9g} rank={rk} "
            f"m_p={mp[r]} tau_k={tk[r]:.9g} tau_p={tp[r]:.9g} cum_lo={lo[r]:.9g} cum_hi={hi[r]:.9g}")
    return stats


def list_from_mask(mask):
    """Ascending kept-block lists (kv_idx, kv_cnt) of a 0/1 mask [..., nb, nb] (host side)."""
    m = np.asarray(mask).astype(bool)
    nb = m.shape[-1]
    flat = m.reshape(-1, nb)
    idx = np.zeros(flat.shape, np.int32)
    cnt = flat.sum(1).astype(np.int32)
    for r in range(flat.shape[0]):
        ids = np.nonzero(flat[r])[0]
        idx[r, :ids.size] = ids
    return idx.reshape(m.shape), cnt.reshape(m.shape[:-1])


def compare_attention(gpu_o, ref):
    """gpu_o: float array of bf16 values; ref: fp64 oracle.  Returns (max_abs, mean_abs)."""
    err = np.abs(np.asarray(gpu_o, np.float64) - ref)
    mx = float(err.max()) if err.size else 0.0
    mean = float(err.mean()) if err.size else 0.0
    assert mx <= ATOL_MAX, f"max abs error {mx:.3e} > {ATOL_MAX}"
    assert mean <= ATOL_MEAN, f"mean abs error {mean:.3e} > {ATOL_MEAN}"
    return mx, mean
