"""Parity rules shared by the GPU tests (test infrastructure, not product code).

Masks: the GPU selection runs in fp32 and the oracle in fp64, so the two may disagree only on
blocks the rounding can flip:
  - near-threshold blocks: the block's score lies within 1e-5 relative of the score of the row's
    threshold block (the last block of the top-k set or of the top-p set):
    |L_j - L_tau| <= 1e-5 * max(|L_tau|, 1), L the block score Qp.Kp*scale.  For |L_tau| <= 1
    this is the same as the probability being within 1e-5 relative of the threshold
    probability; it is also accepted in that probability form;
  - an ambiguous top-p cut: the block just before the cut when the mass before it is within
    1e-5 of p, or the block just after it when the mass at the cut is within 1e-5 of p.
Every other block must match bit for bit.  kv_idx / kv_cnt must be exactly the ascending list
of the GPU mask's kept blocks.

Attention: with the oracle's mask injected, the bf16 output must be within max-abs 2e-2 and
mean-abs 2e-3 of the fp64 oracle.
"""
import numpy as np

REL_TAU = 1e-5
CUM_EPS = 1e-5
ATOL_MAX = 2e-2
ATOL_MEAN = 2e-3


def compare_masks(gpu_mask, gpu_idx, gpu_cnt, sel):
    """Return a dict of counts; raise AssertionError on a mismatch the rule does not allow."""
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
    kk = min(int(sel.topk), nb)
    rows, cols = np.nonzero(gm != om)
    stats = {"rows": gm.shape[0], "blocks": gm.size, "mismatch": int(rows.size), "near_tau": 0,
             "ambiguous_cut": 0, "oracle_kept": int(om.sum()), "gpu_kept": int(gm.sum())}
    p = sel.topp
    for r, j in zip(rows.tolist(), cols.tolist()):
        pj = P[r, j]
        near = False
        if sel.topk > 0 and np.isfinite(tk[r]) and abs(pj - tk[r]) <= REL_TAU * tk[r]:
            near = True
        if mp[r] > 0 and np.isfinite(tp[r]) and abs(pj - tp[r]) <= REL_TAU * tp[r]:
            near = True
        if not near and L is not None:
            for thr_rank in ((kk - 1) if kk > 0 else None, (mp[r] - 1) if mp[r] > 0 else None):
                if thr_rank is None:
                    continue
                jt = np.nonzero(rank[r] == thr_rank)[0][0]
                lt = L[r, jt]
                if abs(L[r, j] - lt) <= REL_TAU * max(abs(lt), 1.0):
                    near = True
        if near:
            stats["near_tau"] += 1
            continue
        rk = rank[r, j]
        if 0.0 < p < 1.0 and ((rk == mp[r] - 1 and p - lo[r] <= CUM_EPS)
                              or (rk == mp[r] and hi[r] - p <= CUM_EPS)):
            stats["ambiguous_cut"] += 1
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
