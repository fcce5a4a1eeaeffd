"""Derive the polynomial the attention softmax uses for part of its 2^x evaluations.

    python block_sparse_attention_blocks_b200/csrc/fit_exp2_poly.py [degree]

Method (textbook range reduction + Remez exchange):
  2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]; 2^n is applied by adding n to
  the exponent field, and 2^f is approximated by the polynomial c0 + c1 f + ... + cd f^d that
  minimises the maximum RELATIVE error on [-1/2, 1/2] (equioscillation via the Remez exchange
  algorithm in float64).  The script prints the coefficients rounded to fp32 and the maximum
  relative error of Horner evaluation with fp32 fused multiply-adds, measured on a dense grid.

The softmax rounds P to bf16 (relative step 2^-8), so a relative error near 1e-4 is far below
what P keeps; the coefficients printed for degree 3 are the ones in attn.cu.
"""
import sys

import numpy as np


def remez(deg: int, lo: float = -0.5, hi: float = 0.5, iters: int = 40):
    n = deg + 2
    # Chebyshev extrema as the initial reference
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new reference: the extremum of each sign run of the error
        s = np.sign(err)
        idx = []
        start = 0
        for k in range(1, len(grid) + 1):
            if k == len(grid) or s[k] != s[start]:
                seg = np.arange(start, k)
                idx.append(seg[np.argmax(np.abs(err[seg]))])
                start = k
        if len(idx) < n:
            break
        # keep n alternating points with the largest errors
        while len(idx) > n:
            if abs(err[idx[0]]) < abs(err[idx[-1]]):
                idx.pop(0)
            else:
                idx.pop()
        x = grid[np.array(idx)]
    return c, np.max(np.abs(err))


def horner_fp32(c32, f):
    """Horner with fp32 fused multiply-add (exact product, one rounding per step)."""
    acc = np.full_like(f, c32[-1], dtype=np.float32)
    for ck in c32[-2::-1]:
        acc = (acc.astype(np.float64) * f.astype(np.float64) + np.float64(ck)).astype(np.float32)
    return acc


def main():
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = remez(deg)
    c32 = c.astype(np.float32)
    f = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    rel = np.abs(horner_fp32(c32, f).astype(np.float64) / 2.0 ** f.astype(np.float64) - 1.0)
    print(f"degree {deg}: minimax relative error {e:.3e} (float64), {rel.max():.3e} (fp32 Horner)")
    for k, ck in enumerate(c32):
        print(f"  c{k} = {float(ck)!r:>24}f  (0x{np.float32(ck).view(np.uint32):08x})")


if __name__ == "__main__":
    main()
