"""The polynomial constants in the attention softmax are the ones the fitting script derives."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_coefficients_match_the_remez_fit():
    import importlib.util

    spec = importlib.util.spec_from_file_location(
        "fit", os.path.join(ROOT, "block_sparse_attention_blocks_b200", "csrc", "fit_exp2_poly.py"))
    fit = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(fit)
    c, err = fit.remez(3)
    assert err < 8e-5
    src = open(os.path.join(ROOT, "block_sparse_attention_blocks_b200", "csrc", "ptx.cuh")).read()
    body = src[src.index("exp2_poly2"):src.index("pack_bf16_int")]
    used = sorted(set(float(v) for v in re.findall(r"(\d\.\d{6,})f", body)))
    want = sorted(float(np.float32(v)) for v in c)
    assert len(used) == 4
    for u, w in zip(used, want):
        assert abs(u - w) <= 2 * np.spacing(np.float32(w)), (u, w)
    # relative error of fp32 Horner on the reduced range
    f = np.linspace(-0.5, 0.5, 100001).astype(np.float32)
    rel = np.abs(fit.horner_fp32(np.asarray(c, np.float32), f) / 2.0 ** f.astype(np.float64) - 1)
    assert rel.max() < 8e-5
