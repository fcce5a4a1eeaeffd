"""The pins must have teeth: plant plausible slips in a copy of the oracle and watch them fail.

Each mutant is a one-line textual change to a temporary copy of oracle/oracle.c (or, for the
numpy steps, of oracle/__init__.py), compiled into its own library and loaded as a separate
module.  The whole pin suite runs against it and at
least one pin has to fail.  The real oracle is never modified.
"""
import importlib.util
import inspect
import os
import shutil
import sys

import pytest

from tests import test_oracle_pins as pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    "pool divides by bs, not the valid count": ("double n = (double)(t1 - t0);",
                                                "double n = (double)bs;"),
    "score scale dropped": ("row[j] = s * scale;\n                if (row[j] > mx)", "row[j] = s;\n                if (row[j] > mx)"),
    "block logits scale dropped": ("row[j] = s * scale;\n            }", "row[j] = s;\n            }"),
    "top-p uses > instead of >=": ("if (cum >= topp) { m = q + 1; break; }",
                                   "if (cum > topp) { m = q + 1; break; }"),
    "top-p cut one block short": ("if (cum >= topp) { m = q + 1; break; }",
                                  "if (cum >= topp) { m = q; break; }"),
    "ties go to the higher block id": ("return (x->j > y->j) - (x->j < y->j);",
                                       "return (x->j < y->j) - (x->j > y->j);"),
    "ascending instead of descending order": ("if (x->p > y->p) return -1;\n    if (x->p < y->p) return 1;",
                                              "if (x->p < y->p) return -1;\n    if (x->p > y->p) return 1;"),
    "intersection instead of union": ("(uint8_t)(in_k[j] | in_p[j])", "(uint8_t)(in_k[j] & in_p[j])"),
    "top-k keeps one block too few": ("for (int64_t q = 0; q < kk; ++q) in_k[ord[q].j] = 1;",
                                      "for (int64_t q = 0; q + 1 < kk; ++q) in_k[ord[q].j] = 1;"),
    "masked attention scale squared": ("x *= scale;\n", "x *= scale * scale;\n"),
    "masked attention not normalised": ("o[c] = acc[c] / z;", "o[c] = acc[c];"),
    "masked attention ignores the mask": ("if (!mrow[j]) continue;\n                    int64_t s1",
                                          "int64_t s1"),
    "dense attention uses the key as value": (
        "const uint16_t *vr = v + (bh * N + sk) * d;\n                for (int64_t c = 0; c < d; ++c) o[c] += e",
        "const uint16_t *vr = k + (bh * N + sk) * d;\n                for (int64_t c = 0; c < d; ++c) o[c] += e"),
    "static band one block narrower": ("if ((flags & 1) && llabs(diff) <= w) keep = 1;",
                                       "if ((flags & 1) && llabs(diff) < w) keep = 1;"),
    "static stripe one block wider": ("if ((flags & 4) && j < s) keep = 1;",
                                      "if ((flags & 4) && j <= s) keep = 1;"),
    "static diagonals only on one side": ("for (int64_t m = -(nb / p) - 1; m <= nb / p + 1 && !keep; ++m)",
                                          "for (int64_t m = 0; m <= nb / p + 1 && !keep; ++m)"),
    "squad global pass takes v, not the local outputs": (
        "softmax_mix(qr, kb, y, NULL, rows, W, d, scale, wt, out + (bh * n + t) * d);",
        "softmax_mix(qr, kb, NULL, vb, rows, W, d, scale, wt, out + (bh * n + t) * d);"),
    "squad local pass over the wrong window": ("for (int64_t x = 0; x < win; ++x) rows[x] = a * win + x;",
                                               "for (int64_t x = 0; x < win; ++x) rows[x] = ((a + 1) % W) * win + x;"),
    "centroid top-p ignores the cluster sizes": (
        "ord[j].p = size_k[j] > 0 ? (double)size_k[j] * exp(logit[j] - mx) : 0.0;",
        "ord[j].p = size_k[j] > 0 ? exp(logit[j] - mx) : 0.0;"),
    "k-means keeps the starting centroids": (
        "cent[c * d + e] = sum[c * d + e] / (double)cnt[c];",
        "cent[c * d + e] = cent[c * d + e];"),
    "cluster attention reads the first query cluster's selection": (
        "const uint8_t *row = sel + (int64_t)aq[t] * Ck;", "const uint8_t *row = sel;"),
    "pool reads the wrong channel": ("s += bf16_to_double(x[(bh * N + t) * d + c]);",
                                     "s += bf16_to_double(x[(bh * N + t) * d + (d - 1 - c)]);"),
    # the probe-fitted correction is numpy code in the module itself
    "probe fit without the affine offset": (
        "X = np.hstack([Os[P], np.ones((len(P), 1))])",
        "X = np.hstack([Os[P], np.zeros((len(P), 1))])", "__init__.py"),
    "probe residual with the wrong sign": ("R = E - Os[P]", "R = Os[P] - E", "__init__.py"),
    "probe fit keeps one residual direction": (
        "r = int(np.count_nonzero(s > rtol * s[0]))", "r = 1", "__init__.py"),
    "SVG2 cluster sizes from the query assignment": (
        "size_k = np.bincount(ak, minlength=cent_k.shape[0])",
        "size_k = np.bincount(aq, minlength=cent_k.shape[0])[:cent_k.shape[0]]", "__init__.py"),
    "probe rows misaligned with their exact outputs": (
        "o, _, _ = probe_fit_correction(o_sparse, P, exact)",
        "o, _, _ = probe_fit_correction(o_sparse, (P + 1) % N, exact)", "__init__.py"),
}


def _pin_calls():
    calls = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        params = list(inspect.signature(fn).parameters)
        if params == ["orc"]:
            calls.append((name, fn, {}))
        elif params == ["orc", "seed"]:
            for seed in range(12):
                calls.append((f"{name}[{seed}]", fn, {"seed": seed}))
    return calls


def _build_mutant(tmp_path, tag, old, new, fname="oracle.c"):
    src_dir = os.path.join(ROOT, "oracle")
    dst = tmp_path / f"oracle_mut_{tag}"
    shutil.copytree(src_dir, dst, ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    c = (dst / fname).read_text()
    assert c.count(old) >= 1, f"mutation anchor not found: {old!r}"
    (dst / fname).write_text(c.replace(old, new, 1))
    name = f"oracle_mut_{tag}"
    spec = importlib.util.spec_from_file_location(name, dst / "__init__.py")
    mod = importlib.util.module_from_spec(spec)
    sys.modules[name] = mod
    spec.loader.exec_module(mod)
    mod.build(force=True)
    return mod


@pytest.mark.parametrize("label", sorted(MUTANTS))
def test_pins_catch_mutant(tmp_path, label):
    old, new, *fname = MUTANTS[label]
    tag = "".join(ch if ch.isalnum() else "_" for ch in label)[:40]
    mod = _build_mutant(tmp_path, tag, old, new, *fname)
    failed = []
    for name, fn, kw in _pin_calls():
        try:
            fn(mod, **kw)
        except AssertionError:
            failed.append(name)
    assert failed, f"no pin caught the mutant '{label}'"
