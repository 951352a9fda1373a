"""The forward kernel's FMA-pipe exp2: its coefficients are the Remez minimax fit of 2^f on
[-1/2, 1/2] (csrc/fit_exp2.py), and its float32 arithmetic (reproduced in numpy) stays within
the fitted relative error over the whole clamped range, including -inf inputs."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "sequence_long_context_ring_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("fit_exp2", os.path.join(CSRC, "fit_exp2.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _kernel_coefficients():
    src = open(os.path.join(CSRC, "sm100.cuh")).read()
    body = src[src.index("void ex2_fma2("):]
    body = body[:body.index("\n}\n")]
    vals = [float(x) for x in re.findall(r"f2_pack\(([0-9.e+-]+)f, \1f\)", body)]
    vals = [v for v in vals if v != 12582912.0]  # the rounding shift 1.5 * 2^23
    # order of appearance: c3, c2, c1, c0 (Horner)
    assert len(vals) == 4, vals
    return [vals[3], vals[2], vals[1], vals[0]]


def test_kernel_coefficients_are_the_remez_fit():
    fit = _fit_module()
    c, err = fit.remez_exp2(3)
    assert err < 1e-4
    np.testing.assert_allclose(_kernel_coefficients(), c, rtol=2e-7)


def test_float32_arithmetic_error_bound_and_tail():
    fit = _fit_module()
    c = _kernel_coefficients()
    xs = np.concatenate([np.linspace(-124, 8, 200001), np.random.default_rng(0).uniform(-124, 8, 100000)])
    xs = xs.astype(np.float32)
    y = fit.exp2_poly_f32(xs, c).astype(np.float64)
    rel = np.abs(y / np.exp2(xs.astype(np.float64)) - 1)
    assert rel.max() < 8e-5
    tail = fit.exp2_poly_f32(np.array([-125, -126, -127, -1e30, -np.inf], np.float32), c)
    assert np.all(np.isfinite(tail)) and np.all(tail >= 0) and np.all(tail < 1e-37)
