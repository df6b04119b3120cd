"""The cubic the prefill softmax uses for part of its exponentials: its
coefficients in gdla_ptx.cuh are the ones the committed fit produces, and the
float32 evaluation stays within the stated error bound of exp2 over the whole
reduced range (so the bf16-rounded probabilities are unaffected)."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "differential_latent_attention_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _kernel_coeffs():
    src = open(os.path.join(CSRC, "gdla_ptx.cuh")).read()
    body = src[src.index("exp2_poly_pair"):]
    vals = [float(v) for v in re.findall(r"f2_pack\(([0-9.]+)f, \1f\)", body)]
    c3, c2, c1, c0 = vals[:4]
    return np.array([c0, c1, c2, c3], dtype=np.float32)


def test_kernel_constants_are_the_fit():
    fit = _fit_module().fit()
    np.testing.assert_array_equal(_kernel_coeffs(), fit)


def test_error_bound_over_reduced_range():
    mod = _fit_module()
    assert mod.max_rel_error(_kernel_coeffs()) < 1e-4


def _emulate(x):
    """The kernel's steps in float32/uint32 numpy: clamp, round via 1.5*2^23,
    cubic in f, exponent add."""
    c = _kernel_coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    shift = np.float32(12582912.0)
    y = (x + shift).astype(np.float32)
    n = (y - shift).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = c[3]
    for k in (2, 1, 0):
        p = (p * f + c[k]).astype(np.float32)
    bits = p.view(np.uint32) + (y.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32)


def test_full_pipeline_relative_error():
    x = np.linspace(-100.0, 8.0, 1_000_003).astype(np.float32)
    got = _emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got / ref - 1.0)) < 1e-4
    assert _emulate(np.array([-np.inf], dtype=np.float32))[0] < 1e-37
