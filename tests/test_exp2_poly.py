"""CPU check of the exp2 evaluation the prefill kernel runs on the FMA pipe for part of its
softmax: the coefficients in the kernel are the ones the fit script derives, and the same
steps (range reduction by rounding, cubic on [-1/2, 1/2], exponent add), carried out in
float32 with numpy, stay within the stated error bound of exp2."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "paged_kv_attention_verify_b200", "csrc")


def _fit():
    spec = importlib.util.spec_from_file_location("fit", os.path.join(CSRC, "exp2_poly_fit.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def kernel_coefficients():
    src = open(os.path.join(CSRC, "pkva_prefill_body.cuh")).read()
    vals = dict(re.findall(r"kExp2C(\d) = ([0-9.e+-]+)f", src))
    return [np.float32(vals[str(i)]) for i in range(4)]


def emulate(x, c):
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    n = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - n).astype(np.float32)
    q = np.float32(c[3])
    for k in (2, 1, 0):
        q = (q * f + np.float32(c[k])).astype(np.float32)
    bits = q.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32)


def test_kernel_uses_the_fitted_coefficients():
    fit = _fit().coefficients()[::-1]
    assert np.allclose(kernel_coefficients(), fit.astype(np.float32), rtol=0, atol=1e-7)


def test_fit_error_bound():
    m = _fit()
    assert m.max_rel_error(m.coefficients()) < 1.1e-4


def test_emulated_exp2_relative_error():
    c = kernel_coefficients()
    x = np.concatenate([np.linspace(-125.0, 8.0, 400001), np.array([0.0, -0.5, 0.5, -1.0, 8.0])])
    got = emulate(x.astype(np.float32), c).astype(np.float64)
    ref = np.exp2(x.astype(np.float32).astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 2e-4, rel.max()


def test_emulated_exp2_underflow_is_tiny_and_finite():
    c = kernel_coefficients()
    x = np.array([-126.0, -200.0, -1e30, -np.inf], dtype=np.float32)
    got = emulate(x, c)
    assert np.all(np.isfinite(got)) and np.all(got >= 0) and np.all(got < 2e-38)
