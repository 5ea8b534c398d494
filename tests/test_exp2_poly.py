"""The attention kernel's polynomial 2^x (Cody-Waite range reduction + degree-3
core) against its error bound: the coefficients compiled into attn.cuh are the
ones the committed fit produces, and the kernel's fp32 arithmetic, replayed in
numpy, stays within 2e-4 relative error of 2^x on [-126, 8] (well below the
2^-9 rounding of the bf16 probabilities it feeds)."""

import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_long_sm_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("exp2_poly_fit", os.path.join(CSRC, "exp2_poly_fit.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _header_coeffs():
    src = open(os.path.join(CSRC, "attn.cuh")).read()
    return [float(re.search(rf"kExp2C{i} = ([0-9.eE+-]+)f;", src).group(1)) for i in range(4)]


def test_header_coefficients_match_the_fit():
    m = _fit_module()
    c, err = m.fit()
    assert err < 1e-4
    np.testing.assert_allclose(_header_coeffs(), [np.float32(v) for v in c], rtol=1e-6, atol=0)


def test_kernel_arithmetic_error_bound():
    m = _fit_module()
    c = _header_coeffs()
    rng = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-126.0, 8.0, 1_000_001), rng.uniform(-30, 8, 200_000),
                        np.arange(-126, 9, dtype=np.float64)]).astype(np.float32)
    y = m.eval_fp32(x, c).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 2e-4
    # masked entries (-inf) clamp to 2^-126, which vanishes next to the row's own key (>= 1)
    tiny = m.eval_fp32(np.array([-np.inf, -1e30], dtype=np.float32), c)
    assert np.all(tiny > 0) and np.all(tiny < 2e-38)
