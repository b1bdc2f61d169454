"""The software base-2 exponential used beside MUFU.EX2 in the tensor-core
forward: the committed header matches what its generator produces, and the
fp32 evaluation of the device algorithm stays within the stated relative
error bound against the mathematical 2^x."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "scaled_dot_product_saving_b200", "csrc")


def _gen():
    spec = importlib.util.spec_from_file_location("gen_exp2_poly",
                                                  os.path.join(CSRC, "gen_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _header():
    text = open(os.path.join(CSRC, "exp2_poly.h")).read()
    coeffs = [float.fromhex(h) for h in re.findall(r"kC\d+ = (0x[0-9a-fp.+-]+)f;", text)]
    bound = float(re.search(r"kMaxRelError = ([0-9.e+-]+);", text).group(1))
    return np.array(coeffs, dtype=np.float32), bound


def test_header_coefficients_match_the_fit():
    gen = _gen()
    c, _ = gen.remez(gen.DEGREE, gen.LO, gen.HI)
    coeffs, _ = _header()
    np.testing.assert_array_equal(c.astype(np.float32), coeffs)


def test_fp32_evaluation_within_bound():
    gen = _gen()
    coeffs, bound = _header()
    assert bound < 1e-4                 # far below bf16's 2^-9 rounding
    # the bound covers (-126, 16]; at -126 and below the clamp test applies
    x = np.concatenate([np.linspace(-125.99, 16.0, 1000003),
                        [0.0, -1.0, -0.5, 0.5, -125.5, 7.5, 8.0, 15.99]])
    y = gen.fp32_eval(coeffs, x).astype(np.float64)
    ref = np.exp2(x.astype(np.float32).astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() <= bound * 1.0001
    # integers are exact up to the polynomial's value at f = 0
    np.testing.assert_allclose(gen.fp32_eval(coeffs, np.array([0.0, -3.0, -20.0])),
                               [coeffs[0], coeffs[0] / 8, coeffs[0] / 2 ** 20], rtol=1e-7)


def test_clamped_below_the_normal_range():
    gen = _gen()
    coeffs, _ = _header()
    y = gen.fp32_eval(coeffs, np.array([-200.0, -np.inf], dtype=np.float32))
    assert np.all(y >= 0) and np.all(y <= 2.0 ** -125)
