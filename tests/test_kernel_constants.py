"""Where the kernels' polynomial constants come from (CPU, reading the
sources as text): each set is what its comment says it is, derived here
from the mathematics, and meets the error bound the comment states.

* The sampled walk's 2^r (walk.cu, draw_poly and its packed copy): the
  degree-7 Taylor polynomial, coefficients (ln 2)^i / i! rounded to fp32.
* The attention softmax's FMA-pipe 2^f (attn_tc.cu, exp2_poly2): a cubic
  fitted by least squares, with relative weighting, to 2^f at 256 Chebyshev
  nodes of [-1/2, 1/2], rounded to fp32; largest relative error below
  7.8e-5 on the interval.
"""
import math
import os
import re

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "block_draft_tree_b200", "csrc")


def _body(path, signature):
    src = open(os.path.join(CSRC, path)).read()
    start = src.index(signature)
    return src[start:src.index("\n}\n", start)]


def _hex_floats(text):
    return [float.fromhex(h) for h in re.findall(r"(-?0x[0-9a-fA-F.]+p-?\d+)f", text)]


def test_walk_polynomial_is_the_taylor_series_of_2_to_the_r():
    taylor = [float(np.float32(math.log(2) ** i / math.factorial(i))) for i in range(7, 0, -1)]
    assert _hex_floats(_body("walk.cu", "float draw_poly(float r)")) == taylor
    packed = _hex_floats(_body("walk.cu", "uint64_t draw_weight2("))
    assert packed == [c for c in taylor for _ in (0, 1)]   # each constant packed twice
    # on |r| <= 1/2 the truncated series is within 2e-8 of 2^r, relative
    r = np.linspace(-0.5, 0.5, 100001)
    p = np.polyval(np.array(taylor + [1.0]), r)
    assert np.max(np.abs(p / 2.0 ** r - 1.0)) < 2e-8


def test_attention_cubic_is_the_stated_least_squares_fit():
    body = _body("attn_tc.cu", "void exp2_poly2(")
    consts = [float(s) for s in re.findall(r"(\d\.\d+e[-+]\d+)f", body)]
    coef = consts[0::2]                     # each constant is packed twice
    assert consts[1::2] == coef and len(coef) == 4
    n = 256
    x = 0.5 * np.cos((2 * np.arange(n) + 1) * np.pi / (2 * n))   # Chebyshev nodes
    y = 2.0 ** x
    fit, *_ = np.linalg.lstsq(np.vander(x, 4) / y[:, None], np.ones(n), rcond=None)
    # the decimal constants are the fit rounded to fp32
    assert np.array_equal(np.float32(coef), np.float32(fit))
    f = np.linspace(-0.5, 0.5, 200001)
    p = np.polyval(np.array(coef, np.float32).astype(np.float64), f)
    assert np.max(np.abs(p / 2.0 ** f - 1.0)) < 7.8e-5
