"""The FMA-pipe 2^x used by the prefill softmax (ex2_poly2 in csrc/sm100.cuh).

Checked on the host in float32 arithmetic that mirrors the device code:
Cody-Waite range reduction with the 1.5 * 2^23 rounding constant, a degree-3
polynomial on [-1/2, 1/2], and the exponent added as an integer.  The
coefficients in the header must be the ones the committed Remez fit produces,
and the result must stay within the fit's relative error bound over the whole
input range the kernel feeds it (x in [-125, 8]).
"""

import os
import re

import numpy as np

from sliding_window_sparse_b200 import fit_exp2_poly

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "sliding_window_sparse_b200", "csrc", "sm100.cuh")


def header_coefficients():
    text = open(HEADER).read()
    body = text[text.index("float2 ex2_poly2"):]
    body = body[body.index("float2 p ="):body.index("return make_float2")]
    vals = [float(v) for v in re.findall(r"make_float2\(([0-9.e+-]+)f, \1f\)", body)]
    # order in the source: c3, c2, c1, c0
    c3, c2, c1, c0 = vals[:4]
    return np.array([c0, c1, c2, c3], dtype=np.float32)


def emulate(x):
    """float32 mirror of ex2_poly2 for an array of inputs."""
    x = np.asarray(x, dtype=np.float32)
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    r = (t - magic).astype(np.float32)
    f = (x - r).astype(np.float32)
    c = header_coefficients()
    p = np.full_like(f, c[3])
    for ci in (c[2], c[1], c[0]):
        p = (p * f + ci).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


def test_header_matches_fit():
    fitted = np.array(fit_exp2_poly.remez(), dtype=np.float32)
    assert np.array_equal(header_coefficients(), fitted)


def test_polynomial_error_bound():
    assert fit_exp2_poly.max_rel_error(header_coefficients()) < 8e-5


def test_range_reduced_exp2_matches_exp2():
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32),
                        np.array([-125.0, -1.5, -0.5, 0.0, 0.5, 1.5, 7.999, 8.0], dtype=np.float32)])
    got = emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert np.all(np.isfinite(got)) and np.all(got > 0)
    assert rel.max() < 8e-5
