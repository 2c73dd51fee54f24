"""The coefficients of the FMA-pipe 2^x in the kernels' PTX helper header
are the output of the Remez exchange in tests/golden/ex2_cubic_fit.py: the
cubic of least maximum relative error for 2^f on [-1/2, 1/2]."""
import os
import re

import numpy as np

from golden.ex2_cubic_fit import max_relative_error, remez_relative

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "sparse_attention_context_b200", "csrc", "tc_ptx.cuh")


def kernel_coefficients():
    text = open(HEADER).read()
    body = text[text.index("float2 ex2_poly2(float2 x)"):]
    body = body[:body.index("return make_float2")]
    vals = [float(v) for v in re.findall(r"make_float2\((0\.[0-9]+)f, \1f\)", body)]
    assert len(vals) == 4, vals
    return np.array(vals[::-1])  # c0, c1, c2, c3


def test_remez_fit_equioscillates_at_the_minimax_error():
    c, E = remez_relative()
    # a cubic's minimax relative error for 2^f on a unit interval: ~7.48e-5
    assert 7.4e-5 < E < 7.6e-5
    assert abs(max_relative_error(c) - E) < 1e-9
    # better than the truncated Taylor cubic and than a cubic interpolant at Chebyshev nodes
    taylor = np.array([1.0, np.log(2), np.log(2) ** 2 / 2, np.log(2) ** 3 / 6])
    assert max_relative_error(taylor) > 3 * E
    nodes = 0.5 * np.cos((2 * np.arange(4) + 1) * np.pi / 8)
    cheb = np.polyfit(nodes, np.exp2(nodes), 3)[::-1]
    assert max_relative_error(cheb) > E


def test_kernel_coefficients_are_the_fit():
    c_fit, E = remez_relative()
    c_k = kernel_coefficients()
    assert np.allclose(c_k, c_fit, rtol=0, atol=5e-11), (c_k, c_fit)
    assert max_relative_error(c_k) <= E * (1 + 1e-6)
