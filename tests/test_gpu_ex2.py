"""The exponentials of the attention softmax on the GPU, against float64
2^x and CUDA's exp2f: the FMA-pipe 2^x (Cody-Waite reduction, minimax cubic
from tests/golden/ex2_cubic_fit.py) that takes 3 of every 16 exponential
pairs of the full-attention kernel, and the MUFU ex2 that takes the rest."""
import numpy as np
import pytest
import torch

from sparse_attention_context_b200 import api

pytestmark = pytest.mark.gpu

POLY_REL = 1.5e-4  # minimax 7.5e-5 plus fp32 evaluation of the cubic


def arguments():
    dense = np.linspace(-126.0, 32.0, 1_000_001)
    ints = np.arange(-126, 33, dtype=np.float64)
    # integers, and the points where n = rint(x) changes (ties to even) and their neighbours
    halves = ints[:-1] + 0.5
    near = np.concatenate([halves, np.nextafter(halves.astype(np.float32), np.float32(-1e9)),
                           np.nextafter(halves.astype(np.float32), np.float32(1e9))])
    edges = np.array([-126.0, -125.9999, -125.5, -0.5, -1e-7, 0.0, 1e-7, 0.5, 31.5, 32.0])
    x = np.concatenate([dense, ints, near, edges]).astype(np.float32)
    return x


def test_fma_pipe_exp2_bound(cuda_ok):
    x = arguments()
    yp, ym, yr = (t.cpu().numpy().astype(np.float64) for t in api.isa_selftest_ex2(torch.from_numpy(x).cuda()))
    truth = np.exp2(x.astype(np.float64))
    rel = np.abs(yp / truth - 1.0)
    worst = int(np.argmax(rel))
    assert rel.max() <= POLY_REL, (float(x[worst]), float(rel.max()))
    # beside CUDA's exp2f (itself within a few ulp of 2^x)
    assert np.all(np.abs(yp / yr - 1.0) <= POLY_REL + 1e-6)
    # the MUFU path the other pairs take is far tighter
    assert np.all(np.abs(ym / truth - 1.0) <= 1e-6)
    # monotone non-decreasing over the sorted dense grid (no jumps at the reduction's seams)
    n = 1_000_001
    assert np.all(np.diff(yp[:n]) >= 0)


def test_fma_pipe_exp2_clamps_below(cuda_ok):
    """Arguments below -126 (including -inf) give the value at -126, a
    positive number near 2^-126 that a softmax row sum never notices."""
    x = np.array([-126.0, -127.0, -200.0, -1e30, -np.inf], dtype=np.float32)
    yp, _, _ = (t.cpu().numpy() for t in api.isa_selftest_ex2(torch.from_numpy(x).cuda()))
    assert np.all(yp == yp[0]) and 0 < yp[0] < 2.0 ** -125
    assert abs(float(yp[0]) / 2.0 ** -126 - 1.0) <= POLY_REL


def test_fma_pipe_exp2_odd_count(cuda_ok):
    """An odd number of arguments: the last one is evaluated alone."""
    x = np.array([-3.25, 0.75, 5.5], dtype=np.float32)
    yp, _, _ = (t.cpu().numpy().astype(np.float64) for t in api.isa_selftest_ex2(torch.from_numpy(x).cuda()))
    assert np.all(np.abs(yp / np.exp2(x.astype(np.float64)) - 1.0) <= POLY_REL)
