"""The keep x rho sweep workload (B=1, d=128, 32768 source + 32768 context
tokens, block 128) through the isa_forward kernels against the float64
oracle at every grid point: kept and routed sets checked whole, outputs on
sampled rows.  One head: the (b, h) are independent units, and the latency
side of the sweep (all 24 heads) is `bench.py --sweep`."""
import numpy as np
import pytest

from workloads import CONFIGS

from _parity import compare_head, inputs, run_fused

pytestmark = pytest.mark.gpu

CFG = CONFIGS["sweep"].replace(H=1)
POINTS = [(k, r) for k in (0.1, 0.25, 0.5, 1.0) for r in (0.0, 0.1, 0.2, 0.5, 1.0)]


@pytest.fixture(scope="module")
def sweep_inputs(cuda_ok):
    return inputs(CFG)


@pytest.mark.parametrize("keep,rho", POINTS)
def test_sweep_point_matches_oracle(sweep_inputs, keep, rho):
    bits, (q, k, v) = sweep_inputs
    g = run_fused(CFG, q, k, v, keep, rho)
    assert g["status"] == 0
    rng = np.random.default_rng(11)
    routed, taylor = g["routed"][0, 0], g["taylor"][0, 0]
    picks = [np.array([0, CFG.N_src - 1, CFG.N_src, CFG.N - 1])]
    if len(routed):
        picks.append(rng.choice(routed, min(64, len(routed)), replace=False))
    if len(taylor):
        picks.append(rng.choice(taylor, min(64, len(taylor)), replace=False))
    rows = np.unique(np.concatenate(picks))
    compare_head(CFG, bits, g, 0, 0, keep, rho, rows=rows)
