"""Routing with exact ties: every query row set to zero has the same
sharpness (max cnt / sum cnt over the kept blocks), on the GPU as in the
oracle.  With most rows zero the routing threshold falls inside that tied
group, so the tie-break (lower index first) decides which of them are
routed; the routed and Taylor sets must then equal the oracle's exactly,
across the chunks of the cluster route kernel."""
import numpy as np
import pytest
import torch

import oracle
from workloads import CONFIGS, bf16_bits_to_f64, make_inputs, to_torch_bf16

from _parity import run_fused, run_stages

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N_src,N_ctx,rho,zero_frac", [(2100, 1900, 0.7, 0.6), (300, 200, 0.5, 0.8),
                                                       (13, 0, 0.4, 0.5)])
def test_tied_sharpness_routes_lower_indices_first(cuda_ok, N_src, N_ctx, rho, zero_frac):
    cfg = CONFIGS["tiny"].replace(H=2, d=64, N_src=N_src, N_ctx=N_ctx, block=64, keep=0.5, rho=rho)
    qb, kb, vb = make_inputs(cfg, 0)
    rng = np.random.default_rng(23)
    zero = rng.random(cfg.N) < zero_frac
    qb = qb.copy()
    qb[:, :, zero, :] = 0  # bf16 +0.0
    q, k, v = (to_torch_bf16(b).cuda() for b in (qb, kb, vb))
    for run in (run_stages, run_fused):
        g = run(cfg, q, k, v)
        assert g["status"] == 0
        for h in range(cfg.H):
            ref = oracle.isa_head(*(bf16_bits_to_f64(x[0, h]) for x in (qb, kb, vb)), cfg.N_src, cfg.block, cfg.keep,
                                  cfg.rho)
            kept = g["kept"][0, h] if ref["n_keep"] else np.zeros(0, np.int64)
            if kept.tolist() != ref["kept_ctx"].tolist():
                ref = oracle.isa_head(*(bf16_bits_to_f64(x[0, h]) for x in (qb, kb, vb)), cfg.N_src, cfg.block,
                                      cfg.keep, cfg.rho, kept_override=kept)
            sh = g["sharp"][0, h]
            tied = sh[zero]
            assert np.all(tied == tied[0]), "zero rows must tie exactly on the GPU"
            thr = oracle.kth_value(ref["sharp"], ref["n_route"])
            assert np.isclose(thr, ref["sharp"][zero][0]), "the threshold lies in the tied group"
            assert g["routed"][0, h].tolist() == ref["routed"].tolist()
            assert g["taylor"][0, h].tolist() == ref["taylor"].tolist()
