"""The oracle reproduces its committed regression record on the tiny workload
(tests/golden/tiny_oracle.json, written by tests/golden/make_golden.py)."""
import json
import os

import numpy as np

import oracle
from workloads import CONFIGS, bf16_bits_to_f64, head_inputs

HERE = os.path.dirname(os.path.abspath(__file__))


def test_oracle_matches_golden_record():
    rec = json.load(open(os.path.join(HERE, "golden", "tiny_oracle.json")))
    cfg = CONFIGS["tiny"]
    for h, g in enumerate(rec["heads"]):
        q, k, v = (bf16_bits_to_f64(x) for x in head_inputs(cfg, 0, h, rec["seed"]))
        r = oracle.isa_head(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho)
        assert r["kept_ctx"].tolist() == g["kept_ctx"]
        assert r["routed"].tolist() == g["routed"]
        assert np.allclose(r["sal_ctx"], g["sal_ctx"], rtol=1e-12)
        for i, s in g["sharp_sample"].items():
            assert abs(r["sharp"][int(i)] - s) <= 1e-12 * max(1.0, abs(s))
        for i, row in g["out_sample"].items():
            assert np.allclose(r["out"][int(i), :8], row, rtol=1e-11, atol=1e-13)
