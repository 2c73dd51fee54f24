"""Write tests/golden/tiny_oracle.json from the float64 oracle alone.

The ISA pages print no worked example, so this fixture is a regression record
of the oracle on the tiny DiT-shaped workload (B=1, H=2, d=64, 256 source +
256 context tokens, block 64, keep 0.5, rho 0.25, seed 0): the kept context
blocks, the routed queries and a sample of output rows.  It is written only
by this script, which calls only ``oracle`` and the seeded input module.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from workloads import CONFIGS, bf16_bits_to_f64, head_inputs  # noqa: E402

SAMPLE_ROWS = [0, 1, 63, 64, 255, 256, 300, 511]


def main():
    cfg = CONFIGS["tiny"]
    heads = []
    for h in range(cfg.H):
        q, k, v = (bf16_bits_to_f64(x) for x in head_inputs(cfg, 0, h, 0))
        r = oracle.isa_head(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho)
        heads.append(dict(
            kept_ctx=r["kept_ctx"].tolist(),
            routed=r["routed"].tolist(),
            sal_ctx=[float(x) for x in r["sal_ctx"]],
            sharp_sample={str(i): float(r["sharp"][i]) for i in SAMPLE_ROWS},
            out_sample={str(i): [float(x) for x in r["out"][i, :8]] for i in SAMPLE_ROWS},
        ))
    rec = dict(config="tiny", seed=0, source="oracle.isa_head (float64)", heads=heads)
    with open(os.path.join(HERE, "tiny_oracle.json"), "w") as f:
        json.dump(rec, f, indent=1)


if __name__ == "__main__":
    main()
