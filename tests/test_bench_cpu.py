"""Host-side rules of bench.py that its report depends on (no GPU): the
kernel launches of the routed full-attention stage mirror the launcher's
split rule (whole waves of 256-row items, a partial last wave split along
the key tiles when that gives at least two pieces per item, then a merge),
and the counts the work model uses."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from workloads import CONFIGS  # noqa: E402


def test_full_stage_launches_480p():
    cfg = CONFIGS["480p"]
    nSB, nCB, n_keep, n_route = bench.counts(cfg)
    assert (nSB, nCB, n_keep, n_route) == (159, 159, 40, 8112)
    # 24 heads x 32 items = 768 = 5 x 148 + 28; 148 // 28 = 5 pieces of each
    # of the 28 items: whole waves, key-split pieces, merge
    assert bench.full_stage_launches(cfg, n_keep, n_route, 148) == 3


def test_full_stage_launches_whole_waves_only():
    cfg = CONFIGS["480p"].replace(H=37)  # 37 x 32 = 1184 = 8 x 148 items
    _, _, n_keep, n_route = bench.counts(cfg)
    assert bench.full_stage_launches(cfg, n_keep, n_route, 148) == 1


def test_full_stage_launches_under_one_wave_without_split():
    cfg = CONFIGS["small"]  # 12 heads x 7 items = 84 < 148: 148 // 84 = 1 piece, no split
    _, _, n_keep, n_route = bench.counts(cfg)
    assert -(-n_route // 256) * cfg.H == 84
    assert bench.full_stage_launches(cfg, n_keep, n_route, 148) == 1


def test_full_stage_launches_nothing_routed():
    cfg = CONFIGS["480p"].replace(rho=0.0)
    _, _, n_keep, n_route = bench.counts(cfg)
    assert n_route == 0 and bench.full_stage_launches(cfg, n_keep, n_route, 148) == 0


def test_work_model_480p():
    cfg = CONFIGS["480p"]
    wm = bench.work_model(cfg, kept_tokens_mean=25400.0)
    BH, N, d = 24, 40560, 128
    assert wm["dense_flops"] == 4.0 * BH * N * N * d
    assert wm["full_flops"] == 4.0 * BH * d * 8112 * 25400.0
    assert wm["fused_flops"] == 6.0 * BH * d * N * 199
    assert wm["full_bytes"] == BH * (2 * 8112 * d * 2 + 2 * 25400.0 * d * 2)
