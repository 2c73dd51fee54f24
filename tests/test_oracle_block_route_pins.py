"""Pins of the oracle's block-granular query grouping (whole query blocks
routed by the mean sharpness of their queries) against facts that do not
come from that code path: hand-worked block means, brute-force rank
counting, the per-token grouping it must reduce to when blocks hold one
token, and library attention for the rows it routes.
"""
import numpy as np
import pytest

import oracle
from workloads import CONFIGS, bf16_bits_to_f64, head_inputs

from test_oracle_pins import sdpa


def tiny_head(h=0, cfg=None):
    cfg = cfg or CONFIGS["tiny"]
    q, k, v = (bf16_bits_to_f64(x) for x in head_inputs(cfg, 0, h, 0))
    return cfg, q, k, v


def test_block_route_counts_closed_form():
    assert oracle.n_route_blocks_of(0.2, 318) == 64        # 480p latent: ceil(63.6)
    assert oracle.n_route_blocks_of(0.25, 8) == 2          # exact product, no round-up
    assert oracle.n_route_blocks_of(0.15, 1182) == 178     # 720p latent: ceil(177.3)
    assert oracle.n_route_blocks_of(0.0, 5) == 0 and oracle.n_route_blocks_of(1.0, 5) == 5


def test_block_mean_sharpness_hand_example():
    starts, cnts, _, _ = oracle.block_layout(5, 3, 2)       # blocks {0,1},{2,3},{4},{5,6},{7}
    s = np.arange(8, dtype=np.float64) * 0.1
    assert np.allclose(oracle.block_mean_sharpness(s, starts, cnts), [0.05, 0.25, 0.4, 0.55, 0.7])


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_block_route_matches_rank_counting(seed):
    """Routed blocks = those with fewer than n_rb blocks ranked ahead
    (higher score, or equal score and lower index), by a double loop."""
    rng = np.random.default_rng(seed)
    starts, cnts, _, _ = oracle.block_layout(1000, 333, 64)
    N = int(starts[-1] + cnts[-1])
    sharp = np.round(rng.random(N), 1)  # coarse values: many tied block means
    sharp[starts[3]:starts[3] + cnts[3]] = sharp[starts[5]:starts[5] + cnts[5]].mean()  # force ties
    sharp[starts[5]:starts[5] + cnts[5]] = sharp[starts[5]:starts[5] + cnts[5]].mean()
    for rho in (0.0, 0.1, 0.33, 0.5, 1.0):
        score, nrb, blocks = oracle.route_query_blocks(sharp, starts, cnts, rho)
        nB = len(starts)
        sel = []
        for b in range(nB):
            ahead = sum(1 for c in range(nB) if score[c] > score[b] or (score[c] == score[b] and c < b))
            if ahead < nrb:
                sel.append(b)
        assert blocks.tolist() == sel
        assert len(sel) == nrb == int(np.ceil(rho * nB - min(1e-6 * nB, 0.5)))


def test_block_route_with_one_token_blocks_is_token_route():
    """block = 1: a query block is one query, its score is its sharpness and
    the block count is N, so the grouping must equal the per-token one."""
    cfg, q, k, v = tiny_head(cfg=CONFIGS["tiny"].replace(N_src=70, N_ctx=50))
    a = oracle.isa_head(q, k, v, cfg.N_src, 1, 0.5, 0.3)
    b = oracle.isa_head(q, k, v, cfg.N_src, 1, 0.5, 0.3, granularity="block")
    assert a["routed"].tolist() == b["routed"].tolist()
    assert np.array_equal(a["out"], b["out"])


@pytest.mark.parametrize("N_src,N_ctx,blk,keep,rho", [
    (256, 256, 64, 0.5, 0.25), (300, 77, 64, 0.6, 0.3), (200, 130, 128, 1.0, 0.5)])
def test_block_route_rows_match_library(N_src, N_ctx, blk, keep, rho):
    """Routed rows are whole query blocks, their outputs equal library
    attention over the kept tokens; the other rows equal library attention
    with every kept key replaced by its block mean (0-th order Taylor)."""
    cfg = CONFIGS["tiny"].replace(N_src=N_src, N_ctx=N_ctx, block=blk)
    _, q, k, v = tiny_head(cfg=cfg)
    r = oracle.isa_head(q, k, v, N_src, blk, keep, rho, granularity="block")
    starts, cnts, nSB, nCB = oracle.block_layout(N_src, N_ctx, blk)
    nrb = oracle.n_route_blocks_of(rho, nSB + nCB)
    assert len(r["routed_blocks"]) == r["n_route_blocks"] == nrb
    # whole blocks: the routed rows are exactly the rows of the routed blocks
    want = sorted(j for b in r["routed_blocks"] for j in range(starts[b], starts[b] + cnts[b]))
    assert r["routed"].tolist() == want
    assert sorted(np.concatenate([r["routed"], r["taylor"]]).tolist()) == list(range(N_src + N_ctx))
    # every routed block scores at least as high as every other block
    sc = r["block_score"]
    others = np.setdiff1d(np.arange(len(sc)), r["routed_blocks"])
    if len(others) and nrb:
        assert sc[r["routed_blocks"]].min() >= sc[others].max()
    T = r["tokens"]
    if nrb:
        assert np.allclose(r["out"][r["routed"]], sdpa(q[r["routed"]], k[T], v[T]), rtol=1e-10, atol=1e-12)
    k_rep = np.empty_like(k)
    for s, c in zip(starts, cnts):
        k_rep[s:s + c] = k[s:s + c].mean(axis=0)
    if len(r["taylor"]):
        assert np.allclose(r["out"][r["taylor"]], sdpa(q[r["taylor"]], k_rep[T], v[T]), rtol=1e-10, atol=1e-12)


def test_block_route_rho1_is_masked_library_dense():
    cfg, q, k, v = tiny_head()
    r = oracle.isa_head(q, k, v, cfg.N_src, cfg.block, 0.5, 1.0, granularity="block")
    assert len(r["routed"]) == cfg.N
    mask = np.zeros((cfg.N, cfg.N), dtype=bool)
    mask[:, r["tokens"]] = True
    assert np.allclose(r["out"], sdpa(q, k, v, mask=mask), rtol=1e-10, atol=1e-12)
