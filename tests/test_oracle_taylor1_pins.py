"""Pins of the oracle's first-order Taylor variant of stage 4 against facts
that do not come from its block algebra: a per-token double loop of the
linearised weights, exactness when the keys of a block are equal, library
attention, the closed form at q = 0, and the order of the approximation
(error quadratic in the spread of the keys around their block mean, where
the 0-th order error is linear)."""
import math

import numpy as np
import pytest

import oracle
from workloads import CONFIGS, bf16_bits_to_f64, head_inputs

from test_oracle_pins import block_constant, rand, sdpa


def head(cfg, h=0):
    return tuple(bf16_bits_to_f64(x) for x in head_inputs(cfg, 0, h, 0))


@pytest.mark.parametrize("N_src,N_ctx,blk,keep", [(64, 40, 16, 0.5), (50, 33, 32, 1.0)])
def test_taylor1_equals_per_token_linearised_weights(N_src, N_ctx, blk, keep):
    """Weight of key j in block b: e^{s q.Kbar_b} (1 + s q.(k_j - Kbar_b)),
    summed token by token in a double loop (numerator and denominator),
    without the C_b matrices or the vanishing of the linear denominator."""
    cfg = CONFIGS["tiny"].replace(N_src=N_src, N_ctx=N_ctx, block=blk, d=16)
    q, k, v = head(cfg)
    r = oracle.isa_head(q, k, v, N_src, blk, keep, 0.0, taylor_order=1)
    starts, cnts = oracle.block_layout(N_src, N_ctx, blk)[:2]
    s = 1.0 / math.sqrt(cfg.d)
    ref = np.empty_like(r["out"])
    for i in range(len(q)):
        num = np.zeros(cfg.d)
        den = 0.0
        for b in r["kept_blocks"]:
            kb = k[starts[b]:starts[b] + cnts[b]].mean(axis=0)
            e = math.exp(s * q[i] @ kb)
            for j in range(starts[b], starts[b] + cnts[b]):
                w = e * (1.0 + s * q[i] @ (k[j] - kb))
                num += w * v[j]
                den += w
        ref[i] = num / den
    assert np.allclose(r["out"], ref, rtol=1e-10, atol=1e-12)


def test_taylor1_exact_for_constant_key_blocks():
    N_src, N_ctx, blk, d = 130, 60, 32, 16
    starts, cnts, nSB, nCB = oracle.block_layout(N_src, N_ctx, blk)
    k = block_constant(rand((len(cnts), d), 30), cnts)
    q, v = rand((N_src + N_ctx, d), 31), rand((N_src + N_ctx, d), 32)
    r = oracle.isa_head(q, k, v, N_src, blk, 0.5, 0.0, taylor_order=1)
    assert np.abs(r["C"]).max() < 1e-12
    mask = np.zeros((len(q), len(q)), dtype=bool)
    mask[:, r["tokens"]] = True
    assert np.allclose(r["out"], sdpa(q, k, v, mask=mask), rtol=1e-10, atol=1e-12)


def test_taylor1_block1_is_exact():
    cfg = CONFIGS["tiny"]
    q, k, v = head(cfg)
    r = oracle.isa_head(q, k, v, cfg.N_src, 1, 1.0, 0.0, taylor_order=1)
    assert np.allclose(r["out"], sdpa(q, k, v), rtol=1e-10, atol=1e-12)


def test_taylor1_zero_query_gives_mean_of_kept_values():
    cfg = CONFIGS["tiny"]
    q, k, v = head(cfg)
    q = np.zeros_like(q)
    r = oracle.isa_head(q, k, v, cfg.N_src, cfg.block, 0.5, 0.25, taylor_order=1)
    assert np.allclose(r["out"], v[r["tokens"]].mean(axis=0)[None, :], rtol=1e-12, atol=1e-13)


def test_correction_matrix_hand_example():
    """Two tokens, d = 1: k = (1, 3) -> deviations (-1, 1); v = (5, 7):
    C = -1*5 + 1*7 = 2."""
    k = np.array([[1.0], [3.0]])
    v = np.array([[5.0], [7.0]])
    C = oracle.correction_matrices(k, v, np.array([0]), np.array([2]), [0])
    assert C.shape == (1, 1, 1) and C[0, 0, 0] == 2.0


def test_taylor1_error_is_second_order_in_key_spread():
    """Keys k_j = Kbar_b + eps * delta_j: against library attention over the
    same keys, the 0-th order error falls like eps and the first-order error
    like eps^2."""
    N_src, N_ctx, blk, d = 96, 64, 32, 16
    starts, cnts, nSB, nCB = oracle.block_layout(N_src, N_ctx, blk)
    N = N_src + N_ctx
    centres = block_constant(rand((len(cnts), d), 40), cnts)
    delta = rand((N, d), 41)
    for s0, c in zip(starts, cnts):
        delta[s0:s0 + c] -= delta[s0:s0 + c].mean(axis=0)
    q, v = rand((N, d), 42), rand((N, d), 43)

    def errs(eps):
        k = centres + eps * delta
        exact = sdpa(q, k, v)
        e = []
        for order in (0, 1):
            r = oracle.isa_head(q, k, v, N_src, blk, 1.0, 0.0, taylor_order=order)
            e.append(np.abs(r["out"] - exact).max())
        return e

    (a0, a1), (b0, b1) = errs(0.02), errs(0.01)
    assert 1.8 < a0 / b0 < 2.2, (a0, b0)
    assert 3.6 < a1 / b1 < 4.4, (a1, b1)
    assert b1 < 0.1 * b0


def test_taylor1_closer_to_full_attention_on_the_workload():
    """On the synthetic DiT-latent inputs the first-order rows are closer to
    full attention over the kept tokens than the 0-th order rows."""
    cfg = CONFIGS["small"]
    q, k, v = head(cfg)
    r0 = oracle.isa_head(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho, taylor_order=0)
    r1 = oracle.isa_head(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho, taylor_order=1)
    t = r0["taylor"]
    full = oracle.full_rows(q[t], k[r0["tokens"]], v[r0["tokens"]], r0["scale"])
    e0 = np.abs(r0["out"][t] - full).sum()
    e1 = np.abs(r1["out"][t] - full).sum()
    assert e1 < 0.85 * e0, (e0, e1)
