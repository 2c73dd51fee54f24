"""Pins of the float64 oracle against facts that do not come from the oracle.

Every check below compares the oracle with something independent of it:
hand-worked closed forms, brute-force rank counting, or token-level attention
computed by torch's scaled_dot_product_attention (a library routine) on
inputs where the block-level formulas of the ISA reading must reduce to it.
Sizes are ragged on purpose (partial last blocks), so a dropped ln(cnt) bias
or a wrong count weight changes the result.
"""
import math

import numpy as np
import pytest
import torch
from scipy.stats import spearmanr

import oracle
from workloads import CONFIGS, bf16_bits_to_f64, head_inputs

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


def sdpa(q, k, v, mask=None, scale=None):
    """Library attention in float64 on the CPU."""
    tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(x))[None, None] for x in (q, k, v))
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=m, scale=scale)
    return o[0, 0].numpy()


def token_attention_matrix(q, k, scale=None):
    """softmax(s q k^T) obtained from the library by attending to the identity."""
    return sdpa(q, k, np.eye(k.shape[0]), scale=scale)


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def block_constant(x_blocks, cnts):
    """Expand per-block rows to a token-level array (each block's rows equal)."""
    return np.concatenate([np.repeat(x_blocks[b:b + 1], c, axis=0) for b, c in enumerate(cnts)])


# --------------------------------------------------------------------- counts
def test_counts_closed_form():
    assert oracle.n_keep_of(0.25, 256) == 64          # exact product, no round-up
    assert oracle.n_keep_of(0.3, 32) == 10            # ceil(9.6)
    assert oracle.n_keep_of(0.25, 159) == 40          # 480p latent: ceil(39.75)
    assert oracle.n_keep_of(0.0, 10) == 0 and oracle.n_keep_of(1.0, 10) == 10
    assert oracle.n_route_of(0.2, 40560) == 8112
    assert oracle.n_route_of(0.25, 512) == 128
    assert oracle.n_route_of(0.15, 151200) == 22680
    assert oracle.n_route_of(0.0, 7) == 0 and oracle.n_route_of(1.0, 7) == 7


def test_block_layout_hand_example():
    starts, cnts, nSB, nCB = oracle.block_layout(5, 3, 2)
    assert (nSB, nCB) == (3, 2)
    assert starts.tolist() == [0, 2, 4, 5, 7]
    assert cnts.tolist() == [2, 2, 1, 2, 1]
    starts, cnts, nSB, nCB = oracle.block_layout(20280, 20280, 128)
    assert nSB == nCB == 159 and cnts[158] == 56 and cnts[-1] == 56 and starts[159] == 20280


def test_block_means_hand_and_cumsum():
    x = np.arange(8, dtype=np.float64)[:, None] * np.array([[1.0, -2.0]])
    starts, cnts, _, _ = oracle.block_layout(5, 3, 2)
    m = oracle.block_means(x, starts, cnts)
    # hand-worked: rows {0,1},{2,3},{4},{5,6},{7}
    assert np.allclose(m[:, 0], [0.5, 2.5, 4.0, 5.5, 7.0])
    assert np.allclose(m[:, 1], [-1.0, -5.0, -8.0, -11.0, -14.0])
    y = rand((300, 5), 1)
    starts, cnts, _, _ = oracle.block_layout(170, 130, 64)
    cs = np.vstack([np.zeros((1, 5)), np.cumsum(y, axis=0)])
    ref = (cs[starts + cnts] - cs[starts]) / cnts[:, None]
    assert np.allclose(oracle.block_means(y, starts, cnts), ref, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------------- top-k
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_topk_matches_rank_counting(seed):
    rng = np.random.default_rng(seed)
    s = rng.integers(0, 6, size=40).astype(np.float64)  # many ties
    for k in range(0, 41):
        got = oracle.topk_ascending(s, k)
        rank = np.array([np.sum((s > s[i]) | ((s == s[i]) & (np.arange(40) < i))) for i in range(40)])
        assert got.tolist() == np.nonzero(rank < k)[0].tolist()


# ------------------------------------------------------------------- saliency
def test_saliency_sums_to_one_and_constant_keys():
    starts, cnts, nSB, nCB = oracle.block_layout(150, 90, 32)
    Q = rand((len(cnts), 16), 3)
    K = np.ones((len(cnts), 16)) * 0.7
    sal = oracle.block_saliency(Q, K, cnts, 240, 0.25)
    assert math.isclose(sal.sum(), 1.0, rel_tol=1e-12)
    # identical keys: every token equally likely -> block mass cnt_c / N
    assert np.allclose(sal, cnts / 240.0, rtol=1e-12)
    K2 = rand((len(cnts), 16), 4)
    assert math.isclose(oracle.block_saliency(Q, K2, cnts, 240, 0.25).sum(), 1.0, rel_tol=1e-12)


def test_saliency_block_constant_reduces_to_token_attention():
    N_src, N_ctx, blk, d = 150, 90, 32, 16
    starts, cnts, nSB, nCB = oracle.block_layout(N_src, N_ctx, blk)
    q = block_constant(rand((len(cnts), d), 5), cnts)
    k = block_constant(rand((len(cnts), d), 6), cnts)
    Qbar = oracle.block_means(q, starts, cnts)
    Kbar = oracle.block_means(k, starts, cnts)
    sal = oracle.block_saliency(Qbar, Kbar, cnts, N_src + N_ctx, 1 / math.sqrt(d))
    A = token_attention_matrix(q, k)                    # [N, N], library softmax
    colmean = A.mean(axis=0)
    ref = np.array([colmean[s:s + c].sum() for s, c in zip(starts, cnts)])
    assert np.allclose(sal, ref, rtol=1e-10, atol=1e-14)


def test_saliency_block_one_is_column_mean():
    q, k = rand((40, 8), 7), rand((40, 8), 8)
    starts, cnts, nSB, nCB = oracle.block_layout(25, 15, 1)
    sal = oracle.block_saliency(q, k, cnts, 40, 1 / math.sqrt(8))
    assert np.allclose(sal, token_attention_matrix(q, k).mean(axis=0), rtol=1e-10)


# ------------------------------------------------------------------ sharpness
def test_sharpness_zero_query_closed_form():
    cnt = np.array([64, 64, 17, 64, 3])
    sh = oracle.sharpness(np.zeros((3, 8)), rand((5, 8), 9), cnt, 0.3)
    assert np.allclose(sh, 64 / cnt.sum(), rtol=1e-13)


def test_sharpness_block_constant_is_block_mass():
    N_src, N_ctx, blk, d = 100, 70, 16, 8
    starts, cnts, nSB, nCB = oracle.block_layout(N_src, N_ctx, blk)
    k = block_constant(rand((len(cnts), d), 10), cnts)
    q = rand((N_src + N_ctx, d), 11) * 2.0
    Kbar = oracle.block_means(k, starts, cnts)
    kept_ctx = np.array([0, 2, 4])
    Kb = oracle.kept_blocks(nSB, kept_ctx)
    T = oracle.kept_tokens(starts, cnts, Kb)
    sh = oracle.sharpness(q, Kbar[Kb], cnts[Kb], 1 / math.sqrt(d))
    onehot = np.zeros((len(T), len(Kb)))
    pos = 0
    for j, b in enumerate(Kb):
        onehot[pos:pos + cnts[b], j] = 1.0
        pos += cnts[b]
    mass = sdpa(q, k[T], onehot)                     # attention mass per kept block
    assert np.allclose(sh, mass.max(axis=1), rtol=1e-10)


def test_sharpness_block_one_is_max_token_probability():
    q, k = rand((30, 8), 12) * 3, rand((30, 8), 13)
    starts, cnts, nSB, nCB = oracle.block_layout(18, 12, 1)
    sh = oracle.sharpness(q, k, cnts, 1 / math.sqrt(8))
    assert np.allclose(sh, token_attention_matrix(q, k).max(axis=1), rtol=1e-10)


# ------------------------------------------------------------- full / Taylor
def tiny_head(seed=0, h=0, cfg=None):
    cfg = cfg or CONFIGS["tiny"]
    q, k, v = (bf16_bits_to_f64(x) for x in head_inputs(cfg, 0, h, seed))
    return cfg, q, k, v


def test_keep1_rho1_equals_library_dense():
    cfg, q, k, v = tiny_head()
    r = oracle.isa_head(q, k, v, cfg.N_src, cfg.block, 1.0, 1.0)
    assert len(r["routed"]) == cfg.N and len(r["tokens"]) == cfg.N
    assert np.allclose(r["out"], sdpa(q, k, v), rtol=1e-10, atol=1e-12)
    assert np.allclose(oracle.dense_head(q, k, v), sdpa(q, k, v), rtol=1e-10, atol=1e-12)


def test_full_rows_keep_lt1_equals_masked_library():
    cfg, q, k, v = tiny_head()
    r = oracle.isa_head(q, k, v, cfg.N_src, cfg.block, 0.5, 1.0)
    mask = np.zeros((cfg.N, cfg.N), dtype=bool)
    mask[:, r["tokens"]] = True
    assert np.allclose(r["out"], sdpa(q, k, v, mask=mask), rtol=1e-10, atol=1e-12)


def test_taylor_block1_is_exact():
    cfg, q, k, v = tiny_head()
    r = oracle.isa_head(q, k, v, cfg.N_src, 1, 1.0, 0.0)
    assert len(r["taylor"]) == cfg.N
    assert np.allclose(r["out"], sdpa(q, k, v), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("N_src,N_ctx,blk,keep", [(256, 256, 64, 0.5), (200, 77, 64, 0.6), (150, 40, 128, 1.0)])
def test_taylor_equals_per_token_key_replacement(N_src, N_ctx, blk, keep):
    """0-th order Taylor: each kept key k_j is replaced by its block mean while
    the values stay per token; library attention over that must equal the
    oracle's block form (ln cnt bias + block-mean values)."""
    cfg = CONFIGS["tiny"].replace(N_src=N_src, N_ctx=N_ctx, block=blk)
    _, q, k, v = tiny_head(cfg=cfg)
    r = oracle.isa_head(q, k, v, N_src, blk, keep, 0.0)
    starts, cnts = oracle.block_layout(N_src, N_ctx, blk)[:2]
    k_rep = np.empty_like(k)
    for b, (s, c) in enumerate(zip(starts, cnts)):
        k_rep[s:s + c] = k[s:s + c].mean(axis=0)
    T = r["tokens"]
    assert np.allclose(r["out"], sdpa(q, k_rep[T], v[T]), rtol=1e-10, atol=1e-12)


def test_taylor_exact_for_constant_key_blocks():
    N_src, N_ctx, blk, d = 130, 60, 32, 16
    starts, cnts, nSB, nCB = oracle.block_layout(N_src, N_ctx, blk)
    k = block_constant(rand((len(cnts), d), 20), cnts)
    q, v = rand((N_src + N_ctx, d), 21), rand((N_src + N_ctx, d), 22)
    r = oracle.isa_head(q, k, v, N_src, blk, 0.5, 0.0)
    mask = np.zeros((len(q), len(q)), dtype=bool)
    mask[:, r["tokens"]] = True
    assert np.allclose(r["out"], sdpa(q, k, v, mask=mask), rtol=1e-10, atol=1e-12)


def test_zero_query_gives_mean_of_kept_values():
    cfg, q, k, v = tiny_head()
    q = np.zeros_like(q)
    r = oracle.isa_head(q, k, v, cfg.N_src, cfg.block, 0.5, 0.25)
    ref = v[r["tokens"]].mean(axis=0)
    assert np.allclose(r["out"], ref[None, :], rtol=1e-12, atol=1e-13)
    assert np.allclose(r["sharp"], r["cnts"][r["kept_blocks"]].max() / len(r["tokens"]))


def test_routing_partition_and_convexity():
    cfg, q, k, v = tiny_head()
    r = oracle.isa_head(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho)
    assert len(r["routed"]) == oracle.n_route_of(cfg.rho, cfg.N)
    assert sorted(np.concatenate([r["routed"], r["taylor"]]).tolist()) == list(range(cfg.N))
    thr = oracle.kth_value(r["sharp"], len(r["routed"]))
    assert r["sharp"][r["routed"]].min() >= thr >= r["sharp"][r["taylor"]].max()
    T = r["tokens"]
    lo, hi = v[T].min(axis=0), v[T].max(axis=0)
    assert np.all(r["out"][r["routed"]] >= lo - 1e-12) and np.all(r["out"][r["routed"]] <= hi + 1e-12)
    Vb = r["Vbar"][r["kept_blocks"]]
    o_t = r["out"][r["taylor"]]
    assert np.all(o_t >= Vb.min(axis=0) - 1e-12) and np.all(o_t <= Vb.max(axis=0) + 1e-12)


# ------------------------------------------------------- the pages' insights
@pytest.mark.parametrize("name,heads", [("tiny", [0, 1]), ("small", [0, 5])])
def test_sharpness_correlates_with_taylor_error(name, heads):
    """Second insight of the ISA abstract: sharper queries suffer a larger
    0-th order Taylor error.  Spearman rank correlation must be positive."""
    cfg = CONFIGS[name]
    for h in heads:
        _, q, k, v = tiny_head(h=h, cfg=cfg)
        r = oracle.isa_head(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho)
        Kb = r["kept_blocks"]
        o_full = oracle.full_rows(q, k[r["tokens"]], v[r["tokens"]], r["scale"])
        o_tay = oracle.taylor_rows(q, r["Kbar"][Kb], r["Vbar"][Kb], r["cnts"][Kb], r["scale"])
        err = np.linalg.norm(o_full - o_tay, axis=1)
        rho_s = spearmanr(r["sharp"], err).statistic
        assert rho_s > 0.2, (name, h, rho_s)


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_context_less_salient_than_source(name):
    """First insight of the ISA abstract (planted here by scaling context keys)."""
    cfg = CONFIGS[name]
    _, q, k, v = tiny_head(cfg=cfg)
    r = oracle.isa_head(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho)
    nSB = r["nSB"]
    assert r["sal_all"][nSB:].mean() < r["sal_all"][:nSB].mean()


# ------------------------------------------------------------ k-th value
def test_kth_value_hand_worked():
    """kth_value sets the tie window of every set comparison, so it is pinned
    by exact values: descending order 0.9, 0.9, 0.5, 0.3, 0.1."""
    s = np.array([0.3, 0.9, 0.1, 0.9, 0.5])
    assert oracle.kth_value(s, 0) == math.inf
    assert oracle.kth_value(s, 1) == 0.9
    assert oracle.kth_value(s, 2) == 0.9          # a tie with the first
    assert oracle.kth_value(s, 3) == 0.5          # the (k+1)-th value would be 0.3
    assert oracle.kth_value(s, 4) == 0.3
    assert oracle.kth_value(s, 5) == 0.1          # k = len: the smallest score
    assert oracle.kth_value(np.array([2.0]), 1) == 2.0


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_kth_value_is_the_order_statistic(seed):
    """Brute-force definition of the k-th largest value t: fewer than k scores
    lie strictly above t and at least k lie at or above it, and t is one of
    the scores; it is also the smallest score of the top-k set."""
    rng = np.random.default_rng(seed)
    s = rng.integers(0, 7, size=23).astype(np.float64) / 7.0  # many ties
    for k in range(1, 24):
        t = oracle.kth_value(s, k)
        assert t in s
        assert np.sum(s > t) < k <= np.sum(s >= t)
        assert t == s[oracle.topk_ascending(s, k)].min()


# ------------------------------------------------------------ count guard
def test_count_guard_hand_worked():
    """Counts are ceil(frac*n - g) with g = min(1e-6*n, 0.5) (a reading: keep
    and rho reach the kernels as float32, whose rounding moves frac*n by up to
    6e-8*n).  Hand-worked cases on both sides of the guard:
      rho = 0.2 as float32 (0.20000000298...), N = 40560: 8112.00012 -> 8112
        (a plain ceiling would give 8113);
      rho = 0.2000101, N = 40560: 8112.41, guard 0.0406 -> 8113;
      rho = 0.2000005, N = 10^6: 200000.5, guard 0.5 (capped) -> 200000;
      rho = 0.200002, N = 10^6: 200002 exactly -> 200002 (an uncapped guard of
        1.0 would give 200001);
      rho = 1, N = 2*10^7: all rows;
      keep = 0.3f, nCB = 32: 9.6000001 -> 10;  keep = 0.25f, nCB = 159: 39.75 -> 40."""
    assert oracle.n_route_of(float(np.float32(0.2)), 40560) == 8112
    assert oracle.n_route_of(0.2000101, 40560) == 8113
    assert oracle.n_route_of(0.2000005, 1_000_000) == 200000
    assert oracle.n_route_of(0.200002, 1_000_000) == 200002
    assert oracle.n_route_of(1.0, 20_000_000) == 20_000_000
    assert oracle.n_keep_of(float(np.float32(0.3)), 32) == 10
    assert oracle.n_keep_of(float(np.float32(0.25)), 159) == 40
    assert oracle.guarded_count(0.5, 7) == 4 and oracle.guarded_count(0.0, 7) == 0


# ------------------------------------------------------- batched entry points
def test_dense_equals_library_over_batch_and_heads():
    """oracle.dense over [B, H, N, d] against torch SDPA (float64), with
    distinct heads so that a swapped or dropped (b, h) index fails."""
    rng = np.random.default_rng(30)
    q, k, v = (rng.standard_normal((2, 3, 70, 16)) for _ in range(3))
    q[1, 2] *= 3.0
    ref = torch.nn.functional.scaled_dot_product_attention(*(torch.from_numpy(x) for x in (q, k, v))).numpy()
    assert np.allclose(oracle.dense(q, k, v), ref, rtol=1e-10, atol=1e-12)
    ref2 = torch.nn.functional.scaled_dot_product_attention(*(torch.from_numpy(x) for x in (q, k, v)),
                                                            scale=0.3).numpy()
    assert np.allclose(oracle.dense(q, k, v, scale=0.3), ref2, rtol=1e-10, atol=1e-12)


def test_isa_fwd_keep1_rho1_equals_library_dense_over_batch():
    """keep = rho = 1: the batched forward is dense attention for every (b, h)."""
    rng = np.random.default_rng(31)
    q, k, v = (rng.standard_normal((2, 2, 150, 16)) for _ in range(3))
    ref = torch.nn.functional.scaled_dot_product_attention(*(torch.from_numpy(x) for x in (q, k, v))).numpy()
    assert np.allclose(oracle.isa_fwd(q, k, v, 90, 32, 1.0, 1.0), ref, rtol=1e-10, atol=1e-12)


def test_isa_fwd_rho0_equals_library_on_replaced_keys_per_head():
    """rho = 0, keep < 1: every row of every (b, h) is Taylor attention, which
    is library attention over the kept tokens with each key replaced by its
    block mean (values per token).  The kept set is taken per head from
    isa_head, the output from isa_fwd, the reference from SDPA."""
    rng = np.random.default_rng(32)
    B, H, N_src, N_ctx, blk, d = 2, 2, 100, 90, 32, 8
    q, k, v = (rng.standard_normal((B, H, N_src + N_ctx, d)) for _ in range(3))
    k[:, :, N_src:] *= 0.5
    out = oracle.isa_fwd(q, k, v, N_src, blk, 0.5, 0.0)
    starts, cnts = oracle.block_layout(N_src, N_ctx, blk)[:2]
    for b in range(B):
        for h in range(H):
            r = oracle.isa_head(q[b, h], k[b, h], v[b, h], N_src, blk, 0.5, 0.0)
            k_rep = np.empty_like(k[b, h])
            for s, c in zip(starts, cnts):
                k_rep[s:s + c] = k[b, h, s:s + c].mean(axis=0)
            T = r["tokens"]
            assert np.allclose(out[b, h], sdpa(q[b, h], k_rep[T], v[b, h, T]), rtol=1e-10, atol=1e-12)
