"""Float64 CPU oracle of the In-context Sparse Attention (ISA) forward.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The product path
(the CUDA library and its Python binding) never calls it, and it shares no
code with that path: it is plain numpy in float64, written from the method's
definitions, one step after another, with no blocking or fusion.

Source of the method: "Lightning Unified Video Editing via In-Context Sparse
Attention" (Shao et al., 2026), abstract (chatpaper.ai page).  The abstract
only outlines ISA: context tokens are less salient than source tokens, so a
pre-selection step drops redundant context; query sharpness tracks the error
of the approximation, so a dynamic grouping step sends high-error (sharp)
queries to full attention and the rest to 0-th order Taylor sparse attention.
The exact formulas below are the plainest reading of that outline:

* scale s = 1/sqrt(d) (the usual scaled-dot-product convention, as in the
  attention-cost notes on the intelliparadigm.com page, TemporalAttention
  listing);
* blocks of ``blk`` consecutive tokens, taken separately in the source and
  the context segment; the last block of a segment may be partial;
  ``cnt_b`` tokens in block b; block means  x_bar_b = mean_{j in b} x_j;
* every token is a query; only context keys are pruned;
* saliency of key block c: mean over query blocks r (weighted by cnt_r) of
  the block-level attention softmax_c( s * Qbar_r . Kbar_c + ln cnt_c ),
  over all key blocks; context blocks are ranked by it and the top
  n_keep = ceil(keep*nCB - g(nCB)) are kept, all source blocks always kept,
  with the guard g(n) = min(1e-6*n, 0.5) (see ``guarded_count``);
* sharpness of query i: the largest probability of the block-level
  distribution softmax_b( s * q_i . Kbar_b + ln cnt_b ) over kept blocks;
* routing: the n_route = ceil(rho*N - g(N)) sharpest queries get full
  attention over every kept token; ties rank the lower index first;
* 0-th order Taylor attention: exp(s q.k_j) is replaced by exp(s q.Kbar_b)
  for every j in block b, in numerator and denominator; summing over the
  block turns this into attention over block means with an additive ln cnt_b
  bias and block-mean values;
* variant stage 4 of first order (``taylor_order=1``): the linear term of
  exp around the block mean is kept, which adds s * C_b^T q per kept block
  to the numerator, C_b = sum_{j in b} (k_j - Kbar_b) v_j^T;
* variant grouping by whole query blocks (``granularity="block"``): a query
  block (same per-segment partition as the keys) scores the mean sharpness
  of its queries, and the n_route_blocks = ceil(rho*nB - g(nB)) best
  blocks (ties: lower block index) are routed whole.

Pins (see tests/test_oracle_pins.py): the saliency and sharpness formulas are
readings, not printed by the pages ("parity unpinned" as to the pages); they
are pinned by closed forms and by reduction to token-level attention computed
with torch's scaled_dot_product_attention, which the pins use as an
independent library routine.  The block-granular grouping (mean sharpness
per query block) is a reading too ("parity unpinned" as to the pages),
pinned by hand-worked means, rank counting, its reduction to per-token
grouping at block = 1 and library attention
(tests/test_oracle_block_route_pins.py).  The first-order Taylor variant
follows from the expansion of exp around the block mean with no further
reading; it is pinned by a per-token double loop, exact special cases and
its second-order error scaling (tests/test_oracle_taylor1_pins.py).
"""
from __future__ import annotations

import math

import numpy as np

NEG_INF = -np.inf


# ---------------------------------------------------------------------------
# Counts and block layout
# ---------------------------------------------------------------------------

def guarded_count(frac: float, n: int) -> int:
    """ceil(frac*n - g) clamped to [0, n], with the guard g = min(1e-6*n, 0.5).

    The fractions keep and rho reach the kernels as float32, whose rounding
    moves frac*n by up to 6e-8*n (0.2f*40560 = 8112.0001 must count 8112).
    The guard 1e-6*n absorbs that; it is capped at one half so that an exact
    integral product never loses a unit (at n >= 10^6 the uncapped guard
    would count 200001 for 0.200002 * 10^6).  A genuinely fractional product
    whose fraction is within the guard rounds down.
    """
    return int(min(max(math.ceil(frac * n - min(1e-6 * n, 0.5)), 0), n))


def n_keep_of(keep: float, nCB: int) -> int:
    """Number of context blocks kept: ceil(keep*nCB - g(nCB)) in [0, nCB]."""
    return guarded_count(keep, nCB)


def n_route_of(rho: float, N: int) -> int:
    """Number of queries routed to full attention: ceil(rho*N - g(N)) in [0, N]."""
    return guarded_count(rho, N)


def block_layout(N_src: int, N_ctx: int, blk: int):
    """Per-segment blocks: (start, count) of source blocks then context blocks.

    Blocks never straddle the source/context boundary; the last block of each
    segment holds the remainder.  Returns (starts, cnts, nSB, nCB).
    """
    nSB = -(-N_src // blk)
    nCB = -(-N_ctx // blk)
    starts, cnts = [], []
    for b in range(nSB):
        starts.append(b * blk)
        cnts.append(min(blk, N_src - b * blk))
    for c in range(nCB):
        starts.append(N_src + c * blk)
        cnts.append(min(blk, N_ctx - c * blk))
    return np.array(starts, dtype=np.int64), np.array(cnts, dtype=np.int64), nSB, nCB


def block_means(x: np.ndarray, starts: np.ndarray, cnts: np.ndarray) -> np.ndarray:
    """Block means x_bar_b = (1/cnt_b) * sum_{j in b} x_j, float64 [nB, d]."""
    out = np.empty((len(starts), x.shape[1]), dtype=np.float64)
    for b, (s, c) in enumerate(zip(starts, cnts)):
        out[b] = x[s:s + c].sum(axis=0) / c
    return out


# ---------------------------------------------------------------------------
# Ranking
# ---------------------------------------------------------------------------

def topk_ascending(scores: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest scores, higher score first, lower index on ties;
    returned sorted ascending (int64)."""
    if k <= 0:
        return np.zeros(0, dtype=np.int64)
    idx = np.arange(len(scores))
    order = np.lexsort((idx, -scores))  # last key is primary: -score, then index
    return np.sort(order[:k]).astype(np.int64)


def kth_value(scores: np.ndarray, k: int) -> float:
    """The k-th largest score (1-based); +inf when k == 0."""
    if k <= 0:
        return math.inf
    return float(np.sort(scores)[::-1][k - 1])


# ---------------------------------------------------------------------------
# Stage 1: context pre-selection (ISA abstract, first insight: context tokens
# carry less saliency than source tokens, so context is pruned up front)
# ---------------------------------------------------------------------------

def block_saliency(Qbar, Kbar, cnts, N, scale):
    """Saliency of every key block (source and context), float64 [nB].

    Block-level logits  l_rc = s * Qbar_r . Kbar_c + ln cnt_c;  row softmax
    over all key blocks c;  saliency_c = sum_r cnt_r * P_rc / N.
    The result sums to 1 over all key blocks.
    """
    logits = scale * (Qbar @ Kbar.T) + np.log(cnts.astype(np.float64))[None, :]
    logits = logits - logits.max(axis=1, keepdims=True)
    P = np.exp(logits)
    P = P / P.sum(axis=1, keepdims=True)
    return (cnts.astype(np.float64)[:, None] * P).sum(axis=0) / N


def kept_blocks(nSB: int, kept_ctx: np.ndarray) -> np.ndarray:
    """Indices (into the source+context block list) of the kept set:
    every source block, then the kept context blocks, ascending."""
    return np.concatenate([np.arange(nSB, dtype=np.int64), nSB + np.asarray(kept_ctx, dtype=np.int64)])


def kept_tokens(starts, cnts, blocks) -> np.ndarray:
    """Token indices of the given blocks, ascending."""
    if len(blocks) == 0:
        return np.zeros(0, dtype=np.int64)
    return np.concatenate([np.arange(starts[b], starts[b] + cnts[b]) for b in blocks]).astype(np.int64)


# ---------------------------------------------------------------------------
# Stage 2: query sharpness (ISA abstract, second insight: sharpness of a
# query goes with the error of the approximation)
# ---------------------------------------------------------------------------

def sharpness(q, Kbar_K, cnt_K, scale):
    """Largest probability of softmax_b( s*q_i.Kbar_b + ln cnt_b ) over kept
    blocks b, for every query row i; float64 [n_q] in (0, 1]."""
    logits = scale * (q @ Kbar_K.T) + np.log(cnt_K.astype(np.float64))[None, :]
    m = logits.max(axis=1, keepdims=True)
    return 1.0 / np.exp(logits - m).sum(axis=1)


# ---------------------------------------------------------------------------
# Variant of the grouping step: whole query blocks.  The abstract names a
# dynamic grouping of queries but not the unit that is grouped; this variant
# groups at the granularity of the token blocks already used for the keys,
# so that a routed group is a run of consecutive query rows.
# ---------------------------------------------------------------------------

def n_route_blocks_of(rho: float, nB: int) -> int:
    """Number of query blocks routed to full attention: ceil(rho*nB - g(nB)) in [0, nB]."""
    return guarded_count(rho, nB)


def block_mean_sharpness(sharp, starts, cnts):
    """Score of every query block: the mean sharpness of its cnt_b queries."""
    return np.array([sharp[s:s + c].sum() / c for s, c in zip(starts, cnts)], dtype=np.float64)


def route_query_blocks(sharp, starts, cnts, rho):
    """Block-granular grouping: the n_route_blocks query blocks of highest
    mean sharpness (ties: lower block index first) are routed whole.
    Returns (block scores, n_route_blocks, routed block indices ascending)."""
    score = block_mean_sharpness(sharp, starts, cnts)
    nrb = n_route_blocks_of(rho, len(starts))
    return score, nrb, topk_ascending(score, nrb)


# ---------------------------------------------------------------------------
# Stage 3: full attention for routed queries
# ---------------------------------------------------------------------------

def full_rows(q_rows, k_T, v_T, scale, chunk=512):
    """Exact softmax attention of each query row over the token set T."""
    out = np.empty((q_rows.shape[0], v_T.shape[1]), dtype=np.float64)
    for a in range(0, q_rows.shape[0], chunk):
        s = scale * (q_rows[a:a + chunk] @ k_T.T)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        out[a:a + chunk] = (p @ v_T) / p.sum(axis=1, keepdims=True)
    return out


# ---------------------------------------------------------------------------
# Stage 4: 0-th order Taylor sparse attention for the remaining queries
# ---------------------------------------------------------------------------

def taylor_rows(q_rows, Kbar_K, Vbar_K, cnt_K, scale, chunk=4096):
    """o_i = sum_b cnt_b e^{s q_i.Kbar_b} Vbar_b / sum_b cnt_b e^{s q_i.Kbar_b}."""
    out = np.empty((q_rows.shape[0], Vbar_K.shape[1]), dtype=np.float64)
    lc = np.log(cnt_K.astype(np.float64))[None, :]
    for a in range(0, q_rows.shape[0], chunk):
        s = scale * (q_rows[a:a + chunk] @ Kbar_K.T) + lc
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        out[a:a + chunk] = (p @ Vbar_K) / p.sum(axis=1, keepdims=True)
    return out


# ---------------------------------------------------------------------------
# Variant of stage 4: first-order Taylor sparse attention.  The abstract's
# "0-th order" names the first member of a family; the next member keeps
# the linear term of exp around the block mean:
#   e^{s q.k_j} ~= e^{s q.Kbar_b} (1 + s q.(k_j - Kbar_b))   for j in b.
# In the denominator the linear terms of a block sum to zero (the deviations
# from the block mean sum to zero), so it stays sum_b cnt_b e^{s q.Kbar_b};
# the numerator gains s * C_b^T q per block, C_b = sum_{j in b} (k_j -
# Kbar_b) v_j^T (a d x d matrix).
# ---------------------------------------------------------------------------

def correction_matrices(k, v, starts, cnts, blocks):
    """C_b = sum_{j in b} (k_j - Kbar_b) v_j^T for the given blocks, float64 [n, d, d]."""
    d = k.shape[1]
    out = np.empty((len(blocks), d, d), dtype=np.float64)
    for r, b in enumerate(blocks):
        kb = k[starts[b]:starts[b] + cnts[b]]
        vb = v[starts[b]:starts[b] + cnts[b]]
        out[r] = (kb - kb.mean(axis=0)).T @ vb
    return out


def taylor1_rows(q_rows, Kbar_K, Vbar_K, C_K, cnt_K, scale, chunk=1024):
    """o_i = [sum_b cnt_b e^{l_ib} Vbar_b + s sum_b e^{l_ib} C_b^T q_i] / sum_b cnt_b e^{l_ib},
    l_ib = s q_i.Kbar_b (shifted by the row max; the shift cancels)."""
    out = np.empty((q_rows.shape[0], Vbar_K.shape[1]), dtype=np.float64)
    cnt = cnt_K.astype(np.float64)
    for a in range(0, q_rows.shape[0], chunk):
        qc = q_rows[a:a + chunk]
        l = scale * (qc @ Kbar_K.T)
        e = np.exp(l - l.max(axis=1, keepdims=True))
        num = (e * cnt[None, :]) @ Vbar_K
        for b in range(len(cnt)):  # s * e_ib * (C_b^T q_i), one kept block at a time
            num += (scale * e[:, b:b + 1]) * (qc @ C_K[b])
        out[a:a + chunk] = num / (e * cnt[None, :]).sum(axis=1, keepdims=True)
    return out


# ---------------------------------------------------------------------------
# The whole forward for one (b, h)
# ---------------------------------------------------------------------------

def isa_head(q, k, v, N_src, blk, keep, rho, scale=None,
             kept_override=None, routed_override=None, rows=None, granularity="token",
             taylor_order=0):
    """ISA forward for one head, all stages in order; float64 inputs [N, d].

    ``kept_override`` / ``routed_override`` replace the selected context
    block set / routed query set (used to re-run the later stages on a set
    that differs from the oracle's only inside the tie window); with
    ``granularity="block"`` the routed override is a set of query blocks.
    ``rows`` restricts which output rows are computed (others are NaN);
    every stage that decides a set still runs on all rows.
    ``granularity`` selects the dynamic query grouping: "token" routes the
    n_route sharpest queries one by one; "block" routes whole query blocks
    (see ``route_query_blocks``).
    ``taylor_order`` 0 (the method) or 1 (``taylor1_rows``) for the rows
    that are not routed.
    Returns a dict of every intermediate and the output.
    """
    N, d = q.shape
    N_ctx = N - N_src
    s = 1.0 / math.sqrt(d) if scale is None else scale
    starts, cnts, nSB, nCB = block_layout(N_src, N_ctx, blk)

    Qbar = block_means(q, starts, cnts)
    Kbar = block_means(k, starts, cnts)
    Vbar = block_means(v, starts, cnts)

    sal_all = block_saliency(Qbar, Kbar, cnts, N, s)
    sal_ctx = sal_all[nSB:]
    nk = n_keep_of(keep, nCB)
    kept_ctx = topk_ascending(sal_ctx, nk) if kept_override is None else np.asarray(kept_override, dtype=np.int64)

    Kb = kept_blocks(nSB, kept_ctx)
    sharp = sharpness(q, Kbar[Kb], cnts[Kb], s)
    extra = {}
    if granularity == "token":
        nr = n_route_of(rho, N)
        routed = topk_ascending(sharp, nr) if routed_override is None else np.asarray(routed_override, dtype=np.int64)
    elif granularity == "block":
        score, nrb, rblocks = route_query_blocks(sharp, starts, cnts, rho)
        if routed_override is not None:
            rblocks = np.asarray(routed_override, dtype=np.int64)
        routed = kept_tokens(starts, cnts, rblocks)
        nr = len(routed)
        extra = dict(block_score=score, n_route_blocks=nrb, routed_blocks=rblocks)
    else:
        raise ValueError(granularity)
    mask = np.ones(N, dtype=bool)
    mask[routed] = False
    taylor = np.nonzero(mask)[0].astype(np.int64)

    T = kept_tokens(starts, cnts, Kb)
    out = np.full((N, d), np.nan, dtype=np.float64)
    want = np.ones(N, dtype=bool) if rows is None else np.isin(np.arange(N), rows)
    r_sel = routed[want[routed]]
    t_sel = taylor[want[taylor]]
    if len(r_sel):
        out[r_sel] = full_rows(q[r_sel], k[T], v[T], s)
    if len(t_sel):
        if taylor_order == 0:
            out[t_sel] = taylor_rows(q[t_sel], Kbar[Kb], Vbar[Kb], cnts[Kb], s)
        elif taylor_order == 1:
            C = correction_matrices(k, v, starts, cnts, Kb)
            extra["C"] = C
            out[t_sel] = taylor1_rows(q[t_sel], Kbar[Kb], Vbar[Kb], C, cnts[Kb], s)
        else:
            raise ValueError(taylor_order)
    return dict(out=out, Qbar=Qbar, Kbar=Kbar, Vbar=Vbar, cnts=cnts, nSB=nSB, nCB=nCB,
                sal_all=sal_all, sal_ctx=sal_ctx, kept_ctx=kept_ctx, kept_blocks=Kb,
                sharp=sharp, routed=routed, taylor=taylor, tokens=T,
                n_keep=nk, n_route=nr, scale=s, **extra)


def isa_fwd(q, k, v, N_src, blk, keep, rho, scale=None):
    """ISA forward over [B, H, N, d] float64 inputs; returns out [B, H, N, d]."""
    B, H = q.shape[:2]
    out = np.empty(q.shape, dtype=np.float64)
    for b in range(B):
        for h in range(H):
            out[b, h] = isa_head(q[b, h], k[b, h], v[b, h], N_src, blk, keep, rho, scale)["out"]
    return out


def dense_head(q, k, v, scale=None, rows=None):
    """Plain softmax(s q k^T) v over all N keys for one head (rows optional)."""
    s = 1.0 / math.sqrt(q.shape[1]) if scale is None else scale
    qq = q if rows is None else q[rows]
    return full_rows(qq, k, v, s)


def dense(q, k, v, scale=None):
    """Dense attention over [B, H, N, d] float64 inputs."""
    B, H = q.shape[:2]
    out = np.empty(q.shape, dtype=np.float64)
    for b in range(B):
        for h in range(H):
            out[b, h] = dense_head(q[b, h], k[b, h], v[b, h], scale)
    return out
