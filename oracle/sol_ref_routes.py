"""Top-k and top-p block routing over the Sol-Attn proxy row.  TEST INFRASTRUCTURE ONLY.

Only tests/, the package smoke check and the benchmark's CPU-baseline leg may import this module.

Source: "Sol-Attn: Accelerating Video Generation Inference via On-the-Fly Attention
Sparsification" (Li et al., 2026), the paragraph on the two limits of existing routing: top-k gives
every query the same fixed number k of key blocks, and top-p keeps adding blocks until their
cumulative probability reaches a threshold.  The fused kernel can route by either of these instead
of the mu + beta*sigma threshold, over the same proxy row S_j = (q_bar . k_bar_j) / sqrt(d) (the
proxy comes from ``sol_ref.route``; everything after it is defined here).

Readings fixed here (the page names the two rules but not their details):
  - order: blocks are ranked by proxy score, highest first; equal scores (as values, so -0.0 equals
    +0.0) rank the lower block index first;
  - top-k keeps the first min(k, Nk) blocks of that order (k = 0 keeps none);
  - top-p: the probability of block j is softmax over the row, w_j / Z with w_j = exp(S_j - max S)
    and Z = sum_j w_j, all in float64 (no weighting by the block's token count); the kept set is
    the shortest prefix of the order whose mass reaches p*Z, so block j is kept iff the mass of the
    blocks ranked before it is < p*Z.  p <= 0 keeps none, p >= 1 keeps every block;
  - the "threshold" statistic reported with a variant is the score of the last kept block
    (+inf when none is kept); mu and sigma are the row's, as for the threshold rule.
"""
from __future__ import annotations

import numpy as np


def order_desc(row: np.ndarray) -> np.ndarray:
    """Block indices of one proxy row, highest score first, ties by ascending index."""
    return np.argsort(-np.asarray(row, np.float64), kind="stable")


def select_topk(proxy: np.ndarray, k: int) -> np.ndarray:
    """Keep mask [U, Nk] (uint8) of the k highest-scoring blocks of every row."""
    proxy = np.atleast_2d(np.asarray(proxy, np.float32))
    U, Nk = proxy.shape
    mask = np.zeros((U, Nk), np.uint8)
    kk = max(0, min(int(k), Nk))
    for u in range(U):
        mask[u, order_desc(proxy[u])[:kk]] = 1
    return mask


def row_masses(row: np.ndarray):
    """float64 w_j = exp(S_j - max S) of one row and their sum Z."""
    s = np.asarray(row, np.float64)
    w = np.exp(s - s.max())
    return w, float(w.sum())


def select_topp(proxy: np.ndarray, p: float, with_boundary: bool = False):
    """Keep mask [U, Nk] (uint8) of the shortest highest-first prefix whose softmax mass reaches p.

    With ``with_boundary`` also returns, per row, (mass before the last kept block, mass including
    it) divided by Z, so that a caller can see how close the decision was to p (the float64 sum of
    the masses depends on the summation order at the 1e-16 relative level)."""
    proxy = np.atleast_2d(np.asarray(proxy, np.float32))
    U, Nk = proxy.shape
    mask = np.zeros((U, Nk), np.uint8)
    bound = np.full((U, 2), np.nan)
    for u in range(U):
        if p >= 1.0:
            mask[u] = 1
            continue
        if not p > 0.0:
            continue
        order = order_desc(proxy[u])
        w, Z = row_masses(proxy[u])
        cum = np.cumsum(w[order])
        target = float(p) * Z
        t = int(np.argmax(cum >= target)) if cum[-1] >= target else Nk - 1
        mask[u, order[:t + 1]] = 1
        bound[u] = ((cum[t - 1] if t > 0 else 0.0) / Z, cum[t] / Z)
    return (mask, bound) if with_boundary else mask


def last_kept_score(proxy: np.ndarray, mask: np.ndarray) -> np.ndarray:
    """Score of the last kept block of every row (the lowest kept score), +inf if none kept."""
    proxy = np.atleast_2d(np.asarray(proxy, np.float32))
    out = np.full(proxy.shape[0], np.inf)
    for u in range(proxy.shape[0]):
        kept = proxy[u][mask[u].astype(bool)]
        if kept.size:
            out[u] = float(kept.min())
    return out


def route_variant(q, kbar, rule: str, param: float, units=None):
    """Routing by top-k (``rule='topk'``, param = k) or top-p (``rule='topp'``, param = p) for the
    query tiles ``units``.  Same dict as ``sol_ref.route`` (tau = last kept score)."""
    from oracle import sol_ref
    r = sol_ref.route(q, kbar, 0.0, units)        # proxy, mu and sigma do not depend on beta
    if rule == "topk":
        m = select_topk(r["proxy"], int(param))
    elif rule == "topp":
        m = select_topp(r["proxy"], float(param))
    else:
        raise ValueError(rule)
    r["mask"] = m
    r["count"] = m.sum(1).astype(np.int32)
    r["tau"] = last_kept_score(r["proxy"], m)
    return r
