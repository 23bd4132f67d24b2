"""Pins for the oracle's top-k / top-p routing (runs without a GPU).

Each selection rule is checked against a second, independently written definition (an O(Nk^2)
rank count instead of a sort), closed forms from the two-block example, limits, and the link
between top-k and the mu + beta*sigma threshold.
"""
import math

import numpy as np
import pytest

from free_sparse_attention_block_b200 import inputs
from oracle import sol_ref
from oracle import sol_ref_routes as rr


def ranks_bruteforce(row):
    """rank_j = number of blocks that come before j: a higher score, or an equal score and a
    lower index."""
    s = np.asarray(row, np.float64)
    n = s.size
    rk = np.zeros(n, np.int64)
    for j in range(n):
        for i in range(n):
            if s[i] > s[j] or (s[i] == s[j] and i < j):
                rk[j] += 1
    return rk


def rows_with_ties(seed, U=6, Nk=9):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((U, Nk)).astype(np.float32)
    x[:, 3] = x[:, 5]                  # an exact tie in every row
    x[0, :] = 0.25                     # an all-equal row
    x[1, 2], x[1, 7] = -0.0, 0.0       # signed zeros compare equal
    return x


@pytest.mark.parametrize("k", [0, 1, 3, 5, 9, 20])
def test_topk_equals_rank_definition(k):
    x = rows_with_ties(1)
    m = rr.select_topk(x, k)
    for u in range(x.shape[0]):
        want = (ranks_bruteforce(x[u]) < k).astype(np.uint8)
        assert np.array_equal(m[u], want)
    assert np.all(m.sum(1) == min(k, x.shape[1]))


@pytest.mark.parametrize("p", [0.0, 1e-9, 0.2, 0.5, 0.77, 0.95, 1.0, 1.5, -0.3])
def test_topp_equals_rank_definition(p):
    x = rows_with_ties(2)
    m = rr.select_topp(x, p)
    for u in range(x.shape[0]):
        rk = ranks_bruteforce(x[u])
        s = x[u].astype(np.float64)
        w = np.array([math.exp(v - s.max()) for v in s])
        Z = math.fsum(w)
        for j in range(s.size):
            before = math.fsum(w[i] for i in range(s.size) if rk[i] < rk[j])
            if p >= 1.0:
                keep = True
            elif p <= 0.0:
                keep = False
            else:
                keep = before < p * Z
            assert m[u, j] == keep, (u, j, p)


def test_topp_two_block_closed_form():
    """Two blocks with proxy (sqrt 2, 0) (the hand-worked example's routing row): the top block
    holds e^sqrt2 / (e^sqrt2 + 1) = 0.8044297 of the mass."""
    x = np.array([[math.sqrt(2.0), 0.0]], np.float32)
    p1 = math.exp(math.sqrt(2.0)) / (math.exp(math.sqrt(2.0)) + 1.0)
    assert abs(p1 - 0.8044297) < 1e-7
    assert rr.select_topp(x, 0.80).tolist() == [[1, 0]]
    assert rr.select_topp(x, 0.81).tolist() == [[1, 1]]
    assert rr.select_topk(x, 1).tolist() == [[1, 0]]
    # reversed order of the blocks: the selection follows the score, not the index
    assert rr.select_topp(x[:, ::-1], 0.80).tolist() == [[0, 1]]


def test_topp_nested_and_monotone_in_p():
    x = rows_with_ties(3, U=4, Nk=30)
    prev = np.zeros_like(x, dtype=np.uint8)
    for p in np.linspace(0.0, 1.0, 41):
        m = rr.select_topp(x, float(p))
        assert np.all(m >= prev)
        prev = m
    assert np.all(prev == 1)


def test_topk_nested_in_k():
    x = rows_with_ties(4, U=4, Nk=30)
    prev = np.zeros_like(x, dtype=np.uint8)
    for k in range(31):
        m = rr.select_topk(x, k)
        assert np.all(m >= prev) and np.all(m.sum(1) == k)
        prev = m


def test_topk_with_threshold_count_equals_threshold_mask():
    """The threshold rule keeps an upper set of the row, so top-k with k = its count keeps the
    same blocks (rows without ties at the threshold)."""
    q, k, _ = inputs.small_workload(64 * 30 + 7, BH=2, seed=12)
    kbar = sol_ref.pool(k)
    for beta in (0.0, 0.5, 1.3):
        r = sol_ref.route(q, kbar, beta)
        for u in range(r["proxy"].shape[0]):
            c = int(r["count"][u])
            assert np.array_equal(rr.select_topk(r["proxy"][u:u + 1], c)[0], r["mask"][u])


def test_route_variant_limits_match_threshold_limits():
    q, k, _ = inputs.small_workload(64 * 11 + 3, BH=2, seed=13)
    kbar = sol_ref.pool(k)
    Nk = 12
    dense = sol_ref.route(q, kbar, float("-inf"))
    none = sol_ref.route(q, kbar, float("inf"))
    for rule, param, ref in [("topk", Nk, dense), ("topk", 10 ** 6, dense), ("topp", 1.0, dense),
                             ("topk", 0, none), ("topp", 0.0, none)]:
        r = rr.route_variant(q, kbar, rule, param)
        assert np.array_equal(r["mask"], ref["mask"]), (rule, param)
        np.testing.assert_array_equal(r["mu"], dense["mu"])
        np.testing.assert_array_equal(r["sigma"], dense["sigma"])
    r = rr.route_variant(q, kbar, "topk", 1)
    np.testing.assert_array_equal(r["tau"], r["proxy"].max(1))
    assert np.all(np.isinf(rr.route_variant(q, kbar, "topk", 0)["tau"]))


def test_topp_boundary_report():
    x = rows_with_ties(5, U=5, Nk=16)
    m, b = rr.select_topp(x, 0.6, with_boundary=True)
    for u in range(x.shape[0]):
        assert b[u, 0] < 0.6 <= b[u, 1] + 1e-15


def test_topp_exact_mass_tie_keeps_the_shortest_prefix():
    """Four equal scores: each block holds 1/4 of the mass, so p = 1/2 is reached exactly after
    two blocks (the lowest indices); a strict ">" would take a third."""
    x = np.zeros((1, 4), np.float32)
    assert rr.select_topp(x, 0.5).tolist() == [[1, 1, 0, 0]]
    assert rr.select_topp(x, 0.25).tolist() == [[1, 0, 0, 0]]
    assert rr.select_topk(x, 3).tolist() == [[1, 1, 1, 0]]
