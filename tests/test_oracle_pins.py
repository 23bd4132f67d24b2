"""Pins for the CPU oracle (runs without a GPU).

Each test ties the oracle to something other than itself: a library routine (torch's
scaled_dot_product_attention, numpy mean/std), a closed form worked by hand, an exact algebraic
identity of the correction term, or an invariance of the definition.  Together they are chosen so
that a plausible mistake in the oracle (a dropped ln n_j, a missing denominator term, the sign of
beta*sigma, sample instead of population sigma, a wrong pooling divisor on the ragged block, a
transposed operand, ">" instead of ">=") fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch

from free_sparse_attention_block_b200 import inputs
from oracle import sol_ref

D = 128
T = 64


def f32(b):
    return inputs.bf16_bits_to_f32(b)


def bf(x):
    return inputs.f32_to_bf16_bits(np.asarray(x, np.float32))


def sdpa64(q, k, v):
    """Library dense softmax attention in float64: softmax(q k^T / sqrt d) v."""
    tq = torch.from_numpy(np.asarray(q, np.float64))[None, None]
    tk = torch.from_numpy(np.asarray(k, np.float64))[None, None]
    tv = torch.from_numpy(np.asarray(v, np.float64))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)[0, 0].numpy()


def all_rows(out, N):
    """[Nq, 64, d] tile outputs of one head -> [N, d]."""
    return out.reshape(-1, out.shape[-1])[:N]


# ---------------------------------------------------------------- pooling

@pytest.mark.parametrize("N", [64, 100, 4096 + 16, 64 * 7 + 1])
def test_pool_matches_float64_block_mean(N):
    x = inputs.random_bf16((2, N, D), seed=N)
    got = sol_ref.pool(x)
    xf = f32(x).astype(np.float64)
    Nk = (N + T - 1) // T
    assert got.shape == (2, Nk, D)
    for j in range(Nk):
        blk = xf[:, j * T:min(N, (j + 1) * T)]
        want = blk.mean(axis=1)
        n = blk.shape[1]
        # sequential float32 summation bound plus the final scaling rounding
        tol = n * 2.0 ** -24 * np.abs(blk).mean(axis=1) + 2.0 ** -23 * np.abs(want)
        assert np.all(np.abs(got[:, j] - want) <= tol + 1e-30), j


def test_pool_ragged_block_divides_by_its_own_length():
    x = np.zeros((1, 70, D), np.uint16)
    x[0, 64:] = bf(np.full((6, D), 3.0))            # last block: 6 tokens of value 3
    x[0, :64] = bf(np.full((64, D), 1.0))
    got = sol_ref.pool(x)
    assert np.all(got[0, 0] == 1.0) and np.all(got[0, 1] == 3.0)


# ---------------------------------------------------------------- attention limits

def _head(N, seed=3, BH=2, d=D):
    q, k, v = inputs.small_workload(N, BH=BH, seed=seed, d=d)
    return q[0], k[0], v[0]


@pytest.mark.parametrize("N,d", [(200, D), (64 * 3, D), (200, 64)])
def test_dense_limit_equals_sdpa(N, d):
    """beta = -inf keeps every block: plain dense softmax attention (scale 1/sqrt(d) from the
    library routine, so a hard-wired head size fails at d = 64)."""
    q, k, v = _head(N, d=d)
    r = sol_ref.forward(q, k, v, float("-inf"))
    Nk = (N + T - 1) // T
    assert np.all(r["count"] == Nk)
    out = r["out"].reshape(2, Nk, T, d)
    for bh in range(2):
        want = sdpa64(f32(q[bh]), f32(k[bh]), f32(v[bh]))
        np.testing.assert_allclose(all_rows(out[bh], N), want, rtol=0, atol=1e-10)


@pytest.mark.parametrize("beta", [1e30, float("inf")])
def test_large_beta_keeps_no_block(beta):
    q, k, v = _head(64 * 5 + 16)
    r = sol_ref.route(q, sol_ref.pool(k), beta)
    assert r["count"].sum() == 0 and r["mask"].sum() == 0


@pytest.mark.parametrize("d", [D, 64])
def test_zero_selection_equals_dense_over_pooled_sequence(d):
    """With nothing kept, each block j acts as n_j copies of (k_bar_j, v_bar_j)."""
    N = 64 * 5 + 16
    q, k, v = _head(N, seed=11, d=d)
    r = sol_ref.forward(q, k, v, float("inf"))
    Nk = (N + T - 1) // T
    lens = [min(N, (j + 1) * T) - j * T for j in range(Nk)]
    out = r["out"].reshape(2, Nk, T, d)
    for bh in range(2):
        kk = np.repeat(r["kbar"][bh].astype(np.float64), lens, axis=0)
        vv = np.repeat(r["vbar"][bh].astype(np.float64), lens, axis=0)
        want = sdpa64(f32(q[bh]), kk, vv)
        np.testing.assert_allclose(all_rows(out[bh], N), want, rtol=0, atol=1e-10)


def test_block_constant_keys_are_exact_for_every_beta():
    """If all keys of a block are equal, the pooled term equals the block's exact terms."""
    N = 64 * 6 + 16
    q, _, v = _head(N, seed=5)
    rng = np.random.default_rng(0)
    Nk = (N + T - 1) // T
    kb = bf(rng.standard_normal((2, Nk, D)).astype(np.float32) * 2.0)
    k = np.repeat(kb, [min(N, (j + 1) * T) - j * T for j in range(Nk)], axis=1)
    mixed = False
    for beta in [float("-inf"), -0.5, 0.3, 1.0, float("inf")]:
        r = sol_ref.forward(q, k, v, beta)
        mixed |= bool(np.any((r["count"] > 0) & (r["count"] < Nk)))
        out = r["out"].reshape(2, Nk, T, D)
        for bh in range(2):
            want = sdpa64(f32(q[bh]), f32(k[bh]), f32(v[bh]))
            # exact up to the float32 rounding of the pooled values v_bar (|v| <~ 5, 2^-24 rel)
            np.testing.assert_allclose(all_rows(out[bh], N), want, rtol=0, atol=2e-6)
    assert mixed, "no beta produced a mix of kept and skipped blocks"


@pytest.mark.parametrize("N", [64 * 4 + 23, 64 * 3])
def test_any_mask_equals_dense_over_substituted_sequence(N):
    """For any mask, a tile's output equals dense attention of its rows over the sequence in
    which every skipped block j is replaced by n_j copies of (k_bar_j, v_bar_j)."""
    q, k, v = _head(N, seed=21)
    Nk = (N + T - 1) // T
    kbar, vbar = sol_ref.pool(k), sol_ref.pool(v)
    units = np.arange(2 * Nk, dtype=np.int64)
    rng = np.random.default_rng(N)
    mask = (rng.random((units.size, Nk)) < 0.5).astype(np.uint8)
    mask[0] = 0
    mask[1] = 1
    out = sol_ref.attend(q, k, v, kbar, vbar, units, mask)
    for u in units:
        bh, i = divmod(int(u), Nk)
        ks, vs = [], []
        for j in range(Nk):
            lo, hi = j * T, min(N, (j + 1) * T)
            if mask[u, j]:
                ks.append(f32(k[bh, lo:hi]).astype(np.float64))
                vs.append(f32(v[bh, lo:hi]).astype(np.float64))
            else:
                ks.append(np.repeat(kbar[bh, j:j + 1].astype(np.float64), hi - lo, 0))
                vs.append(np.repeat(vbar[bh, j:j + 1].astype(np.float64), hi - lo, 0))
        rows = slice(i * T, min(N, (i + 1) * T))
        want = sdpa64(f32(q[bh, rows]), np.concatenate(ks), np.concatenate(vs))
        np.testing.assert_allclose(out[u, :want.shape[0]], want, rtol=0, atol=1e-10)


# ---------------------------------------------------------------- hand-worked closed forms

def _two_block(three=False):
    N = 192 if three else 128
    q = np.zeros((1, N, D), np.float32)
    k = np.zeros((1, N, D), np.float32)
    v = np.zeros((1, N, D), np.float32)
    q[0, :, 0] = 8.0
    k[0, :64, 0] = 2.0
    v[0, :64, 0] = 1.0
    k[0, 64:96, 0] = 1.0
    v[0, 64:96, 1] = 1.0
    k[0, 96:128, 0] = -1.0
    v[0, 96:128, 1] = -1.0
    if three:
        k[0, 128:192, 0] = -1.0
    return bf(q), bf(k), bf(v)


def test_two_block_example_routing(golden):
    q, k, v = _two_block()
    r = sol_ref.route(q, sol_ref.pool(k), 0.5)
    for i in range(2):
        np.testing.assert_allclose(r["proxy"][i], [golden["proxy0"], golden["proxy1"]], atol=1e-6)
        np.testing.assert_allclose(r["mu"][i], golden["mu"], atol=1e-6)
        np.testing.assert_allclose(r["sigma"][i], golden["sigma"], atol=1e-6)
    expected_masks = {0.5: [1, 0], 1.5: [0, 0], -1.5: [1, 1], 0.999: [1, 0], 1.001: [0, 0],
                      -0.999: [1, 0], -1.001: [1, 1],
                      1.0: [1, 0], -1.0: [1, 1]}        # exact ties: ">=" keeps the block
    for beta, m in expected_masks.items():
        r = sol_ref.route(q, sol_ref.pool(k), beta)
        assert r["mask"].tolist() == [m, m], beta


@pytest.mark.parametrize("beta", [0.5, 1.5, -1.5])
def test_two_block_example_output(golden, beta):
    q, k, v = _two_block()
    r = sol_ref.forward(q, k, v, beta)
    out = r["out"].reshape(-1, D)
    want = np.zeros(D)
    want[0] = golden[f"out_beta_{beta}_ch0"]
    want[1] = golden[f"out_beta_{beta}_ch1"]
    np.testing.assert_allclose(out, np.broadcast_to(want, out.shape), atol=1e-6)


def test_three_block_population_sigma(golden):
    q, k, v = _two_block(three=True)
    r = sol_ref.route(q, sol_ref.pool(k), 0.0)
    z = (r["proxy"][0].astype(np.float64) - r["mu"][0]) / r["sigma"][0]
    np.testing.assert_allclose(z, [golden["z3_0"], golden["z3_1"], golden["z3_2"]], atol=1e-6)
    cases = {1.2: [1, 0, 0],      # population z0 = 1.336 >= 1.2; a sample sigma would give 1.091
             1.4: [0, 0, 0], -0.5: [1, 1, 0], -1.1: [1, 1, 1], 0.0: [1, 0, 0]}
    for beta, m in cases.items():
        r = sol_ref.route(q, sol_ref.pool(k), beta)
        assert r["mask"][0].tolist() == m, beta


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_two_blocks_have_unit_z_scores(seed):
    """Nk = 2: the z-scores are exactly +-1 whatever the data, so the upper block is kept iff
    beta <= 1 and the lower one iff beta <= -1."""
    q, k, _ = _head(128, seed=seed, BH=1)
    kbar = sol_ref.pool(k)
    for beta, n in [(0.99, 1), (1.01, 0), (-0.99, 1), (-1.01, 2)]:
        r = sol_ref.route(q, kbar, beta)
        assert np.all(r["count"] == n), (beta, r["count"])


# ---------------------------------------------------------------- routing vs library statistics

@pytest.mark.parametrize("beta,d", [(0.0, D), (0.7, D), (1.3, D), (-0.4, D), (0.7, 64)])
def test_routing_matches_numpy_statistics(beta, d):
    N = 64 * 40 + 16
    q, k, _ = _head(N, seed=9, d=d)
    Nk = (N + T - 1) // T
    r = sol_ref.route(q, sol_ref.pool(k), beta)
    qf, kf = f32(q).astype(np.float64), f32(k).astype(np.float64)
    band = 1e-5
    for bh in range(2):
        qb = np.stack([qf[bh, j * T:(j + 1) * T].mean(0) for j in range(Nk)])
        kb = np.stack([kf[bh, j * T:(j + 1) * T].mean(0) for j in range(Nk)])
        S = qb @ kb.T / math.sqrt(d)
        mu, sd = S.mean(1), S.std(1)
        tau = mu + beta * sd
        sl = slice(bh * Nk, (bh + 1) * Nk)
        np.testing.assert_allclose(r["proxy"][sl], S, atol=2e-5)
        np.testing.assert_allclose(r["mu"][sl], mu, atol=2e-5)
        np.testing.assert_allclose(r["sigma"][sl], sd, atol=2e-5)
        far = np.abs(S - tau[:, None]) > band
        assert np.array_equal(r["mask"][sl][far], (S >= tau[:, None])[far])
        assert far.mean() > 0.99


def test_routing_density_is_moderate_on_the_field_workload():
    """Diagnostic sanity: beta = 0.5 keeps a fraction of blocks in the range a normal row gives."""
    q, k, _ = _head(64 * 64, seed=4)
    r = sol_ref.route(q, sol_ref.pool(k), 0.5)
    dens = r["count"].mean() / 64
    assert 0.1 < dens < 0.5


# ---------------------------------------------------------------- invariances

def _int_head(N, seed):
    rng = np.random.default_rng(seed)
    q = bf(rng.integers(-1, 2, size=(1, N, D)).astype(np.float32))
    k = bf(rng.integers(-1, 2, size=(1, N, D)).astype(np.float32))
    v = bf(rng.integers(-3, 4, size=(1, N, D)).astype(np.float32))   # exact block sums
    return q, k, v


def test_mask_invariant_to_query_scaling():
    q, k, _ = _head(64 * 12 + 5, seed=13)
    kbar = sol_ref.pool(k)
    q2 = bf(f32(q) * 2.0)
    for beta in [0.2, 1.0]:
        a, b = sol_ref.route(q, kbar, beta), sol_ref.route(q2, kbar, beta)
        assert np.array_equal(a["mask"], b["mask"])
        assert np.array_equal(a["proxy"] * 2.0, b["proxy"])


def test_common_key_shift_changes_nothing():
    N = 64 * 8
    q, k, v = _int_head(N, 1)
    w = np.random.default_rng(2).integers(-1, 2, size=(D,)).astype(np.float32)
    k2 = bf(f32(k) + w)
    for beta in [-0.3, 0.5, 1.2]:
        a = sol_ref.forward(q, k, v, beta)
        b = sol_ref.route(q, sol_ref.pool(k2), beta)
        far = np.abs(a["proxy"] - a["tau"][:, None].astype(np.float32)) > 1e-5
        assert np.array_equal(a["mask"][far], b["mask"][far])
        ob = sol_ref.forward(q, k2, v, beta, mask_override=a["mask"])["out"]
        np.testing.assert_allclose(a["out"], ob, atol=1e-12)


def test_permutations_within_and_across_blocks():
    N = 64 * 6
    Nk = N // T
    q, k, v = _int_head(N, 3)
    rng = np.random.default_rng(4)
    beta = 0.4
    a = sol_ref.forward(q, k, v, beta)
    # within each key block
    perm = np.concatenate([j * T + rng.permutation(T) for j in range(Nk)])
    b = sol_ref.forward(q, k[:, perm], v[:, perm], beta)
    assert np.array_equal(a["mask"], b["mask"])
    np.testing.assert_allclose(a["out"], b["out"], atol=1e-12)
    # whole key/value blocks: masks permute with the blocks, outputs are unchanged
    bp = rng.permutation(Nk)
    tok = np.concatenate([np.arange(j * T, (j + 1) * T) for j in bp])
    c = sol_ref.forward(q, k[:, tok], v[:, tok], beta)
    assert np.array_equal(a["mask"][:, bp], c["mask"])
    np.testing.assert_allclose(a["out"], c["out"], atol=1e-12)
    # query rows within a tile: routing unchanged, output rows permute
    qp = np.concatenate([j * T + rng.permutation(T) for j in range(Nk)])
    d_ = sol_ref.forward(q[:, qp], k, v, beta)
    assert np.array_equal(a["mask"], d_["mask"])
    np.testing.assert_allclose(a["out"].reshape(-1, D)[qp], d_["out"].reshape(-1, D), atol=1e-12)
