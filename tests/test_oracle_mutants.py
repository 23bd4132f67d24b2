"""The oracle pins must catch plausible mistakes.

Each case plants one mistake into a temporary copy of oracle/sol_ref.c (on the CPU only), builds
it, and checks that at least one independent pin rejects the mutant: a dropped ln(n_j), a missing
denominator term, the sign of beta*sigma, a sample standard deviation, a wrong pooling divisor on
the partial block, ">" instead of ">=", a missing 1/sqrt(d), or the wrong tile's rows.
"""
import ctypes as C
import math
import os
import subprocess

import numpy as np
import pytest
import torch

from free_sparse_attention_block_b200 import inputs
from oracle import sol_ref

SRC = sol_ref.SRC
D, T = 128, 64

MUTANTS = {
    "drop_ln_nj": ("z[p++] = s * scale + log((double)nj);", "z[p++] = s * scale;"),
    "numerator_only": ("const float *vb = vbar + (bh * Nk + j) * d;\n                    den += w;",
                       "const float *vb = vbar + (bh * Nk + j) * d;"),
    "minus_beta_sigma": ("tau = mu + (double)beta * sigma;", "tau = mu - (double)beta * sigma;"),
    "sample_sigma": ("sqrt(ss / (double)Nk)", "sqrt(ss / (double)(Nk > 1 ? Nk - 1 : 1))"),
    "pool_divides_by_T": ("const float inv = 1.0f / (float)n;", "const float inv = 1.0f / (float)SOL_REF_T;"),
    "strict_threshold": ("(double)row[j] >= tau ? 1 : 0", "(double)row[j] > tau ? 1 : 0"),
    "no_score_scale": ("z[p++] = s * scale;\n", "z[p++] = s;\n"),
    "wrong_query_tile": ("const int64_t tok = i * SOL_REF_T + r;", "const int64_t tok = (i + 1) % Nq * SOL_REF_T + r;"),
}


class Mutant:
    def __init__(self, lib):
        self.lib = lib

    def pool(self, x):
        x = np.ascontiguousarray(x, np.uint16).reshape(-1, x.shape[-2], x.shape[-1])
        BH, N, d = x.shape
        out = np.empty((BH, (N + T - 1) // T, d), np.float32)
        assert self.lib.sol_ref_pool(sol_ref._ptr(x), BH, N, d, sol_ref._ptr(out)) == 0
        return out

    def route(self, q, kbar, beta):
        q = np.ascontiguousarray(q, np.uint16).reshape(-1, q.shape[-2], q.shape[-1])
        BH, N, d = q.shape
        Nk = (N + T - 1) // T
        units = np.arange(BH * Nk, dtype=np.int64)
        mask = np.empty((units.size, Nk), np.uint8)
        stats = np.empty((units.size, 3))
        rc = self.lib.sol_ref_route(sol_ref._ptr(q), sol_ref._ptr(np.ascontiguousarray(kbar)), BH, N, d,
                                    C.c_float(beta), sol_ref._ptr(units), units.size, None,
                                    sol_ref._ptr(stats), sol_ref._ptr(mask), None)
        assert rc == 0
        return mask, stats

    def forward(self, q, k, v, beta):
        q = np.ascontiguousarray(q, np.uint16).reshape(-1, q.shape[-2], q.shape[-1])
        BH, N, d = q.shape
        kbar, vbar = self.pool(k), self.pool(v)
        mask, _ = self.route(q, kbar, beta)
        units = np.arange(mask.shape[0], dtype=np.int64)
        out = np.zeros((units.size, T, d))
        rc = self.lib.sol_ref_attend(*(sol_ref._ptr(np.ascontiguousarray(a)) for a in
                                       (q, k.reshape(q.shape), v.reshape(q.shape), kbar, vbar)),
                                     BH, N, d, sol_ref._ptr(units), units.size, sol_ref._ptr(mask),
                                     sol_ref._ptr(out))
        assert rc == 0
        return out.reshape(BH, -1, d)[:, :N], mask


def build_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert old in src, f"mutation site for {name} not found"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new, 1))
    so = tmp_path / f"{name}.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
                    "-o", str(so), str(path), "-lm"], check=True)
    lib = C.CDLL(str(so))
    i64, p = C.c_int64, C.c_void_p
    lib.sol_ref_pool.argtypes = [p, i64, i64, i64, p]
    lib.sol_ref_route.argtypes = [p, p, i64, i64, i64, C.c_float, p, i64, p, p, p, p]
    lib.sol_ref_attend.argtypes = [p, p, p, p, p, i64, i64, i64, p, i64, p, p]
    return Mutant(lib)


def f32(b):
    return inputs.bf16_bits_to_f32(b)


def sdpa64(q, k, v):
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v))[0, 0].numpy()


def pins_pass(m: Mutant) -> bool:
    """A compact run of the independent pins; False as soon as one rejects the oracle."""
    # pooling vs float64 means on a ragged length
    x = inputs.random_bf16((1, 100, D), seed=3)
    want = np.stack([f32(x[0, j * T:(j + 1) * T]).astype(np.float64).mean(0) for j in range(2)])
    if not np.allclose(m.pool(x)[0], want, atol=1e-5):
        return False
    # dense limit, ragged
    N = 200
    q, k, v = (a[0] for a in inputs.small_workload(N, BH=1, seed=3))
    out, _ = m.forward(q, k, v, -math.inf)
    if not np.allclose(out[0], sdpa64(f32(q[0]), f32(k[0]), f32(v[0])), atol=1e-9):
        return False
    # nothing kept: dense over the pooled sequence
    out, mask = m.forward(q, k, v, math.inf)
    if mask.sum() != 0:
        return False
    kb, vb = m.pool(k), m.pool(v)
    lens = [min(N, (j + 1) * T) - j * T for j in range((N + T - 1) // T)]
    want = sdpa64(f32(q[0]), np.repeat(kb[0].astype(np.float64), lens, 0), np.repeat(vb[0].astype(np.float64), lens, 0))
    if not np.allclose(out[0], want, atol=1e-9):
        return False
    # hand-worked closed forms
    from test_oracle_pins import _two_block
    q2, k2, v2 = _two_block()
    for beta, mm in [(0.5, [1, 0]), (1.5, [0, 0]), (-1.5, [1, 1]), (1.0, [1, 0]), (-1.0, [1, 1])]:
        mask, _ = m.route(q2, m.pool(k2), beta)
        if mask.tolist() != [mm, mm]:
            return False
    out, _ = m.forward(q2, k2, v2, 0.5)
    if not np.allclose(out[0, :, 0], math.exp(math.sqrt(2)) / (math.exp(math.sqrt(2)) + 1), atol=1e-6):
        return False
    q3, k3, v3 = _two_block(three=True)
    for beta, mm in [(1.2, [1, 0, 0]), (-0.5, [1, 1, 0])]:
        mask, _ = m.route(q3, m.pool(k3), beta)
        if mask[0].tolist() != mm:
            return False
    return True


def test_unmutated_oracle_passes_compact_pins(tmp_path):
    src = open(SRC).read()
    path = tmp_path / "same.c"
    path.write_text(src)
    MUTANTS["_identity"] = ("", "")
    try:
        m = build_mutant("_identity", tmp_path)
    finally:
        MUTANTS.pop("_identity")
    assert pins_pass(m)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    assert not pins_pass(build_mutant(name, tmp_path)), f"mutant {name} passed every pin"
