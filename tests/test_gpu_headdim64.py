"""Head dimension d = 64 (the other video-DiT head size): the same fused forward, compiled for
64-channel rows, against the CPU oracle at d = 64, element by element."""
import dataclasses

import numpy as np
import pytest

from free_sparse_attention_block_b200 import inputs
from parity import check_parity, default_units, gpu_run

pytestmark = pytest.mark.gpu

INF = float("inf")
D = 64


@pytest.mark.parametrize("N", [1, 63, 65, 128, 129, 200, 64 * 9 + 16, 2048 + 77])
@pytest.mark.parametrize("beta", [0.3, 1.2])
def test_ragged_lengths_d64(N, beta):
    q, k, v = inputs.small_workload(N, BH=3, seed=N + 100, d=D)
    g = gpu_run(q, k, v, beta)
    check_parity(q, k, v, beta, g, default_units(3, (N + 63) // 64, None))


@pytest.mark.parametrize("beta", [-INF, INF, 0.0, 2.5])
def test_extreme_betas_d64(beta):
    q, k, v = inputs.small_workload(64 * 20 + 16, BH=2, seed=5, d=D)
    g = gpu_run(q, k, v, beta)
    Nq = 21
    check_parity(q, k, v, beta, g, default_units(2, Nq, None))
    if beta == INF:
        assert np.all(g["density"] == 0)
    if beta == -INF:
        assert np.all(g["density"] == Nq)


def test_block_constant_keys_match_dense_d64():
    N = 64 * 12 + 16
    q, _, v = inputs.small_workload(N, BH=2, seed=9, d=D)
    rng = np.random.default_rng(2)
    Nk = 13
    kb = inputs.f32_to_bf16_bits(rng.standard_normal((1, 2, Nk, D)).astype(np.float32) * 2)
    k = np.repeat(kb, [64] * 12 + [16], axis=2)
    for beta in [-INF, 0.3, INF]:
        g = gpu_run(q, k, v, beta)
        check_parity(q, k, v, beta, g, default_units(2, Nk, None))


@pytest.mark.parametrize("beta", [0.5, 1.5])
def test_mid_shape_d64_sampled_tiles(beta):
    """The 12-head, 16384-token field workload generated with 64-channel heads."""
    wl = dataclasses.replace(inputs.WORKLOADS["mid"], d=D)
    q, k, v = inputs.gen_workload(wl)
    g = gpu_run(q, k, v, beta)
    check_parity(q, k, v, beta, g, default_units(wl.B * wl.H, wl.nq, per_head=6, seed=int(beta * 10)))
