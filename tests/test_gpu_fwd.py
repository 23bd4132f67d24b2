"""Fused forward (CUDA, through the C ABI) against the CPU oracle, element by element."""
import math

import numpy as np
import pytest

from free_sparse_attention_block_b200 import inputs
from parity import MAX_ABS, MEAN_ABS, check_parity, default_units, gpu_run

pytestmark = pytest.mark.gpu

INF = float("inf")


@pytest.mark.parametrize("beta", [-INF, 0.5, 1.0])
def test_tiny_all_tiles(beta):
    wl = inputs.WORKLOADS["tiny"]
    q, k, v = inputs.gen_workload(wl)
    g = gpu_run(q, k, v, beta)
    BH, Nq = wl.B * wl.H, wl.nq
    check_parity(q, k, v, beta, g, default_units(BH, Nq, None))
    if beta == -INF:
        assert np.all(g["density"] == Nq)


@pytest.mark.parametrize("N", [1, 63, 64, 65, 127, 128, 129, 191, 200, 64 * 9 + 16, 1000, 2048 + 77])
@pytest.mark.parametrize("beta", [0.3, 1.2])
def test_ragged_lengths(N, beta):
    """Partial last tiles/blocks, odd tile counts (a CTA with one routing tile), N < 64."""
    q, k, v = inputs.small_workload(N, BH=3, seed=N)
    g = gpu_run(q, k, v, beta)
    check_parity(q, k, v, beta, g, default_units(3, (N + 63) // 64, None))


@pytest.mark.parametrize("beta", [-INF, INF, 1e30, -1e30, 0.0, 2.5])
def test_extreme_betas(beta):
    q, k, v = inputs.small_workload(64 * 20 + 16, BH=2, seed=3)
    g = gpu_run(q, k, v, beta)
    Nq = 21
    check_parity(q, k, v, beta, g, default_units(2, Nq, None))
    if beta in (INF, 1e30):
        assert np.all(g["density"] == 0)
    if beta in (-INF, -1e30):
        assert np.all(g["density"] == Nq)


def test_hand_worked_example(golden):
    """The two-block closed form (tests/golden/hand_worked_blocks.txt) on the GPU."""
    from test_oracle_pins import _two_block
    q, k, v = _two_block()
    for beta, key in [(0.5, "0.5"), (1.5, "1.5"), (-1.5, "-1.5")]:
        g = gpu_run(q[None], k[None], v[None], beta)
        out = g["out"].reshape(-1, 128)
        want = np.zeros(128)
        want[0] = golden[f"out_beta_{key}_ch0"]
        want[1] = golden[f"out_beta_{key}_ch1"]
        err = np.abs(out - want[None, :])
        # the suite's output bar (bf16 output and bf16 probabilities against the exact value)
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    for beta, m in [(1.0, [1, 0]), (-1.0, [1, 1])]:      # exact ties: ">=" keeps the block
        g = gpu_run(q[None], k[None], v[None], beta)
        assert g["mask"].reshape(2, 2).tolist() == [m, m]


def test_block_constant_keys_match_dense():
    """Block-constant keys make the correction exact: output equals dense attention for any beta."""
    N = 64 * 12 + 16
    q, _, v = inputs.small_workload(N, BH=2, seed=8)
    rng = np.random.default_rng(1)
    Nk = 13
    kb = inputs.f32_to_bf16_bits(rng.standard_normal((1, 2, Nk, 128)).astype(np.float32) * 2)
    k = np.repeat(kb, [64] * 12 + [16], axis=2)
    for beta in [-INF, 0.3, INF]:
        g = gpu_run(q, k, v, beta)
        check_parity(q, k, v, beta, g, default_units(2, Nk, None))


@pytest.mark.parametrize("beta", [0.5, 1.0, 1.5, 2.0])
def test_mid_sampled_tiles(beta):
    wl = inputs.WORKLOADS["mid"]
    q, k, v = inputs.gen_workload(wl)
    g = gpu_run(q, k, v, beta)
    check_parity(q, k, v, beta, g, default_units(wl.B * wl.H, wl.nq, per_head=6, seed=int(beta * 10)))
