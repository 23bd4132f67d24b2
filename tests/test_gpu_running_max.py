"""Rows whose running maximum keeps rising, against the oracle.

Queries and keys share one direction u per head: q = u + noise, and key block j is
(1 + j) * (u + noise), so the logits of block j grow in proportion to 1 + j and in the undamped
query rows (odd rows) the largest logit of each block exceeds that of the block before by more
than 2^8 in the log2 domain; the even rows are damped by 0.05 and settle after their first item.
Every item then moves the running maximum of half the rows of each warp and not of the other
half, which drives the online-softmax rescale of O (both head sizes) and, at d = 64, the repeated
exponential pass in some lanes only.
"""
import math

import numpy as np
import pytest

from free_sparse_attention_block_b200 import inputs
from parity import check_parity, default_units, gpu_run

INF = float("inf")


def growing_inputs(N: int, BH: int, d: int, seed: int):
    rng = np.random.default_rng(seed)
    u = rng.standard_normal((1, BH, 1, d)).astype(np.float32)
    q = u + 0.3 * rng.standard_normal((1, BH, N, d)).astype(np.float32)
    q[:, :, 0::2, :] *= 0.05
    k = u + 0.3 * rng.standard_normal((1, BH, N, d)).astype(np.float32)
    k *= (1.0 + np.arange(N) // 64).astype(np.float32)[None, None, :, None]
    v = rng.standard_normal((1, BH, N, d)).astype(np.float32)
    return tuple(inputs.f32_to_bf16_bits(x) for x in (q, k, v))


def block_row_max_log2(q, k, d):
    """[rows, blocks] largest logit of each key block, log2 domain, head 0 (float64)."""
    qf = inputs.bf16_bits_to_f32(q[0, 0]).astype(np.float64)
    kf = inputs.bf16_bits_to_f32(k[0, 0]).astype(np.float64)
    s = qf @ kf.T / math.sqrt(d) * math.log2(math.e)
    N = s.shape[1]
    return np.stack([s[:, j:j + 64].max(1) for j in range(0, N, 64)], axis=1)


def test_premise_on_cpu_inputs_grow():
    for d in (64, 128):
        q, k, _ = growing_inputs(64 * 12 + 20, 2, d, seed=d)
        mx = block_row_max_log2(q, k, d)
        rises = np.diff(mx, axis=1)
        assert (rises[1::2] > 8.0).mean() > 0.9        # undamped rows: nearly every block moves it
        assert (rises[0::2] > 8.0).mean() == 0.0       # damped rows: never after the first block


@pytest.mark.gpu
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("beta", [-INF, 0.5])
def test_running_max_growth(d, beta):
    N = 64 * 12 + 20
    q, k, v = growing_inputs(N, 2, d, seed=d)
    g = gpu_run(q, k, v, beta)
    check_parity(q, k, v, beta, g, default_units(2, (N + 63) // 64, None))
