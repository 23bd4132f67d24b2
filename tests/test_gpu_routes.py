"""Top-k and top-p routing (the page's prior-art rules) on the fused CUDA kernel, against the CPU
oracle's selection and attention, through the C ABI."""
import dataclasses

import numpy as np
import pytest

from free_sparse_attention_block_b200 import inputs
from parity import check_rule_parity, default_units, gpu_run_rule

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rule,param", [("topk", 1), ("topk", 8), ("topk", 37), ("topk", 64),
                                        ("topk", 1000), ("topk", 0), ("topp", 0.5), ("topp", 0.9),
                                        ("topp", 0.99), ("topp", 1.0), ("topp", 0.0), ("topp", 1e-6)])
def test_tiny_all_tiles(rule, param):
    wl = inputs.WORKLOADS["tiny"]
    q, k, v = inputs.gen_workload(wl)
    g = gpu_run_rule(q, k, v, rule, param)
    check_rule_parity(q, k, v, rule, param, g)
    Nk = wl.nq
    if rule == "topk":
        assert np.all(g["density"] == min(param, Nk))
    if rule == "topp" and param >= 1.0:
        assert np.all(g["density"] == Nk)
    if rule == "topp" and param <= 0.0:
        assert np.all(g["density"] == 0)


@pytest.mark.parametrize("N", [1, 65, 129, 64 * 9 + 16, 2048 + 77])
@pytest.mark.parametrize("rule,param", [("topk", 5), ("topp", 0.8)])
def test_ragged_lengths(N, rule, param):
    q, k, v = inputs.small_workload(N, BH=3, seed=N + 7)
    g = gpu_run_rule(q, k, v, rule, param)
    check_rule_parity(q, k, v, rule, param, g)


@pytest.mark.parametrize("rule,param", [("topk", 5), ("topk", 2), ("topk", 11), ("topp", 0.5),
                                        ("topp", 0.3)])
def test_exact_score_ties_are_broken_by_block_index(rule, param):
    """Three distinct key blocks repeated over 13 blocks: every proxy row has groups of exactly
    equal scores, so the cut falls inside a tie group and the kernel must keep the lowest
    indices of it."""
    N = 64 * 12 + 16
    q, _, v = inputs.small_workload(N, BH=2, seed=31)
    rng = np.random.default_rng(5)
    base = inputs.f32_to_bf16_bits(rng.standard_normal((3, 64, 128)).astype(np.float32))
    pattern = [0, 1, 2, 1, 0, 2, 2, 1, 0, 0, 1, 2]
    k = np.concatenate([base[p] for p in pattern] + [base[1][:16]], axis=0)
    k = np.broadcast_to(k, (1, 2, N, 128)).copy()
    g = gpu_run_rule(q, k, v, rule, param)
    check_rule_parity(q, k, v, rule, param, g)


def test_head_dim_64():
    q, k, v = inputs.small_workload(64 * 20 + 9, BH=2, seed=44, d=64)
    for rule, param in [("topk", 6), ("topp", 0.85)]:
        g = gpu_run_rule(q, k, v, rule, param)
        check_rule_parity(q, k, v, rule, param, g)


@pytest.mark.parametrize("rule,param", [("topk", 64), ("topp", 0.9)])
def test_mid_sampled_tiles(rule, param):
    wl = inputs.WORKLOADS["mid"]
    q, k, v = inputs.gen_workload(wl)
    units = default_units(wl.B * wl.H, wl.nq, per_head=6, seed=3)
    g = gpu_run_rule(q, k, v, rule, param, units=units)
    check_rule_parity(q, k, v, rule, param, g)


def test_wan_shape_sampled_heads():
    """Wan2.1-shaped rows (1182 blocks, last block 16 tokens) on two heads."""
    wl = dataclasses.replace(inputs.WORKLOADS["wan"], H=2)
    q, k, v = inputs.gen_workload(wl)
    units = default_units(2, wl.nq, per_head=4, seed=9)
    for rule, param in [("topk", 300), ("topp", 0.95)]:
        g = gpu_run_rule(q, k, v, rule, param, units=units)
        check_rule_parity(q, k, v, rule, param, g)
