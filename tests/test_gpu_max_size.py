"""The largest supported sequence: N = 524288 tokens = 8192 key blocks, whose two float proxy rows
fill the 64 KB of shared memory set aside for them (at d = 128 the whole K/V ring, at d = 64 the
ring plus the space after it).  One head of the long-video generator, sampled query tiles checked
against the oracle, for the threshold rule and the rank rules."""
import dataclasses
import functools

import numpy as np
import pytest

from free_sparse_attention_block_b200 import inputs
from parity import check_parity, check_rule_parity, default_units, gpu_run, gpu_run_rule

pytestmark = pytest.mark.gpu

N_MAX = 8192 * 64


def max_workload(d: int):
    wl = dataclasses.replace(inputs.WORKLOADS["long"], name=f"max_d{d}", H=1, N=N_MAX,
                             grid=(128, 64, 64), d=d)
    assert wl.nq == 8192
    return wl


@functools.lru_cache(maxsize=2)
def max_inputs(d: int):
    """q, k, v of the maximum-length head (about 30 s to generate; shared by the tests)."""
    return inputs.gen_workload(max_workload(d))


@pytest.mark.parametrize("d", [128, 64])
def test_threshold_rule_at_max_length(d):
    wl = max_workload(d)
    q, k, v = max_inputs(d)
    units = default_units(1, wl.nq, per_head=6, seed=11)
    g = gpu_run(q, k, v, 2.5, units=units, with_proxy=True)
    check_parity(q, k, v, 2.5, g, units)


@pytest.mark.parametrize("rule,param", [("topk", 150), ("topp", 0.5)])
def test_rank_rules_at_max_length(rule, param):
    wl = max_workload(128)
    q, k, v = max_inputs(128)
    units = default_units(1, wl.nq, per_head=4, seed=12)
    g = gpu_run_rule(q, k, v, rule, param, units=units)
    check_rule_parity(q, k, v, rule, param, g)
    if rule == "topk":
        assert np.all(g["density"] == 150)
