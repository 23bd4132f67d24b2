"""Full-size workloads (Wan2.1-14B-shaped, HunyuanVideo-shaped, long-video stress) in the launch
configuration the benchmark times (sol_attn_pool + sol_attn_fwd over all heads), over each
workload's whole beta sweep, checked against the oracle on sampled query tiles: per head the
first, second, second-to-last and last tile (the last one partial for Wan and Hunyuan) plus random
ones, on four heads.  One case runs the Wan2.1 shape with 64-channel heads."""
import dataclasses

import numpy as np
import pytest

from free_sparse_attention_block_b200 import inputs
from parity import check_parity, default_units, gpu_run

pytestmark = pytest.mark.gpu

CASES = ([("wan", 128, b) for b in (0.5, 1.0, 1.5, 2.0)] + [("wan", 64, 0.5)] +
         [("hunyuan", 128, b) for b in (0.5, 1.0, 1.5, 2.0, 2.5)] +
         [("long", 128, b) for b in (1.5, 2.0, 2.5)])

_last = {}


def workload_inputs(name, d):
    """Inputs of one workload, kept while consecutive cases use it (one workload at a time)."""
    if (name, d) not in _last:
        _last.clear()
        wl = dataclasses.replace(inputs.WORKLOADS[name], d=d)
        _last[(name, d)] = (wl, inputs.gen_workload(wl))
    return _last[(name, d)]


@pytest.mark.parametrize("name,d,beta", CASES)
def test_full_size_sampled(name, d, beta):
    wl, (q, k, v) = workload_inputs(name, d)
    BH, Nq = wl.B * wl.H, wl.nq
    rng = np.random.default_rng(wl.seed)
    heads = sorted({0, BH - 1, *rng.integers(0, BH, size=2).tolist()})
    units = default_units(BH, Nq, per_head=6, seed=wl.seed)
    units = units[np.isin(units // Nq, heads)]
    g = gpu_run(q, k, v, beta, units=units, with_proxy=True)
    rep = {}
    check_parity(q, k, v, beta, g, units, report=rep)
    print(f"{name} d={d} beta={beta}: {rep}")


def teardown_module():
    _last.clear()
