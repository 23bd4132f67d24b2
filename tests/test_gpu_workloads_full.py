"""Full-size workloads (Wan2.1-14B-shaped, HunyuanVideo-shaped, long-video stress) in the launch
configuration the benchmark times (sol_attn_pool + sol_attn_fwd over all heads), checked against
the oracle on sampled query tiles: per head the first, second, second-to-last and last tile (the
last one partial for Wan and Hunyuan) plus random ones."""
import numpy as np
import pytest

from free_sparse_attention_block_b200 import inputs
from parity import check_parity, default_units, gpu_run

pytestmark = pytest.mark.gpu

CASES = [("wan", 0.5), ("wan", 2.0), ("hunyuan", 1.0), ("long", 2.0)]


@pytest.mark.parametrize("name,beta", CASES)
def test_full_size_sampled(name, beta):
    wl = inputs.WORKLOADS[name]
    q, k, v = inputs.gen_workload(wl)
    BH, Nq = wl.B * wl.H, wl.nq
    rng = np.random.default_rng(wl.seed)
    heads = sorted({0, BH - 1, *rng.integers(0, BH, size=2).tolist()})
    units = default_units(BH, Nq, per_head=6, seed=wl.seed)
    units = units[np.isin(units // Nq, heads)]
    g = gpu_run(q, k, v, beta, units=units, with_proxy=True)
    rep = {}
    check_parity(q, k, v, beta, g, units, report=rep)
    print(f"{name} beta={beta}: {rep}")
