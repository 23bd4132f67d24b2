"""Work units (query-tile pairs) split over two CTAs, against the oracle.

sol_attn_fwd splits the units of a last wave of CTAs that would run less than half full: each of
two CTAs takes every other item of the unit's work list, and the second to finish merges the two
partial rows (their own running max and sum).  The debug entry point's fault flag 2 splits every
unit the workspace holds (up to 128), so small shapes exercise the merge, including halves with no
item at all (a unit with a single item)."""
import numpy as np
import pytest
import torch

import free_sparse_attention_block_b200 as sol
from free_sparse_attention_block_b200 import inputs
from parity import check_parity, check_rule_parity, default_units, gpu_run_rule, to_dev

pytestmark = pytest.mark.gpu

INF = float("inf")
SPLIT_ALL = 2
SPLIT_CNT = slice(256, 256 + 4 * 128)   # split counters in the workspace header


def split_run(q, k, v, beta, flags=SPLIT_ALL):
    B, H, N, d = q.shape
    Nq = (N + 63) // 64
    tq, tk, tv = to_dev(q), to_dev(k), to_dev(v)
    ws = torch.full((sol.sol_attn_workspace_bytes(B, H, N, d),), 0x5A, dtype=torch.uint8, device="cuda")
    out = torch.full_like(tq, float("nan"))
    dens = torch.full((B, H, Nq), -1, dtype=torch.int32, device="cuda")
    proxy = torch.full((B, H, Nq, Nq), float("nan"), dtype=torch.float32, device="cuda")
    mask = torch.full((B, H, Nq, Nq), 255, dtype=torch.uint8, device="cuda")
    stats = torch.full((B, H, Nq, 3), float("nan"), dtype=torch.float32, device="cuda")
    sol.sol_attn_pool(tk, tv, ws)        # also clears the header (status words, split counters)
    st = sol.sol_attn_fwd_debug(tq, tk, tv, beta, ws, out, dens, proxy, mask, stats, fault_flags=flags)
    assert st == 0, sol.STATUS.get(st)
    torch.cuda.synchronize()
    # every merging CTA returned its counter to zero
    assert int(ws[SPLIT_CNT].view(torch.int32).abs().sum()) == 0
    kb32 = sol.workspace_views(ws, B, H, N, d)[0]
    return dict(out=out.float().cpu().numpy(), density=dens.cpu().numpy(), mask=mask.cpu().numpy(),
                proxy=proxy.cpu().numpy(), stats=stats.cpu().numpy(), kbar32=kb32.cpu().numpy(),
                units=None)


@pytest.mark.parametrize("beta", [-INF, 0.5, INF])
def test_tiny_every_unit_split(beta):
    wl = inputs.WORKLOADS["tiny"]
    q, k, v = inputs.gen_workload(wl)
    g = split_run(q, k, v, beta)
    check_parity(q, k, v, beta, g, default_units(wl.B * wl.H, wl.nq, None))


@pytest.mark.parametrize("N", [1, 64, 65, 200, 64 * 9 + 16, 1000])
def test_ragged_every_unit_split(N):
    """N = 1 and 64: one tile, one block -- one item, so one half of the unit has none."""
    q, k, v = inputs.small_workload(N, BH=3, seed=N + 100)
    g = split_run(q, k, v, 0.4)
    check_parity(q, k, v, 0.4, g, default_units(3, (N + 63) // 64, None))


def test_head_dim_64_every_unit_split():
    q, k, v = inputs.small_workload(64 * 20 + 5, BH=4, seed=64, d=64)
    g = split_run(q, k, v, 0.5)
    check_parity(q, k, v, 0.5, g, default_units(4, 21, None))


def test_more_units_than_the_workspace_splits():
    """144 units: the first 16 run whole, the last 128 split."""
    N = 64 * 24
    q, k, v = inputs.small_workload(N, BH=12, seed=5)
    g = split_run(q, k, v, 0.6)
    check_parity(q, k, v, 0.6, g, default_units(12, 24, None))


def test_production_split_of_the_last_wave_on_mid():
    """The 12-head, 16384-token call has 1536 units, 56 past five full waves of 296 CTAs: the
    production path splits the last 84 (all in the last head).  Every tile of that head against
    the oracle; the other heads are left zero (every block kept, since sigma = 0)."""
    wl = inputs.WORKLOADS["mid"]
    q, k, v = inputs.gen_workload(wl, heads=[(0, 11)])
    g = split_run(q, k, v, 0.5, flags=0)
    check_parity(q, k, v, 0.5, g, np.arange(11 * wl.nq, 12 * wl.nq, dtype=np.int64))


@pytest.mark.parametrize("rule,param", [("topk", 62), ("topp", 0.5)])
def test_production_split_of_the_last_wave_rank_rules(rule, param):
    """The rank rules' kernel splits the same last 84 units of the 12-head, 16384-token call
    (after its radix selection); the last head's tiles against the oracle's selection and
    outputs."""
    wl = inputs.WORKLOADS["mid"]
    q, k, v = inputs.gen_workload(wl, heads=[(0, 11)])
    units = np.arange(11 * wl.nq, 12 * wl.nq, dtype=np.int64)
    g = gpu_run_rule(q, k, v, rule, param, units=units)
    check_rule_parity(q, k, v, rule, param, g)
