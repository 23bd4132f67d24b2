"""Failure detection without a GPU fault: a pipeline wait that nothing will ever satisfy must give
up after its time limit, report SOL_ERR_TIMEOUT through the status words, free its resources and
leave the CUDA context usable for the next call."""
import numpy as np
import pytest
import torch

import free_sparse_attention_block_b200 as sol
from free_sparse_attention_block_b200 import inputs
from parity import check_parity, default_units, gpu_run, to_dev

pytestmark = pytest.mark.gpu


def test_stalled_wait_reports_timeout_and_context_survives():
    N = 64 * 8
    q, k, v = inputs.small_workload(N, BH=2, seed=5)
    tq, tk, tv = to_dev(q), to_dev(k), to_dev(v)
    ws = torch.zeros(sol.sol_attn_workspace_bytes(1, 2, N, 128), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(tq)
    sol.sol_attn_pool(tk, tv, ws)
    st = sol.sol_attn_fwd_debug(tq, tk, tv, 0.5, ws, out, fault_flags=1, timeout_ms=50)
    assert sol.STATUS[st] == "SOL_ERR_TIMEOUT"
    # the status words were read and cleared; the context still runs a correct forward
    assert sol.sol_attn_read_status(ws)[0] == 0
    g = gpu_run(q, k, v, 0.5)
    check_parity(q, k, v, 0.5, g, default_units(2, 8, None))


def test_split_merge_wait_reports_timeout_and_context_survives():
    """The second half of a split work unit waits (bounded) for the first half's rows; with the
    first half's final count withheld (fault flag 4, every unit split by flag 2) that wait must
    run out, report SOL_ERR_TIMEOUT and leave the context usable."""
    N = 64 * 8
    q, k, v = inputs.small_workload(N, BH=2, seed=6)
    tq, tk, tv = to_dev(q), to_dev(k), to_dev(v)
    ws = torch.zeros(sol.sol_attn_workspace_bytes(1, 2, N, 128), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(tq)
    sol.sol_attn_pool(tk, tv, ws)
    st = sol.sol_attn_fwd_debug(tq, tk, tv, 0.5, ws, out, fault_flags=2 | 4, timeout_ms=50)
    assert sol.STATUS[st] == "SOL_ERR_TIMEOUT"
    assert sol.sol_attn_read_status(ws)[0] == 0
    g = gpu_run(q, k, v, 0.5)
    check_parity(q, k, v, 0.5, g, default_units(2, 8, None))


def test_call_after_a_timed_out_split_merge_on_the_same_workspace():
    """A split unit whose merge wait ran out leaves its counter part way (both halves arrived,
    the final count withheld).  The next call on the same pooled workspace, without re-pooling and
    with different queries, must not take those counts for arrivals of its own (it would merge
    the previous call's partial rows): every unit split again, against the oracle."""
    N = 64 * 8
    q, k, v = inputs.small_workload(N, BH=2, seed=6)
    q2, _, _ = inputs.small_workload(N, BH=2, seed=66)
    tq, tk, tv = to_dev(q), to_dev(k), to_dev(v)
    ws = torch.zeros(sol.sol_attn_workspace_bytes(1, 2, N, 128), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(tq)
    sol.sol_attn_pool(tk, tv, ws)
    st = sol.sol_attn_fwd_debug(tq, tk, tv, 0.5, ws, out, fault_flags=2 | 4, timeout_ms=50)
    assert sol.STATUS[st] == "SOL_ERR_TIMEOUT"
    counters = ws[256:256 + 4 * 8].view(torch.int32)
    assert int((counters & 3).max()) == 2            # left part way by the launch that gave up
    Nq = 8
    tq2 = to_dev(q2)
    out2 = torch.full_like(tq2, float("nan"))
    dens = torch.full((1, 2, Nq), -1, dtype=torch.int32, device="cuda")
    mask = torch.full((1, 2, Nq, Nq), 255, dtype=torch.uint8, device="cuda")
    stats = torch.full((1, 2, Nq, 3), float("nan"), dtype=torch.float32, device="cuda")
    st = sol.sol_attn_fwd_debug(tq2, tk, tv, 0.5, ws, out2, dens, None, mask, stats, fault_flags=2)
    assert st == 0, sol.STATUS.get(st)
    kb32 = sol.workspace_views(ws, 1, 2, N, 128)[0]
    g = dict(out=out2.float().cpu().numpy(), density=dens.cpu().numpy(), mask=mask.cpu().numpy(),
             stats=stats.cpu().numpy(), kbar32=kb32.cpu().numpy(), units=None)
    check_parity(q2, k, v, 0.5, g, default_units(2, Nq, None))
