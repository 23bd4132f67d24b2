"""sol_attn_fwd_noalloc: the entry point for callers that cannot allocate device memory (a fixed
memory budget, a host allocator that must not be re-entered, a plugin without an allocator).
It keeps the pooled keys/values in the library's built-in scratch instead of a caller workspace.

Called through the C ABI and checked against the oracle (outputs, with the GPU's own block masks
from the workspace entry points' debug outputs for near ties) and against the workspace entry
points (sol_attn_pool + sol_attn_fwd), on calls in a row with different shapes, head sizes and
inputs, so that no call may see anything an earlier one left in the shared scratch; and on a shape
exactly at the scratch limit.  Collected last so that a failure here cannot hide the result of any
other test."""
import numpy as np
import pytest
import torch

import free_sparse_attention_block_b200 as sol
from free_sparse_attention_block_b200 import inputs
from parity import MAX_ABS, MEAN_ABS, T, check_parity, default_units, gpu_run, to_dev

pytestmark = pytest.mark.gpu


def noalloc_call(q, k, v, beta):
    """One sol_attn_fwd_noalloc call through the C ABI; returns (out float32, density)."""
    lib = sol.load_library()
    B, BH, N, d = q.shape
    Nq = (N + T - 1) // T
    tq, tk, tv = to_dev(q), to_dev(k), to_dev(v)
    out = torch.full_like(tq, float("nan"))
    dens = torch.full((1, BH, Nq), -1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    st = lib.sol_attn_fwd_noalloc(tq.data_ptr(), tk.data_ptr(), tv.data_ptr(), 1, BH, N, d,
                                  float(beta), out.data_ptr(), dens.data_ptr(), stream)
    assert st == 0, sol.STATUS.get(st)
    st, where = sol.sol_attn_read_status(None)      # the scratch's own status words
    assert st == 0, (sol.STATUS.get(st), where)
    return out, dens


def test_noalloc_against_oracle_and_workspace_entry_points_on_calls_in_a_row():
    cases = [(64 * 40 + 16, 3, 1, 0.5, 128), (64 * 17, 2, 2, 1.2, 128), (64 * 21 + 5, 4, 3, 0.5, 64)]
    for N, BH, seed, beta, d in cases:            # (N, heads, seed, beta, head dim)
        q, k, v = inputs.small_workload(N, BH=BH, seed=seed, d=d)
        ref = gpu_run(q, k, v, beta, debug=True)
        out, dens = noalloc_call(q, k, v, beta)
        got = out.float().cpu().numpy()
        assert np.all(np.isfinite(got))
        # same masks as the workspace path (same routing code), so its debug masks apply
        assert np.array_equal(dens.cpu().numpy(), ref["density"])
        err = np.abs(got - ref["out"])
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
        g = dict(ref, out=got, density=dens.cpu().numpy())
        check_parity(q, k, v, beta, g, default_units(BH, (N + T - 1) // T, None))


def test_noalloc_exactly_at_its_scratch_limit():
    """2 heads x 5461 key blocks at d = 128: 10922 pooled rows, 12 B per pooled channel plus the
    1 KB header = exactly SOL_ATTN_NOALLOC_MAX_BYTES.  Sampled tiles against the oracle."""
    N, BH, beta = 64 * 5461, 2, 1.0
    assert 1024 + 12 * BH * 5461 * 128 == sol.NOALLOC_MAX_BYTES      # header + pooled rows
    q, k, v = inputs.small_workload(N, BH=BH, seed=11)
    Nq = (N + T - 1) // T
    units = default_units(BH, Nq, per_head=6, seed=3)
    ref = gpu_run(q, k, v, beta, units=units, with_proxy=False)
    out, dens = noalloc_call(q, k, v, beta)
    assert np.array_equal(dens.cpu().numpy(), ref["density"])
    sel = torch.as_tensor(units, device="cuda")
    got = out.view(BH * Nq, T, 128).index_select(0, sel).float().cpu().numpy()
    g = dict(ref, out_units=got, density=dens.cpu().numpy())
    check_parity(q, k, v, beta, g, units)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    lib = sol.load_library()
    A = 0x10000                       # never dereferenced: the size check comes first
    # 12 heads x 65536 tokens needs 12 * 1024 pooled rows * 1536 B > 16 MiB
    st = lib.sol_attn_fwd_noalloc(A, A, A, 1, 12, 65536, 128, 0.5, A, None, None)
    assert sol.STATUS[st] == "SOL_ERR_SCRATCH_LIMIT"
    # the first row counts past the documented limits (10922 pooled rows at d = 128, 21844 at
    # d = 64): 3 heads x 3641 blocks and 5 heads x 4369 blocks
    for H, nblk, d in [(3, 3641, 128), (5, 4369, 64)]:
        st = lib.sol_attn_fwd_noalloc(A, A, A, 1, H, 64 * nblk, d, 0.5, A, None, None)
        assert sol.STATUS[st] == "SOL_ERR_SCRATCH_LIMIT", (H, nblk, d)
