"""sol_attn_fwd_noalloc: the entry point for callers that cannot allocate device memory (a fixed
memory budget, a host allocator that must not be re-entered, a plugin without an allocator).
It keeps the pooled keys/values in the library's built-in scratch instead of a caller workspace.
Checked through the C ABI against the workspace entry points (sol_attn_pool + sol_attn_fwd) on two
calls in a row with different shapes and inputs, so the second call must not see anything the
first one left in the shared scratch.  Collected last so that a failure here cannot hide the
result of any other test."""
import numpy as np
import pytest
import torch

import free_sparse_attention_block_b200 as sol
from free_sparse_attention_block_b200 import inputs
from parity import MAX_ABS, MEAN_ABS, gpu_run, to_dev

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_points_on_two_calls():
    lib = sol.load_library()
    stream = torch.cuda.current_stream().cuda_stream
    cases = [(64 * 40 + 16, 3, 1, 0.5), (64 * 17, 2, 2, 1.2)]      # (N, heads, seed, beta)
    for N, BH, seed, beta in cases:
        q, k, v = inputs.small_workload(N, BH=BH, seed=seed)
        ref = gpu_run(q, k, v, beta, debug=False)
        tq, tk, tv = to_dev(q), to_dev(k), to_dev(v)
        out = torch.full_like(tq, float("nan"))
        Nq = (N + 63) // 64
        dens = torch.full((1, BH, Nq), -1, dtype=torch.int32, device="cuda")
        st = lib.sol_attn_fwd_noalloc(tq.data_ptr(), tk.data_ptr(), tv.data_ptr(), 1, BH, N, 128,
                                      float(beta), out.data_ptr(), dens.data_ptr(), stream)
        assert st == 0, sol.STATUS.get(st)
        torch.cuda.synchronize()
        got = out.float().cpu().numpy()
        assert np.all(np.isfinite(got))
        err = np.abs(got - ref["out"])
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
        assert np.array_equal(dens.cpu().numpy(), ref["density"])


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
