"""The binding's forward on a stream other than the current one (a torch stream or a raw handle)
returns exactly what it returns on the current stream.  Right after each call the test allocates
and fills a buffer of the workspace's size on the current stream: the caching allocator must not
hand out the workspace (freed when the call returns) while the side stream's kernels still use
it."""
import numpy as np
import pytest
import torch

import free_sparse_attention_block_b200 as sol
from free_sparse_attention_block_b200 import inputs

pytestmark = pytest.mark.gpu


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("raw_handle", [False, True])
def test_forward_on_a_side_stream(raw_handle):
    N, BH = 64 * 200 + 7, 4
    q, k, v = inputs.small_workload(N, BH=BH, seed=31)
    tq, tk, tv = dev(q), dev(k), dev(v)
    want_out, want_dens = sol.forward(tq, tk, tv, 0.6)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    nbytes = sol.sol_attn_workspace_bytes(1, BH, N, 128)
    got = []
    for _ in range(4):
        got.append(sol.forward(tq, tk, tv, 0.6, stream=side.cuda_stream if raw_handle else side))
        junk = torch.full((nbytes,), 0x7F, dtype=torch.uint8, device="cuda")
        del junk
    side.synchronize()
    torch.cuda.synchronize()
    for out, dens in got:
        assert torch.equal(out.view(torch.int16), want_out.view(torch.int16))
        assert torch.equal(dens, want_dens)
