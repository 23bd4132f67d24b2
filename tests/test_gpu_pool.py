"""sol_attn_pool against the oracle's block means: bit-identical float32 (same summation order),
and the bf16 copies are the round-to-nearest-even of the float32 values."""
import numpy as np
import pytest
import torch

import free_sparse_attention_block_b200 as sol
from free_sparse_attention_block_b200 import inputs
from oracle import sol_ref
from parity import to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,N,d", [(1, 2, 4096, 128), (2, 3, 64 * 9 + 16, 128), (1, 1, 1, 128),
                                     (1, 2, 63, 128), (1, 4, 1000, 128), (1, 2, 4096, 64),
                                     (2, 3, 64 * 9 + 16, 64), (1, 1, 1, 64), (1, 3, 1000, 64)])
def test_pool_bit_exact(B, H, N, d):
    k = inputs.random_bf16((B, H, N, d), seed=N + 1, scale=3.0)
    v = inputs.random_bf16((B, H, N, d), seed=N + 2)
    ws = torch.zeros(sol.sol_attn_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")
    sol.sol_attn_pool(to_dev(k), to_dev(v), ws)
    torch.cuda.synchronize()
    k32, v32, k16, v16 = (t.cpu() for t in sol.workspace_views(ws, B, H, N, d))
    Nk = (N + 63) // 64
    rk, rv = sol_ref.pool(k).reshape(B, H, Nk, d), sol_ref.pool(v).reshape(B, H, Nk, d)
    assert np.array_equal(k32.numpy(), rk)
    assert np.array_equal(v32.numpy(), rv)
    assert np.array_equal(k16.view(torch.int16).numpy().view(np.uint16), inputs.f32_to_bf16_bits(rk))
    assert np.array_equal(v16.view(torch.int16).numpy().view(np.uint16), inputs.f32_to_bf16_bits(rv))


def test_pool_full_wan_shape_sampled():
    """Wan2.1-shaped K/V (40 heads x 75600 tokens, last block 16 tokens), sampled heads."""
    wl = inputs.WORKLOADS["wan"]
    heads = [(0, 0), (0, 17), (0, 39)]
    q, k, v = inputs.gen_workload(wl, heads=heads)
    ws = torch.zeros(sol.sol_attn_workspace_bytes(wl.B, wl.H, wl.N, 128), dtype=torch.uint8, device="cuda")
    sol.sol_attn_pool(to_dev(k), to_dev(v), ws)
    torch.cuda.synchronize()
    k32, v32, _, _ = sol.workspace_views(ws, wl.B, wl.H, wl.N)
    for b, h in heads:
        assert np.array_equal(k32[b, h].cpu().numpy(), sol_ref.pool(k[b, h][None])[0])
        assert np.array_equal(v32[b, h].cpu().numpy(), sol_ref.pool(v[b, h][None])[0])
