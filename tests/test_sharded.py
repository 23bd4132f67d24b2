"""Head sharding over ranks (host logic, no GPU): the head ranges, and the all-gather of head
shards over 2- and 3-rank gloo groups.  Each rank computes its heads with the CPU oracle; the
gathered outputs and densities must equal the oracle's single-process forward of all heads,
bit for bit (heads are independent, so sharding changes no arithmetic)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from free_sparse_attention_block_b200.sharded import gather_heads, head_range

N = 64 * 3 + 10
BETA = 0.5


def test_head_range_partitions_contiguously():
    for H in range(0, 20):
        for world in range(1, 9):
            ranges = [head_range(H, r, world) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == H
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [b - a for a, b in ranges]
            assert min(sizes) >= 0 and max(sizes) - min(sizes) <= 1
            assert sizes == sorted(sizes, reverse=True)      # the larger ranges come first
    assert head_range(12, 3, 8) == (6, 8) and head_range(12, 4, 8) == (8, 9)
    for bad in [(-1, 0, 1), (4, 2, 2), (4, -1, 2), (4, 0, 0)]:
        with pytest.raises(ValueError):
            head_range(*bad)


def oracle_heads(q, k, v, h0, h1):
    """Oracle forward of heads [h0, h1): out float64 [1, h1-h0, N, d], counts int32 [1, h1-h0, Nq]."""
    from oracle import sol_ref
    r = sol_ref.forward(q[:, h0:h1], k[:, h0:h1], v[:, h0:h1], BETA)
    hl, d = h1 - h0, q.shape[-1]
    nq = -(-N // 64)
    out = r["out"].reshape(1, hl, nq * 64, d)[:, :, :N]
    return out, r["count"].reshape(1, hl, nq)


def _worker(rank, world, port, H, res):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from free_sparse_attention_block_b200 import inputs
        q, k, v = inputs.small_workload(N, BH=H, seed=11)
        h0, h1 = head_range(H, rank, world)
        out, cnt = oracle_heads(q, k, v, h0, h1)
        g_out = gather_heads(torch.from_numpy(np.ascontiguousarray(out)), H)
        g_cnt = gather_heads(torch.from_numpy(np.ascontiguousarray(cnt)), H)
        # a shard of the wrong size is refused before the collective, so every rank raises and
        # none is left waiting
        try:
            gather_heads(torch.zeros(1, h1 - h0 + 1, 4), H)
            bad = "no error"
        except ValueError:
            bad = "ValueError"
        res[rank] = (g_out.numpy(), g_cnt.numpy(), bad)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,H", [(2, 5), (3, 5)])
def test_gathered_shards_equal_the_single_process_oracle(world, H):
    from free_sparse_attention_block_b200 import inputs
    from oracle import sol_ref
    sol_ref.build()                         # built once here, not concurrently by the ranks
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    res = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_worker, args=(world, port, H, res), nprocs=world, start_method="spawn", join=True)
    q, k, v = inputs.small_workload(N, BH=H, seed=11)
    want_out, want_cnt = oracle_heads(q, k, v, 0, H)
    for r in range(world):
        got_out, got_cnt, bad = res[r]
        assert got_out.shape == want_out.shape and got_cnt.shape == want_cnt.shape
        assert np.array_equal(got_out, want_out)
        assert np.array_equal(got_cnt, want_cnt)
        assert bad == "ValueError"

