"""sol_attn_fwd_sharded through a one-rank NCCL group on one GPU: the sharded entry point (head
range, CUDA forward of the rank's heads, NCCL all-gather of outputs and densities) is checked
against the oracle on every tile (with the GPU's own masks from the debug outputs for near ties)
and must return exactly what the single-GPU forward returns.  The multi-rank gather itself is
covered on CPU with gloo (tests/test_sharded.py)."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import free_sparse_attention_block_b200 as sol
from free_sparse_attention_block_b200 import inputs
from free_sparse_attention_block_b200.sharded import sol_attn_fwd_sharded
from parity import check_parity, default_units, gpu_run

pytestmark = pytest.mark.gpu


def test_one_rank_nccl_group_against_the_oracle():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        H, N = 5, 64 * 7 + 9
        q, k, v = inputs.small_workload(N, BH=H, seed=21)
        dev = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
        tq, tk, tv = dev(q), dev(k), dev(v)
        want_out, want_dens = sol.forward(tq, tk, tv, 0.7)
        got_out, got_dens = sol_attn_fwd_sharded(tq, tk, tv, 0.7, H)
        torch.cuda.synchronize()
        assert torch.equal(got_out.view(torch.int16), want_out.view(torch.int16))
        assert torch.equal(got_dens, want_dens)
        ref = gpu_run(q, k, v, 0.7)           # the GPU's masks and statistics (debug outputs)
        g = dict(ref, out=got_out.float().cpu().numpy(), density=got_dens.cpu().numpy())
        check_parity(q, k, v, 0.7, g, default_units(H, (N + 63) // 64, None))
        side = torch.cuda.Stream()     # the gather must wait for a forward queued on another stream
        got_out, got_dens = sol_attn_fwd_sharded(tq, tk, tv, 0.7, H, stream=side)
        torch.cuda.synchronize()
        assert torch.equal(got_out.view(torch.int16), want_out.view(torch.int16))
        assert torch.equal(got_dens, want_dens)
        with pytest.raises(ValueError):
            sol_attn_fwd_sharded(tq[:, :4], tk[:, :4], tv[:, :4], 0.7, H)   # not this rank's heads
    finally:
        dist.destroy_process_group()
