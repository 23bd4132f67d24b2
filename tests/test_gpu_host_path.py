"""sol_attn_fwd_host (host buffers in and out, copies pipelined with the compute by groups of heads)
against the device entry points (sol_attn_pool + sol_attn_fwd), bit for bit."""
import numpy as np
import pytest
import torch

import free_sparse_attention_block_b200 as sol
from free_sparse_attention_block_b200 import inputs

pytestmark = pytest.mark.gpu


def pinned(x_u16):
    return torch.from_numpy(np.ascontiguousarray(x_u16).view(np.int16)).view(torch.bfloat16).pin_memory()


def device_reference(q, k, v, beta):
    B, H, N, d = q.shape
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    tq, tk, tv = dev(q), dev(k), dev(v)
    ws = torch.zeros(sol.sol_attn_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(tq)
    dens = torch.empty((B, H, (N + 63) // 64), dtype=torch.int32, device="cuda")
    sol.sol_attn_pool(tk, tv, ws)
    sol.sol_attn_fwd(tq, tk, tv, beta, ws, out, dens)
    torch.cuda.synchronize()
    return out.cpu(), dens.cpu()


class HostCall:
    """Device buffers for one shape, reused across calls (as a serving loop would)."""

    def __init__(self, B, H, N, d):
        self.shape = (B, H, N, d)
        self.Nq = (N + 63) // 64
        self.dq = torch.empty(self.shape, dtype=torch.bfloat16, device="cuda")
        self.dk = torch.empty_like(self.dq)
        self.dv = torch.empty_like(self.dq)
        self.dout = torch.empty_like(self.dq)
        self.ddens = torch.empty((B, H, self.Nq), dtype=torch.int32, device="cuda")
        self.ws = torch.zeros(sol.sol_attn_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")

    def __call__(self, hq, hk, hv, beta, stream=None, with_density=True):
        B, H, N, d = self.shape
        hout = torch.full(self.shape, float("nan"), dtype=torch.bfloat16).pin_memory()
        hdens = torch.full((B, H, self.Nq), -1, dtype=torch.int32).pin_memory() if with_density else None
        sol.sol_attn_fwd_host(hq, hk, hv, beta, self.dq, self.dk, self.dv, self.ws, self.dout, hout,
                              self.ddens if with_density else None, hdens, stream=stream)
        return hout, hdens


@pytest.mark.parametrize("B,H,N,d", [(1, 1, 1000, 128), (1, 3, 64 * 9 + 16, 128), (2, 7, 4096 + 5, 128),
                                     (1, 12, 4096, 64), (1, 9, 2048, 128), (1, 12, 4096, 128),
                                     (1, 12, 37888, 128)])
def test_host_path_matches_device_path(B, H, N, d):
    """(1, 12, 4096, 128) uploads 37.7 MB, so the host path runs two head groups, and its 384
    work units leave a last wave of 88 of 296 CTAs, so the call splits its last 128 units: each
    group launch must split exactly the call's units among its own.  (1, 12, 37888, 128) uploads
    349 MB with 296 tile pairs per head, which fill their last wave of CTAs on a 148-SM part, so
    the host path runs 11 head groups (the rule that allows more than 8)."""
    q, k, v = inputs.small_workload(N, BH=B * H, seed=N + d, d=d)
    q, k, v = (x.reshape(B, H, N, d) for x in (q, k, v))
    ref_out, ref_dens = device_reference(q, k, v, 0.7)
    call = HostCall(B, H, N, d)
    host = [pinned(x) for x in (q, k, v)]
    hout, hdens = call(*host, 0.7)
    torch.cuda.synchronize()
    assert torch.equal(hout.view(torch.int16), ref_out.view(torch.int16))
    assert torch.equal(hdens, ref_dens)
    st, where = sol.sol_attn_read_status(call.ws)
    assert st == 0, (st, where)


def test_back_to_back_calls_on_reused_buffers_and_a_side_stream():
    """Two calls queued without a synchronisation in between reuse the same device buffers: the
    second call's uploads must wait for the first call's compute."""
    B, H, N, d = 1, 10, 64 * 24 + 3, 128
    qa, ka, va = (x.reshape(B, H, N, d) for x in inputs.small_workload(N, BH=H, seed=1))
    qb, kb, vb = (x.reshape(B, H, N, d) for x in inputs.small_workload(N, BH=H, seed=2))
    ref_a, dens_a = device_reference(qa, ka, va, 0.4)
    ref_b, dens_b = device_reference(qb, kb, vb, 1.1)
    call = HostCall(B, H, N, d)
    side = torch.cuda.Stream()
    # host inputs must outlive the asynchronous copies: keep them until the stream is done
    host_a = [pinned(x) for x in (qa, ka, va)]
    host_b = [pinned(x) for x in (qb, kb, vb)]
    with torch.cuda.stream(side):
        out_a, da = call(*host_a, 0.4, stream=side)
        out_b, db = call(*host_b, 1.1, stream=side)
    side.synchronize()
    del host_a, host_b
    assert torch.equal(out_a.view(torch.int16), ref_a.view(torch.int16))
    assert torch.equal(out_b.view(torch.int16), ref_b.view(torch.int16))
    assert torch.equal(da, dens_a) and torch.equal(db, dens_b)


def test_host_path_without_density():
    B, H, N, d = 1, 4, 3000, 128
    q, k, v = (x.reshape(B, H, N, d) for x in inputs.small_workload(N, BH=H, seed=5))
    ref_out, _ = device_reference(q, k, v, 0.5)
    call = HostCall(B, H, N, d)
    host = [pinned(x) for x in (q, k, v)]
    hout, _ = call(*host, 0.5, with_density=False)
    torch.cuda.synchronize()
    assert torch.equal(hout.view(torch.int16), ref_out.view(torch.int16))
