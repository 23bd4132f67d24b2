"""The Python binding checks every tensor before its pointer reaches the library (which sees no
sizes, so a short buffer would be written past its end on the GPU).  All checks run before the
device check, so they are exercised here on host tensors without a GPU."""
import pytest
import torch

import free_sparse_attention_block_b200 as sol

B, H, N, d = 1, 2, 200, 128
NQ = (N + 63) // 64


def bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def ok_args():
    q, k, v, out = (bf16(B, H, N, d) for _ in range(4))
    ws = torch.zeros(sol.sol_attn_workspace_bytes(B, H, N, d), dtype=torch.uint8)
    dens = torch.zeros((B, H, NQ), dtype=torch.int32)
    return dict(q=q, k=k, v=v, beta=0.5, workspace=ws, out=out, density_out=dens)


def call(**kw):
    a = ok_args()
    a.update(kw)
    return sol.sol_attn_fwd(a["q"], a["k"], a["v"], a["beta"], a["workspace"], a["out"], a["density_out"])


@pytest.mark.parametrize("kw,exc,msg", [
    (dict(k=bf16(B, H, N + 1, d)), ValueError, "k: expected shape"),
    (dict(v=bf16(B, H, d, N).transpose(2, 3)), ValueError, "v: must be contiguous"),
    (dict(out=torch.zeros((B, H, N, d), dtype=torch.float32)), TypeError, "out: expected torch.bfloat16"),
    (dict(workspace=torch.zeros(100, dtype=torch.uint8)), ValueError, "workspace: needs at least"),
    (dict(workspace=torch.zeros(10 ** 6, dtype=torch.int32)), TypeError, "workspace: expected torch.uint8"),
    (dict(density_out=torch.zeros((B, H, NQ - 1), dtype=torch.int32)), ValueError, "density: needs at least"),
    (dict(density_out=torch.zeros((B, H, NQ), dtype=torch.int64)), TypeError, "density: expected torch.int32"),
    (dict(q=bf16(B, H, N)), ValueError, "[B, H, N, d]"),
    (dict(), ValueError, "must be a CUDA tensor"),          # everything else right, but on the host
])
def test_fwd_refuses_bad_tensors_before_the_library_sees_them(kw, exc, msg):
    with pytest.raises(exc, match=msg.replace("[", r"\[").replace("]", r"\]")):
        call(**kw)


def test_debug_outputs_are_size_checked():
    a = ok_args()
    short = torch.zeros(B * H * NQ * NQ - 1, dtype=torch.float32)
    with pytest.raises(ValueError, match="proxy_out: needs at least"):
        sol.sol_attn_fwd_debug(a["q"], a["k"], a["v"], 0.5, a["workspace"], a["out"], None, short)
    with pytest.raises(ValueError, match="stats_out: needs at least"):
        sol.sol_attn_fwd_debug_route(a["q"], a["k"], a["v"], "topk", 3, a["workspace"], a["out"],
                                     stats_out=torch.zeros(5, dtype=torch.float32))


def test_pool_and_host_entry_are_checked():
    a = ok_args()
    with pytest.raises(ValueError, match="v: expected shape"):
        sol.sol_attn_pool(a["k"], bf16(B, H + 1, N, d), a["workspace"])
    # the host entry wants host inputs and outputs and device buffers
    with pytest.raises(ValueError, match="d_q: must be a CUDA tensor"):
        sol.sol_attn_fwd_host(a["q"], a["k"], a["v"], 0.5, a["q"], a["k"], a["v"], a["workspace"],
                              a["out"], a["out"])
    with pytest.raises(ValueError, match="h_out: expected shape"):
        sol.sol_attn_fwd_host(a["q"], a["k"], a["v"], 0.5, a["q"], a["k"], a["v"], a["workspace"],
                              a["out"], bf16(B, H, N, 64))


def test_raw_pointers_and_absent_buffers_pass_unchecked():
    # integers are the caller's own device pointers, which the binding cannot inspect
    sol._arg("x", 1234, torch.bfloat16, shape=(1,))
    sol._arg("x", None, torch.bfloat16, shape=(1,))
