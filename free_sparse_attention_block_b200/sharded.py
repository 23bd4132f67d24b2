"""Head-sharded forward over several GPUs: one process per GPU, torch.distributed for the plumbing.

In "Sol-Attn: Accelerating Video Generation Inference via On-the-Fly Attention Sparsification"
(routing and fused-operator paragraphs) every quantity of a query tile -- its proxy row, mu,
sigma, tau, kept blocks and the pooled correction -- comes from its own head's Q, K and V and
that head's pooled keys and values.  So the heads split into contiguous ranges, one per rank,
and the computation needs no exchange: each rank pools and attends its own heads with the
single-GPU library.  The one collective is an optional all-gather of the outputs and densities,
for callers that want the whole [B, H, N, d] result on every rank (NCCL over NVLink on GPUs);
it moves each rank's B * (h1 - h0) * N * d bf16 output to every other rank.
"""
from __future__ import annotations


def head_range(H: int, rank: int, world: int) -> tuple[int, int]:
    """Heads [h0, h1) of `rank` among `world` ranks: contiguous ranges in rank order whose sizes
    differ by at most one (the first H % world ranks take one more head)."""
    if H < 0 or world < 1 or not 0 <= rank < world:
        raise ValueError(f"head_range: H={H}, rank={rank}, world={world}")
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def gather_heads(local, H: int, group=None):
    """All-gather head shards along dim 1.  `local` is this rank's [B, h1 - h0, ...] slice of an
    H-head tensor (head_range of this rank in `group`); every rank receives the [B, H, ...]
    tensor.  Shards are zero-padded to the largest range for the collective, which needs equal
    sizes."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    h0, h1 = head_range(H, rank, world)
    if local.dim() < 2 or local.shape[1] != h1 - h0:
        raise ValueError(f"rank {rank} holds {tuple(local.shape)}, expected heads [{h0}, {h1}) in dim 1")
    B, rest = local.shape[0], tuple(local.shape[2:])
    hmax = -(-H // world)
    padded = local.new_zeros((B, hmax) + rest)
    padded[:, : h1 - h0] = local
    parts = [torch.empty_like(padded) for _ in range(world)]
    dist.all_gather(parts, padded, group=group)
    out = local.new_empty((B, H) + rest)
    for r, part in enumerate(parts):
        a, b = head_range(H, r, world)
        out[:, a:b] = part[:, : b - a]
    return out


def sol_attn_fwd_sharded(q, k, v, beta: float, H: int, group=None, gather: bool = True, stream=None):
    """Forward of this rank's heads of an H-head call.

    q, k, v: bf16 [B, h1 - h0, N, d] on this rank's GPU, where [h0, h1) = head_range(H, rank,
    world) of `group`.  Pools and attends them with the single-GPU library (which fails loudly if
    its CUDA build is missing); every rank must hold at least one head.  With gather=True the
    outputs and densities of all ranks are all-gathered.  Returns (out, density): [B, H, N, d]
    bf16 and [B, H, Nq] int32 when gathered, else this rank's slices."""
    import torch.distributed as dist

    from . import forward

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    h0, h1 = head_range(H, rank, world)
    if h1 == h0:
        raise ValueError(f"{H} heads over {world} ranks leaves rank {rank} without a head")
    for name, x in (("q", q), ("k", k), ("v", v)):
        if x.dim() != 4 or x.shape[1] != h1 - h0:
            raise ValueError(f"{name} of rank {rank} has shape {tuple(x.shape)}, expected heads [{h0}, {h1})")
    out, dens = forward(q, k, v, beta, stream)
    if not gather:
        return out, dens
    if stream is not None and q.is_cuda:
        # the collective is ordered after the current stream's work, so that stream waits for
        # the forward's
        import torch

        from . import _torch_stream
        torch.cuda.current_stream(q.device).wait_stream(_torch_stream(stream, q.device))
    return gather_heads(out, H, group), gather_heads(dens, H, group)
