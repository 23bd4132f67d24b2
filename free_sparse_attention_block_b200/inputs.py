"""Seeded synthetic video-attention inputs (shared by the tests, the smoke check and the bench).

This module only *draws* inputs; it holds none of the attention arithmetic.  Both the CUDA path
and the CPU oracle consume the arrays it returns, so nothing here may depend on either of them.

Each workload stands in for the activations of a video diffusion transformer ("Sol-Attn:
Accelerating Video Generation Inference via On-the-Fly Attention Sparsification", evaluation
paragraphs: Wan2.1-14B, HunyuanVideo, long videos).  No model weights or prompts exist here, so
queries and keys are a smooth spatio-temporal field plus noise, which gives the local, block
structured attention that block-sparse routing exploits:

    F_c(t, y, x) = sum_{s=1..4} sin(2*pi*(f_t t/T + f_h y/H + f_w x/W) + phi)      per channel c
    q = 0.5*F + N(0, 1)      k = 0.5*F + N(0, 1)   (same F, independent noise)      v ~ N(0, 1)

with f_* ~ U[0, f_max] cycles per axis extent and phi ~ U[0, 2*pi).  Tokens are ordered
n = (t*H + y)*W + x.  Values are drawn in float32 and rounded to bfloat16 (round to nearest even);
arrays are returned as uint16 bit patterns, shape [B, H, N, d].

Every (workload, b, h) head has its own numpy PCG64 stream seeded with [seed, b, h], so any head
can be regenerated alone.
"""
from __future__ import annotations

import math
import os
from dataclasses import dataclass, field

import numpy as np

HEAD_DIM = 128
TILE = 64


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    grid: tuple            # (T, H, W) latent grid, T*H*W == N
    betas: tuple           # routing offsets swept for this workload
    seed: int
    f_max: float = 1.5     # highest field frequency, cycles per axis extent
    d: int = HEAD_DIM
    note: str = ""

    @property
    def nq(self) -> int:
        return (self.N + TILE - 1) // TILE

    def dense_flops(self) -> float:
        """4*B*H*N^2*d: QK^T plus PV of dense attention."""
        return 4.0 * self.B * self.H * float(self.N) ** 2 * self.d

    def bytes_qkv(self) -> int:
        return 3 * self.B * self.H * self.N * self.d * 2


NEG_INF = float("-inf")

WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 4096, (4, 32, 32), (NEG_INF, 0.5, 1.0), seed=1),
    "mid": Workload("mid", 1, 12, 16384, (16, 32, 32), (0.5, 1.0, 1.5, 2.0), seed=2),
    "wan": Workload("wan", 1, 40, 75600, (21, 45, 80), (0.5, 1.0, 1.5, 2.0), seed=3,
                    note="Wan2.1-14B-shaped self-attention"),
    "hunyuan": Workload("hunyuan", 1, 24, 118800, (33, 45, 80), (0.5, 1.0, 1.5, 2.0, 2.5), seed=4,
                        note="HunyuanVideo-shaped self-attention"),
    "long": Workload("long", 1, 32, 262144, (64, 64, 64), (1.5, 2.0, 2.5), seed=5, f_max=4.0,
                     note="long-video stress, sharper spatial falloff"),
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns uint16 bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    r = np.right_shift(u, 16)          # in place from here on: one uint32 temporary
    r &= np.uint32(1)
    r += np.uint32(0x7FFF)
    r += u
    r >>= np.uint32(16)
    out = r.astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _field(rng: np.random.Generator, grid, d: int, f_max: float) -> np.ndarray:
    """Sum of 4 random sinusoids per channel over the (T, H, W) grid -> float32 [N, d].

    The phase is separable, angle = a(t) + b(y) + (c(x) + phi), so with A = a + b and
    C = c + phi each term is sin(A) cos(C) + cos(A) sin(C): per channel, the field over
    ((t, y), x) is a product of a [T*H, 8] and an [8, W] matrix (4 terms x 2 products), evaluated
    in float64 as one batched matrix product over the channels.
    """
    T, Hg, Wg = grid
    f = rng.uniform(0.0, f_max, size=(d, 4, 3))
    phi = rng.uniform(0.0, 2.0 * math.pi, size=(d, 4))
    t = np.arange(T, dtype=np.float64) / T
    y = np.arange(Hg, dtype=np.float64) / Hg
    x = np.arange(Wg, dtype=np.float64) / Wg
    ang_a = 2.0 * math.pi * (f[None, None, :, :, 0] * t[:, None, None, None] +
                             f[None, None, :, :, 1] * y[None, :, None, None])         # [T, H, d, 4]
    ang_c = 2.0 * math.pi * f[None, :, :, 2] * x[:, None, None] + phi[None, :, :]   # [W, d, 4]
    left = np.concatenate([np.sin(ang_a), np.cos(ang_a)], axis=3).reshape(T * Hg, d, 8)
    right = np.concatenate([np.cos(ang_c), np.sin(ang_c)], axis=2)                     # [W, d, 8]
    prod = np.matmul(np.ascontiguousarray(left.transpose(1, 0, 2)),
                     np.ascontiguousarray(right.transpose(1, 2, 0)))                   # [d, T*H, W]
    return np.ascontiguousarray(prod.transpose(1, 2, 0), dtype=np.float32).reshape(T * Hg * Wg, d)


def gen_head(seed: int, b: int, h: int, grid, d: int = HEAD_DIM, f_max: float = 1.5,
             n_tokens: int | None = None):
    """One head's (q, k, v) as bf16 bit patterns [N, d].

    ``n_tokens`` truncates the grid sequence (ragged lengths in tests); default is the full grid.
    """
    rng = np.random.Generator(np.random.PCG64([seed, b, h]))
    F = _field(rng, grid, d, f_max)
    n = F.shape[0] if n_tokens is None else n_tokens
    assert n <= F.shape[0]
    F = F[:n]
    F *= np.float32(0.5)                  # exact; 0.5*F + noise below, in float32
    out = []
    for with_field in (True, True, False):   # q, k (field + noise), then v (noise)
        x = rng.standard_normal((n, d), dtype=np.float32)
        if with_field:
            x += F
        out.append(f32_to_bf16_bits(x))
    return tuple(out)


def gen_workload(wl: Workload, heads=None, processes: int | None = None, n_tokens: int | None = None,
                 out=None):
    """All heads of a workload: q, k, v uint16 [B, H, N, d].

    ``heads`` restricts generation to a list of (b, h) pairs (others are left zero).
    ``out`` = (q, k, v): caller arrays of that shape and dtype to fill instead (for example views
    of pinned host buffers); heads not generated are left as they are.
    Heads are generated by a pool of threads (numpy releases the GIL in the random draws, the
    matrix products and the element-wise passes), each writing its own slices of the outputs;
    ``processes`` caps the thread count (default: the usable cores, at most 32).
    """
    n = wl.N if n_tokens is None else n_tokens
    shape = (wl.B, wl.H, n, wl.d)
    if out is None:
        q, k, v = (np.zeros(shape, np.uint16) for _ in range(3))
    else:
        q, k, v = out
        assert all(a.shape == shape and a.dtype == np.uint16 for a in out)
    todo = [(b, h) for b in range(wl.B) for h in range(wl.H)] if heads is None else list(heads)

    def one(bh):
        b, h = bh
        q[b, h], k[b, h], v[b, h] = gen_head(wl.seed, b, h, wl.grid, wl.d, wl.f_max, n)

    if processes is None:
        processes = min(len(todo), len(os.sched_getaffinity(0)), 32) if n * len(todo) > 4_000_000 else 1
    if processes > 1 and len(todo) > 1:
        from concurrent.futures import ThreadPoolExecutor

        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1, user_api="blas"), ThreadPoolExecutor(processes) as ex:
            list(ex.map(one, todo))   # one BLAS thread per head: the heads are the parallelism
    else:
        for bh in todo:
            one(bh)
    return q, k, v


def random_bf16(shape, seed: int, scale: float = 1.0) -> np.ndarray:
    """Plain N(0, scale^2) bf16 bit patterns, for shape and edge-case tests."""
    rng = np.random.Generator(np.random.PCG64([seed, 12345]))
    return f32_to_bf16_bits(scale * rng.standard_normal(shape, dtype=np.float32))


def small_workload(N: int, BH: int = 2, seed: int = 7, grid=None, f_max: float = 1.5,
                   d: int = HEAD_DIM):
    """A small field+noise case with arbitrary (possibly ragged) N, shape [1, BH, N, d]."""
    if grid is None:
        W = 32
        Hg = 16
        T = max(1, -(-N // (W * Hg)))
        grid = (T, Hg, W)
    wl = Workload(f"small{N}", 1, BH, int(np.prod(grid)), tuple(grid), (), seed=seed, f_max=f_max, d=d)
    return gen_workload(wl, n_tokens=N, processes=1)
