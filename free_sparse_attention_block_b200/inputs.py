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
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    out = ((u + bias) >> 16).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _field(rng: np.random.Generator, grid, d: int, f_max: float) -> np.ndarray:
    """Sum of 4 random sinusoids per channel over the (T, H, W) grid -> float32 [N, d].

    The phase is separable, angle = a(t) + b(y) + c(x) + phi, so each term is evaluated as
    Im(e^{i a} e^{i b} e^{i (c + phi)}) with the small per-axis exponentials broadcast over the grid.
    """
    T, Hg, Wg = grid
    f = rng.uniform(0.0, f_max, size=(d, 4, 3))
    phi = rng.uniform(0.0, 2.0 * math.pi, size=(d, 4))
    t = np.arange(T, dtype=np.float64) / T
    y = np.arange(Hg, dtype=np.float64) / Hg
    x = np.arange(Wg, dtype=np.float64) / Wg
    out = np.zeros((T, Hg, Wg, d), dtype=np.float64)
    for s in range(4):
        ea = np.exp(2j * math.pi * f[:, s, 0][None, :] * t[:, None])                  # [T, d]
        eb = np.exp(2j * math.pi * f[:, s, 1][None, :] * y[:, None])                  # [H, d]
        ec = np.exp(1j * (2.0 * math.pi * f[:, s, 2][None, :] * x[:, None] + phi[:, s][None, :]))  # [W, d]
        eab = ea[:, None, :] * eb[None, :, :]                                          # [T, H, d]
        out += eab.real[:, :, None, :] * ec.imag[None, None, :, :]
        out += eab.imag[:, :, None, :] * ec.real[None, None, :, :]
    return out.reshape(T * Hg * Wg, d).astype(np.float32)


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
    q = 0.5 * F + rng.standard_normal((n, d), dtype=np.float32)
    k = 0.5 * F + rng.standard_normal((n, d), dtype=np.float32)
    v = rng.standard_normal((n, d), dtype=np.float32)
    return f32_to_bf16_bits(q), f32_to_bf16_bits(k), f32_to_bf16_bits(v)


def _gen_head_star(args):
    return gen_head(*args)


def gen_workload(wl: Workload, heads=None, processes: int | None = None, n_tokens: int | None = None):
    """All heads of a workload: q, k, v uint16 [B, H, N, d].

    ``heads`` restricts generation to a list of (b, h) pairs (others are left zero).
    Large workloads are generated in a spawn-started process pool (safe after CUDA init).
    """
    n = wl.N if n_tokens is None else n_tokens
    shape = (wl.B, wl.H, n, wl.d)
    q = np.zeros(shape, np.uint16)
    k = np.zeros(shape, np.uint16)
    v = np.zeros(shape, np.uint16)
    todo = [(b, h) for b in range(wl.B) for h in range(wl.H)] if heads is None else list(heads)
    args = [(wl.seed, b, h, wl.grid, wl.d, wl.f_max, n) for (b, h) in todo]
    if processes is None:
        processes = min(len(todo), os.cpu_count() or 1, 16) if n * len(todo) > 4_000_000 else 1
    if processes > 1:
        import multiprocessing as mp
        with mp.get_context("spawn").Pool(processes) as pool:
            results = pool.map(_gen_head_star, args, chunksize=1)
    else:
        results = [_gen_head_star(a) for a in args]
    for (b, h), (qh, kh, vh) in zip(todo, results):
        q[b, h], k[b, h], v[b, h] = qh, kh, vh
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
