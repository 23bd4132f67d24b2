"""Per-head beta calibration to a target block density.

The threshold paragraph of "Sol-Attn: Accelerating Video Generation Inference via On-the-Fly
Attention Sparsification" observes that a query's proxy scores over key blocks are close to
normal, so the fraction of blocks at or above mu + beta*sigma is about 1 - Phi(beta), and one
global beta keeps the overall density stable.  Heads still differ, so this helper finds one beta
per head that holds every head at the same measured density (block-count fraction, kept pairs /
(Nq * Nk)).  It starts each head at beta = Phi^-1(1 - target) and corrects it in z-space from the
densities the kernel reports (secant steps on z(beta) = Phi^-1(1 - density(beta))).

The iteration itself is host arithmetic on the densities; every forward pass runs in the CUDA
kernels (sol_attn_fwd_betas).
"""
from __future__ import annotations

from statistics import NormalDist

import numpy as np

_N = NormalDist()
_EPS = 1e-4


def beta_for_density(target: float) -> float:
    """Normal-model beta whose expected kept fraction is `target`."""
    if not 0.0 < target < 1.0:
        raise ValueError("target density must lie strictly between 0 and 1")
    return _N.inv_cdf(1.0 - target)


def _z(density: np.ndarray) -> np.ndarray:
    d = np.clip(np.asarray(density, np.float64), _EPS, 1.0 - _EPS)
    return np.array([_N.inv_cdf(1.0 - x) for x in d.ravel()]).reshape(d.shape)


def calibrate(measure, n_heads: int, target: float, iters: int = 5, tol: float = 0.005):
    """Find per-head betas with measure(betas) ~= target for every head.

    measure: callable taking a float64 array [n_heads] of betas and returning the measured
    densities [n_heads].  Returns (betas, densities, history of (betas, densities)).
    """
    zt = _N.inv_cdf(1.0 - target)
    beta = np.full(n_heads, zt, np.float64)
    rho = np.asarray(measure(beta), np.float64)
    hist = [(beta.copy(), rho.copy())]
    prev_beta, prev_z = None, None
    for _ in range(iters):
        if np.all(np.abs(rho - target) <= tol):
            break
        z = _z(rho)
        step = zt - z                                   # unit-slope step in z-space
        if prev_beta is not None:
            dz = z - prev_z
            db = beta - prev_beta
            ok = np.abs(dz) > 1e-6
            slope = np.where(ok, db / np.where(ok, dz, 1.0), 1.0)
            slope = np.clip(slope, 0.2, 5.0)           # keep the secant sane on plateaus
            step = (zt - z) * slope
        prev_beta, prev_z = beta.copy(), z
        beta = beta + step
        rho = np.asarray(measure(beta), np.float64)
        hist.append((beta.copy(), rho.copy()))
    return beta, rho, hist


def calibrate_betas(q, k, v, target: float, iters: int = 5, tol: float = 0.005, stream=None):
    """Per-head betas for device tensors q, k, v (bf16 [B, H, N, 128]) so that every head keeps
    about `target` of its (query tile, key block) pairs.  Returns (betas float32 [B*H] on the
    device, measured densities numpy [B*H])."""
    import torch

    import free_sparse_attention_block_b200 as sol

    B, H, N, d = q.shape
    nq = (N + sol.TILE - 1) // sol.TILE
    ws = torch.empty(sol.sol_attn_workspace_bytes(B, H, N, d), dtype=torch.uint8, device=q.device)
    out = torch.empty_like(q)
    dens = torch.empty((B, H, nq), dtype=torch.int32, device=q.device)
    sol.sol_attn_pool(k, v, ws, stream)
    bt = torch.empty(B * H, dtype=torch.float32, device=q.device)

    def measure(betas):
        bt.copy_(torch.from_numpy(np.asarray(betas, np.float32)))
        sol.sol_attn_fwd_betas(q, k, v, bt, ws, out, dens, stream)
        return (dens.view(B * H, nq).double().sum(1) / (nq * nq)).cpu().numpy()

    beta, rho, _ = calibrate(measure, B * H, target, iters, tol)
    bt.copy_(torch.from_numpy(beta.astype(np.float32)))
    return bt, rho
