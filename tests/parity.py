"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI and compare it
with the CPU oracle on the same seeded inputs.

Acceptance (per query tile compared):
  - block masks identical, except blocks whose oracle proxy lies within BAND of the oracle's tau
    (near ties: counted, and the oracle output is then recomputed with the GPU's decision);
  - mu, sigma within 1e-5 absolute; tau within 1e-5 absolute + 1e-5 relative (large |beta|);
    proxy rows within 1e-5 absolute + 1e-6 relative;
  - kept-block counts equal to the GPU's own mask, and to the oracle's up to near ties;
  - outputs (bf16) against the float64 oracle: max-abs <= 2e-2, mean-abs <= 5e-3.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import free_sparse_attention_block_b200 as sol
from oracle import sol_ref

BAND = 1e-5
MAX_ABS = 2e-2
MEAN_ABS = 5e-3
STAT_ATOL = 1e-5
T = 64


def to_dev(x_u16: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x_u16).view(np.int16)).view(torch.bfloat16).cuda()


def gpu_run(q, k, v, beta: float, debug: bool = True, units=None, with_proxy: bool = True):
    """Pool + forward on the GPU.  With debug=True the debug entry point also returns the proxy
    rows, masks and statistics.  The production entry point is always run too and must give a
    bit-identical output and density.  ``units`` (bh*Nq + i) restricts what is copied back."""
    B, H, N, d = q.shape
    Nq = (N + T - 1) // T
    tq, tk, tv = to_dev(q), to_dev(k), to_dev(v)
    ws = torch.zeros(sol.sol_attn_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")
    out = torch.full_like(tq, float("nan"))
    dens = torch.full((B, H, Nq), -1, dtype=torch.int32, device="cuda")
    sol.sol_attn_pool(tk, tv, ws)
    sol.sol_attn_fwd(tq, tk, tv, beta, ws, out, dens)
    st, where = sol.sol_attn_read_status(ws)
    assert st == 0, (sol.STATUS.get(st), where)
    sel = None if units is None else torch.as_tensor(np.asarray(units), device="cuda")
    pick = (lambda t: t.reshape(B * H * Nq, *t.shape[3:]).index_select(0, sel)) if sel is not None else (lambda t: t)
    kb32 = sol.workspace_views(ws, B, H, N, d)[0]
    res = dict(density=dens.cpu().numpy(), units=units, kbar32=kb32.cpu().numpy())
    if sel is None:
        res["out"] = out.float().cpu().numpy()
    else:
        # rows of the chosen tiles: [U, 64, d] (rows past N padded with NaN)
        pad = Nq * T - N
        o = torch.nn.functional.pad(out.view(B * H, N, d), (0, 0, 0, pad), value=float("nan"))
        res["out_units"] = o.view(B * H * Nq, T, d).index_select(0, sel).float().cpu().numpy()
    if debug:
        out2 = torch.full_like(tq, float("nan"))
        dens2 = torch.full((B, H, Nq), -1, dtype=torch.int32, device="cuda")
        proxy = torch.full((B, H, Nq, Nq), float("nan"), dtype=torch.float32, device="cuda") if with_proxy else None
        mask = torch.full((B, H, Nq, Nq), 255, dtype=torch.uint8, device="cuda")
        stats = torch.full((B, H, Nq, 3), float("nan"), dtype=torch.float32, device="cuda")
        st = sol.sol_attn_fwd_debug(tq, tk, tv, beta, ws, out2, dens2, proxy, mask, stats)
        assert st == 0, sol.STATUS.get(st)
        assert torch.equal(out.view(torch.int16), out2.view(torch.int16)), "debug/production outputs differ"
        assert torch.equal(dens, dens2)
        res.update(mask=pick(mask).cpu().numpy(), stats=pick(stats).cpu().numpy())
        if with_proxy:
            res["proxy"] = pick(proxy).cpu().numpy()
        del proxy, mask, stats, out2
    del tq, tk, tv, out
    return res


def default_units(BH: int, Nq: int, per_head: int | None, seed: int = 0) -> np.ndarray:
    """All tiles, or per head the first, the last, a pair neighbour and random ones."""
    if per_head is None or per_head >= Nq:
        return np.arange(BH * Nq, dtype=np.int64)
    rng = np.random.default_rng(seed)
    units = []
    for bh in range(BH):
        pick = {0, Nq - 1, min(1, Nq - 1), max(0, Nq - 2)}
        while len(pick) < per_head:
            pick.add(int(rng.integers(0, Nq)))
        units += [bh * Nq + i for i in sorted(pick)]
    return np.asarray(units, dtype=np.int64)


def check_parity(q, k, v, beta: float, g: dict, units: np.ndarray, report: dict | None = None):
    B, H, N, d = q.shape
    BH = B * H
    Nq = Nk = (N + T - 1) // T
    kbar, vbar = sol_ref.pool(k), sol_ref.pool(v)
    # pooled keys are bit-identical (same float32 summation order on both sides)
    assert np.array_equal(g["kbar32"].reshape(BH, Nk, d), kbar)
    r = sol_ref.route(q, kbar, beta, units)
    near_total = 0
    sub = g.get("units") is not None
    if "mask" in g:
        gm = g["mask"].reshape(-1, Nk) if sub else g["mask"].reshape(BH * Nq, Nk)[units]
        assert np.all((gm == 0) | (gm == 1))
        gs = g["stats"].reshape(-1, 3) if sub else g["stats"].reshape(BH * Nq, 3)[units]
        tau = r["tau"]
        near = np.abs(r["proxy"].astype(np.float64) - tau[:, None]) <= BAND
        near_total = int(near.sum())
        mism = (gm != r["mask"]) & ~near
        assert not mism.any(), f"{int(mism.sum())} mask mismatches outside the tie band"
        if "proxy" in g:
            gp = g["proxy"].reshape(-1, Nk) if sub else g["proxy"].reshape(BH * Nq, Nk)[units]
            np.testing.assert_allclose(gp, r["proxy"], rtol=1e-6, atol=STAT_ATOL)
        np.testing.assert_allclose(gs[:, 0], r["mu"], rtol=0, atol=STAT_ATOL)
        np.testing.assert_allclose(gs[:, 1], r["sigma"], rtol=0, atol=STAT_ATOL)
        fin = np.isfinite(tau)
        # tau = mu + beta*sigma: sigma agrees to ~1e-6 relative, so large |beta| needs a relative bound
        np.testing.assert_allclose(gs[fin, 2], tau[fin], rtol=1e-5, atol=STAT_ATOL)
        assert np.array_equal(gs[~fin, 2], tau[~fin].astype(np.float32))
        gd = g["density"].reshape(-1)[units]
        assert np.array_equal(gd, gm.sum(1).astype(np.int32))
        assert np.all(np.abs(gd - r["count"]) <= near.sum(1))
        mask_used = gm
    else:
        mask_used = r["mask"]
    o = sol_ref.attend(q, k, v, kbar, vbar, units, mask_used)          # [U, 64, d]
    errs = []
    for u_i, u in enumerate(units):
        bh, i = divmod(int(u), Nq)
        lo, hi = i * T, min(N, (i + 1) * T)
        got = g["out_units"][u_i, :hi - lo] if sub else g["out"].reshape(BH, N, d)[bh, lo:hi]
        assert np.all(np.isfinite(got))
        errs.append(np.abs(got.astype(np.float64) - o[u_i, :hi - lo]))
    err = np.concatenate(errs)
    max_abs, mean_abs = float(err.max()), float(err.mean())
    if report is not None:
        report.update(max_abs=max_abs, mean_abs=mean_abs, near_ties=near_total,
                      density=float(mask_used.mean()))
    assert max_abs <= MAX_ABS, max_abs
    assert mean_abs <= MEAN_ABS, mean_abs
    return max_abs, mean_abs, near_total
