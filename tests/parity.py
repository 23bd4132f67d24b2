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


# ------------------------------------------------------------------ top-k / top-p routing rules

TOPP_MASS_BAND = 1e-9     # float64 mass sums in a different order: decisions this close to p*Z may differ
TOPP_MASS_TOL = 1e-4      # proxy differences (<= 1e-5) move the masses, checked on the oracle's proxy


def gpu_run_rule(q, k, v, rule: str, param, units=None):
    """Pool + forward with a rank rule through the production entry point (sol_attn_fwd_topk /
    sol_attn_fwd_topp) and the debug entry point; both must agree bit for bit."""
    B, H, N, d = q.shape
    Nq = (N + T - 1) // T
    tq, tk, tv = to_dev(q), to_dev(k), to_dev(v)
    ws = torch.zeros(sol.sol_attn_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")
    out = torch.full_like(tq, float("nan"))
    dens = torch.full((B, H, Nq), -1, dtype=torch.int32, device="cuda")
    sol.sol_attn_pool(tk, tv, ws)
    if rule == "topk":
        sol.sol_attn_fwd_topk(tq, tk, tv, int(param), ws, out, dens)
    else:
        sol.sol_attn_fwd_topp(tq, tk, tv, float(param), ws, out, dens)
    st, where = sol.sol_attn_read_status(ws)
    assert st == 0, (sol.STATUS.get(st), where)
    out2 = torch.full_like(tq, float("nan"))
    dens2 = torch.full((B, H, Nq), -1, dtype=torch.int32, device="cuda")
    proxy = torch.full((B, H, Nq, Nq), float("nan"), dtype=torch.float32, device="cuda")
    mask = torch.full((B, H, Nq, Nq), 255, dtype=torch.uint8, device="cuda")
    stats = torch.full((B, H, Nq, 3), float("nan"), dtype=torch.float32, device="cuda")
    st = sol.sol_attn_fwd_debug_route(tq, tk, tv, rule, float(param), ws, out2, dens2, proxy, mask, stats)
    assert st == 0, sol.STATUS.get(st)
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16)), "debug/production outputs differ"
    assert torch.equal(dens, dens2)
    if units is None:
        units = np.arange(B * H * Nq, dtype=np.int64)
    sel = torch.as_tensor(np.asarray(units), device="cuda")
    pick = lambda t: t.reshape(B * H * Nq, *t.shape[3:]).index_select(0, sel).cpu().numpy()
    pad = Nq * T - N
    o = torch.nn.functional.pad(out.view(B * H, N, d), (0, 0, 0, pad), value=float("nan"))
    res = dict(units=units, density=dens.cpu().numpy(), mask=pick(mask), proxy=pick(proxy),
               stats=pick(stats),
               out_units=o.view(B * H * Nq, T, d).index_select(0, sel).float().cpu().numpy())
    return res


def check_rule_parity(q, k, v, rule: str, param, g: dict, report: dict | None = None):
    """Acceptance for a rank rule, per query tile:
      - the GPU proxy row matches the oracle's (as for the threshold rule), mu/sigma too;
      - the GPU mask is exactly the oracle's selection applied to the GPU's own proxy row (top-p:
        a prefix one block longer or shorter is accepted when the mass sum lies within
        TOPP_MASS_BAND of p);
      - against the oracle's own proxy: top-k keeps min(k, Nk) blocks and any disagreement with
        the oracle's mask lies within BAND of the oracle's k-th score; top-p's kept mass reaches
        p and drops below it without the lowest kept block, within TOPP_MASS_TOL;
      - the threshold statistic is the lowest kept GPU score (+inf if none), density = mask sums;
      - outputs match the oracle's attention under the GPU's mask (MAX_ABS / MEAN_ABS)."""
    from oracle import sol_ref_routes as rr
    B, H, N, d = q.shape
    Nk = (N + T - 1) // T
    units = g["units"]
    kbar, vbar = sol_ref.pool(k), sol_ref.pool(v)
    r = rr.route_variant(q, kbar, rule, param, units)
    gm = g["mask"].reshape(-1, Nk)
    gp = g["proxy"].reshape(-1, Nk)
    gs = g["stats"].reshape(-1, 3)
    assert np.all((gm == 0) | (gm == 1))
    np.testing.assert_allclose(gp, r["proxy"], rtol=1e-6, atol=STAT_ATOL)
    np.testing.assert_allclose(gs[:, 0], r["mu"], rtol=0, atol=STAT_ATOL)
    np.testing.assert_allclose(gs[:, 1], r["sigma"], rtol=0, atol=STAT_ATOL)
    cnt = gm.sum(1)
    assert np.array_equal(g["density"].reshape(-1)[units], cnt.astype(np.int32))
    low = np.array([gp[u][gm[u] == 1].min() if cnt[u] else np.inf for u in range(len(units))],
                   np.float32)
    assert np.array_equal(gs[:, 2], low)
    band_rows = 0
    if rule == "topk":
        want = rr.select_topk(gp, int(param))
        assert np.array_equal(gm, want), f"{int((gm != want).sum())} blocks differ on the GPU proxy"
        assert np.all(cnt == min(int(param), Nk))
        om = r["mask"]
        for u in np.nonzero((gm != om).any(1))[0]:
            kk = min(int(param), Nk)
            kth = np.sort(r["proxy"][u].astype(np.float64))[::-1][kk - 1]
            diff = np.nonzero(gm[u] != om[u])[0]
            assert np.all(np.abs(r["proxy"][u, diff] - kth) <= 2 * BAND), (u, diff)
            band_rows += 1
    else:
        p = float(param)
        want, bound = rr.select_topp(gp, p, with_boundary=True)
        for u in range(len(units)):
            if np.array_equal(gm[u], want[u]):
                continue
            # the GPU's prefix may end one block away only for a decision at the band
            lo_b, hi_b = bound[u]
            near = abs(lo_b - p) <= TOPP_MASS_BAND or abs(hi_b - p) <= TOPP_MASS_BAND
            assert near and abs(int(gm[u].sum()) - int(want[u].sum())) == 1, u
            band_rows += 1
        if 0.0 < p < 1.0:
            for u in range(len(units)):
                s = r["proxy"][u].astype(np.float64)
                w = np.exp(s - s.max())
                kept = gm[u] == 1
                frac = w[kept].sum() / w.sum()
                assert frac >= p - TOPP_MASS_TOL, (u, frac)
                lowest = np.argmin(np.where(kept, gp[u], np.inf))
                assert (w[kept].sum() - w[lowest]) / w.sum() < p + TOPP_MASS_TOL, u
    o = sol_ref.attend(q, k, v, kbar, vbar, units, gm)
    errs = []
    for u_i, u in enumerate(units):
        bh, i = divmod(int(u), Nk)
        lo, hi = i * T, min(N, (i + 1) * T)
        got = g["out_units"][u_i, :hi - lo]
        assert np.all(np.isfinite(got))
        errs.append(np.abs(got.astype(np.float64) - o[u_i, :hi - lo]))
    err = np.concatenate(errs)
    max_abs, mean_abs = float(err.max()), float(err.mean())
    if report is not None:
        report.update(max_abs=max_abs, mean_abs=mean_abs, band_rows=band_rows,
                      density=float(gm.mean()), tile_density_std=float(gm.mean(1).std()))
    assert max_abs <= MAX_ABS, max_abs
    assert mean_abs <= MEAN_ABS, mean_abs
    return max_abs, mean_abs
