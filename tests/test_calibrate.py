"""Per-head beta calibration: the z-space secant iteration on a synthetic density model (CPU),
and on the GPU against the kernel's own densities, with the calibrated per-head betas checked
against the oracle head by head."""
import numpy as np
import pytest

from free_sparse_attention_block_b200 import calibrate as cal


def test_normal_model_start():
    assert abs(cal.beta_for_density(0.5)) < 1e-12
    assert abs(cal.beta_for_density(0.1587) - 1.0) < 1e-3


@pytest.mark.parametrize("target", [0.05, 0.2, 0.35])
def test_secant_converges_on_shifted_scaled_normals(target):
    rng = np.random.default_rng(1)
    a = rng.uniform(-0.8, 0.8, 16)        # per-head location of the z-scores
    s = rng.uniform(0.6, 1.6, 16)         # and their spread
    from statistics import NormalDist
    nd = NormalDist()
    measure = lambda b: np.array([1.0 - nd.cdf((bi - ai) / si) for bi, ai, si in zip(b, a, s)])
    beta, rho, hist = cal.calibrate(measure, 16, target, iters=8, tol=1e-3)
    assert np.all(np.abs(rho - target) <= 1e-3), rho
    assert len(hist) <= 9


@pytest.mark.gpu
def test_calibrated_betas_on_gpu_match_oracle_per_head():
    import torch

    import free_sparse_attention_block_b200 as sol
    from free_sparse_attention_block_b200 import inputs
    from parity import T, check_parity, default_units, gpu_run, to_dev

    wl = inputs.WORKLOADS["mid"]
    q, k, v = inputs.gen_workload(wl)
    tq, tk, tv = to_dev(q), to_dev(k), to_dev(v)
    bt, rho = cal.calibrate_betas(tq, tk, tv, target=0.2, iters=6, tol=0.01)
    assert np.all(np.abs(rho - 0.2) <= 0.02), rho
    betas = bt.cpu().numpy()
    assert np.ptp(betas) > 0.0              # the heads did need different betas
    # parity of the per-head entry point: four heads against the oracle at their own beta, with
    # the GPU's own masks for near ties (the head run alone through the debug outputs at that beta)
    B, H, N, d = q.shape
    Nq = wl.nq
    ws = torch.zeros(sol.sol_attn_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(tq)
    dens = torch.empty((B, H, Nq), dtype=torch.int32, device="cuda")
    sol.sol_attn_pool(tk, tv, ws)
    sol.sol_attn_fwd_betas(tq, tk, tv, bt, ws, out, dens)
    torch.cuda.synchronize()
    got = out.view(B * H * Nq, T, d)
    for h in (0, 4, 7, H - 1):
        qh, kh, vh = q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1]
        units = default_units(1, Nq, per_head=12, seed=h)
        ref = gpu_run(qh, kh, vh, float(betas[h]), units=units)
        assert np.array_equal(dens.cpu().numpy()[0, h], ref["density"].reshape(-1))
        sel = torch.as_tensor(h * Nq + units, device="cuda")
        g = dict(ref, out_units=got.index_select(0, sel).float().cpu().numpy())
        check_parity(qh, kh, vh, float(betas[h]), g, units)
