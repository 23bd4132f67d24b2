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
    from oracle import sol_ref
    from parity import BAND, MAX_ABS, MEAN_ABS, T, to_dev

    wl = inputs.WORKLOADS["mid"]
    q, k, v = inputs.gen_workload(wl)
    tq, tk, tv = to_dev(q), to_dev(k), to_dev(v)
    bt, rho = cal.calibrate_betas(tq, tk, tv, target=0.2, iters=6, tol=0.01)
    assert np.all(np.abs(rho - 0.2) <= 0.02), rho
    betas = bt.cpu().numpy()
    assert np.ptp(betas) > 0.0              # the heads did need different betas
    # parity of the per-head entry point: two heads against the oracle at their own beta
    B, H, N, d = q.shape
    Nq = wl.nq
    ws = torch.zeros(sol.sol_attn_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(tq)
    dens = torch.empty((B, H, Nq), dtype=torch.int32, device="cuda")
    sol.sol_attn_pool(tk, tv, ws)
    sol.sol_attn_fwd_betas(tq, tk, tv, bt, ws, out, dens)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy().reshape(B * H, N, d)
    for h in (0, H - 1):
        qh, kh, vh = q[0, h:h + 1], k[0, h:h + 1], v[0, h:h + 1]
        tiles = np.array([0, 1, Nq // 2, Nq - 1], np.int64)
        r = sol_ref.forward(qh, kh, vh, float(betas[h]), units=tiles)
        near = np.abs(r["proxy"].astype(np.float64) - r["tau"][:, None]) <= BAND
        assert np.abs(dens.cpu().numpy()[0, h, tiles] - r["count"]).max() <= near.sum(1).max()
        for ti, i in enumerate(tiles):
            if near[ti].any():          # the GPU may have decided a near tie the other way
                continue
            e = np.abs(got[h, i * T:(i + 1) * T] - r["out"][ti])
            assert e.max() <= MAX_ABS and e.mean() <= MEAN_ABS
