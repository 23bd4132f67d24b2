#!/usr/bin/env python
"""Benchmark of the Sol-Attn forward (pool + fused routing/attention) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload long] [--beta 1.5]
    python bench.py --impl reference ...      # the CPU oracle on the host cores

One step = sol_attn_pool + sol_attn_fwd over one batch of the seeded synthetic workload (the
whole hot path).  Inputs are resident in HBM; L2 is flushed (a 256 MiB write) before every timed
step and the step is timed on the device with CUDA events.  Rank 0 prints one JSON line.

Metric: dense-equivalent TFLOP/s = 4*B*H*N^2*d / (time of one call); ms per call in
``ms_per_step``; the fraction of the B200 bf16 tensor peak on the kept (computed) tiles in
``computed_tile_frac`` and, with the correction flops included, in ``roofline``.
With N GPUs every rank runs its own replica (no data-path collective); ``value`` sums the work of
all ranks over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from free_sparse_attention_block_b200 import inputs  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FLUSH_BYTES = 256 << 20

# DRAM bytes (read + write) per head of one launch of the fused kernel, from one ncu capture of a
# launch over the workload's first heads (heads are independent, so traffic scales with them),
# keyed by (workload, head dim, beta); valid only for the kernel source whose sha256 prefix is given.
NCU_TRAFFIC = {
    # full capture of one launch of the whole workload (profiles/sol_fwd_mid_beta0.5.md)
    ("mid", 128, 0.5): {"bytes_per_head": (154629632 + 34969344) / 12, "kernel": "100d3f0f82386635"},
    # two-head slice of the long-video stress shape (profiles/sol_fwd_long_beta1.5.md)
    ("long", 128, 1.5): {"bytes_per_head": (2187119616 + 131701504) / 2, "kernel": "100d3f0f82386635"},
}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def _code_only(src: str) -> str:
    """C++ source without comments and blank lines (so that comment edits keep the hash)."""
    import re
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(line.rstrip() for line in src.splitlines() if line.strip())


def kernel_hash() -> str:
    """Identity of the fused kernel's code (comments ignored): recorded ncu counters apply only
    while it is unchanged."""
    h = hashlib.sha256()
    for name in ("sol_fwd.cu", "sm100.cuh", "internal.h"):
        with open(os.path.join(ROOT, "free_sparse_attention_block_b200", "csrc", name)) as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


# ------------------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML every ~2 ms (read-only)."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, torch_device):
        self.samples, self.reasons, self.ok = [], 0, False
        self.max_mhz = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            uuid = str(torch.cuda.get_device_properties(torch_device).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ------------------------------------------------------------------------------ multi-GPU timing

def max_over_ranks(x: float, device=None) -> float:
    """Slowest rank's value (device-timed milliseconds) when a process group is up, else x."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(dense_flops_per_replica: float, world: int, t_max_ms: float) -> float:
    """Whole-job dense-equivalent TFLOP/s of `world` independent replicas over the slowest rank's
    time (weak scaling: each rank runs the full workload)."""
    return world * dense_flops_per_replica / (t_max_ms * 1e-3) / 1e12


# ------------------------------------------------------------------------------ flops

def block_lengths(N: int) -> np.ndarray:
    Nk = (N + 63) // 64
    n = np.full(Nk, 64, np.int64)
    n[-1] = N - 64 * (Nk - 1)
    return n


def flop_counts(mask: np.ndarray, N: int, d: int = 128):
    """Algorithmic flops of one call from the block mask [BH, Nq, Nk] (uint8):
    kept = 4 d sum_{kept (i,j)} n_i n_j; correction = 4 d sum_{skipped (i,j)} n_i;
    executed = what the 128x64 MMA tiles of the kernel actually run (union of a tile pair's kept
    blocks, plus the correction chunks it needs).
    density = kept blocks / all (tile, block) pairs; density_tokens = the fraction of the N^2
    (query, key) pairs that are computed exactly (a ragged last tile/block weighs n_i n_j)."""
    n = block_lengths(N).astype(np.float64)
    m = mask.astype(bool)
    kept = 4.0 * d * float(np.einsum("bij,i,j->", m, n, n))
    corr = 4.0 * d * float(np.einsum("bij,i->", ~m, n))
    BH, Nq, Nk = m.shape
    if Nq % 2:
        m = np.concatenate([m, np.ones((BH, 1, Nk), bool)], axis=1)
    a, b = m[:, 0::2], m[:, 1::2]
    union = (a | b).sum()
    nchunks = (Nk + 63) // 64
    pad = np.ones((BH, a.shape[1], nchunks * 64 - Nk), bool)
    both = np.concatenate([a & b, pad], axis=2).reshape(BH, a.shape[1], nchunks, 64)
    corr_chunks = (~both.all(axis=3)).sum()
    executed = 4.0 * d * 128 * 64 * float(union + corr_chunks)
    density_tokens = kept / (4.0 * d * BH * float(N) ** 2)
    return dict(kept=kept, corr=corr, executed=executed, density=float(mask.mean()),
                density_tokens=density_tokens)


def mask_flop_counts(mask, N: int, d: int = 128):
    """flop_counts computed with torch on the mask's own device (the full-size masks stay on the
    GPU): mask is a uint8 tensor [BH, Nq, Nk].  Same definitions and results as flop_counts."""
    import torch
    BH, Nq, Nk = mask.shape
    n_last = N - 64 * (Nk - 1)
    n = torch.full((Nq,), 64, dtype=torch.int64, device=mask.device)
    n[-1] = n_last
    cnt = mask.sum(-1, dtype=torch.int64)                                   # kept blocks per tile
    row = 64 * cnt - (64 - n_last) * mask[..., -1].to(torch.int64)       # sum_j kept n_j per tile
    kept = 4.0 * d * float((row * n).sum())
    corr = 4.0 * d * float(((Nk - cnt) * n).sum())
    m = mask.bool()
    if Nq % 2:
        m = torch.cat([m, torch.ones((BH, 1, Nk), dtype=torch.bool, device=mask.device)], dim=1)
    a, b = m[:, 0::2], m[:, 1::2]
    union = int((a | b).sum())
    nchunks = (Nk + 63) // 64
    both = torch.cat([a & b, torch.ones((BH, a.shape[1], nchunks * 64 - Nk), dtype=torch.bool,
                                        device=mask.device)], dim=2)
    corr_chunks = int((~both.view(BH, a.shape[1], nchunks, 64).all(-1)).sum())
    executed = 4.0 * d * 128 * 64 * float(union + corr_chunks)
    return dict(kept=kept, corr=corr, executed=executed, density=float(cnt.sum()) / (BH * Nq * Nk),
                density_tokens=kept / (4.0 * d * BH * float(N) ** 2))


def density_spread(dens: np.ndarray, Nk: int) -> dict:
    """Density statistics of one call from the per-tile kept-block counts [B, H, Nq]: the overall
    block fraction, its spread over query tiles, and its spread over heads (the page contrasts a
    stable overall density with top-p's fluctuating one)."""
    per_tile = dens.reshape(-1, dens.shape[-1]).astype(np.float64) / Nk
    return {"density": float(per_tile.mean()), "tile_density_std": float(per_tile.std()),
            "head_density_std": float(per_tile.mean(1).std())}


def compare_routes(sol, tq, tk, tv, ws, out, dens, flush, stream, beta: float, steps: int):
    """Routing rules at one matched overall density: the threshold rule at ``beta`` sets it;
    per-head betas (calibrated), top-k (k = density * Nk) and top-p (p found by bisection) are
    brought to the same density; each is timed (fwd only, L2 flushed) and its spread reported."""
    import torch
    from free_sparse_attention_block_b200 import calibrate

    B, H, N, d = tq.shape
    Nk = dens.shape[-1]
    runs = {
        "threshold": lambda: sol.sol_attn_fwd(tq, tk, tv, beta, ws, out, dens),
    }

    def measure(fn):
        fn()
        torch.cuda.synchronize()
        return dens.cpu().numpy()

    target = density_spread(measure(runs["threshold"]), Nk)["density"]
    t0 = time.perf_counter()
    betas, _ = calibrate.calibrate_betas(tq, tk, tv, target)
    calib_s = time.perf_counter() - t0
    runs["per_head_beta"] = lambda: sol.sol_attn_fwd_betas(tq, tk, tv, betas, ws, out, dens)
    k_match = max(1, int(round(target * Nk)))
    runs["topk"] = lambda: sol.sol_attn_fwd_topk(tq, tk, tv, k_match, ws, out, dens)
    lo, hi = 0.0, 1.0
    for _ in range(30):
        mid = 0.5 * (lo + hi)
        got = density_spread(measure(lambda: sol.sol_attn_fwd_topp(tq, tk, tv, mid, ws, out, dens)), Nk)
        if got["density"] < target:
            lo = mid
        else:
            hi = mid
    p_match = hi
    runs["topp"] = lambda: sol.sol_attn_fwd_topp(tq, tk, tv, p_match, ws, out, dens)
    params = {"threshold": beta, "per_head_beta": "calibrated", "topk": k_match, "topp": p_match}
    res = []
    for name, fn in runs.items():
        stats = density_spread(measure(fn), Nk)
        ts = []
        for _ in range(max(3, steps)):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            ts.append((a, b))
        torch.cuda.synchronize()
        ms = float(np.mean([a.elapsed_time(b) for a, b in ts]))
        res.append({"rule": name, "param": params[name], "fwd_ms": round(ms, 4)} |
                   {k2: round(v2, 5) for k2, v2 in stats.items()})
    st, where = sol.sol_attn_read_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {sol.STATUS.get(st)} at wait site {where}")
    return {"target_density": round(target, 5), "calibration_s": round(calib_s, 3), "rules": res}


# ------------------------------------------------------------------------------ oracle arm

def oracle_sample(wl, beta: float, q, k, v, ntiles: int, seed: int = 0):
    """Time the CPU oracle (as it stands) on ``ntiles`` query tiles; returns (seconds, dense-eq
    flops of those tiles, description)."""
    from oracle import sol_ref
    rng = np.random.default_rng(seed)
    BH = wl.B * wl.H
    Nq = wl.nq
    # whole heads where possible (each sampled head's K and V are pooled once, as in the full
    # job), distinct, as many as ntiles needs
    nh = min(BH, max(1, -(-ntiles // Nq)))
    heads = sorted(int(h) for h in rng.choice(BH, size=nh, replace=False))
    per = int(math.ceil(ntiles / len(heads)))
    qh = q.reshape(BH, wl.N, wl.d)
    kh = k.reshape(BH, wl.N, wl.d)
    vh = v.reshape(BH, wl.N, wl.d)
    t0 = time.perf_counter()
    done = 0
    for h in heads:
        tiles = np.sort(rng.choice(Nq, size=min(per, Nq), replace=False)).astype(np.int64)
        r = sol_ref.forward(qh[h:h + 1], kh[h:h + 1], vh[h:h + 1], beta, units=tiles)
        assert np.isfinite(r["out"]).all()
        done += tiles.size
    dt = time.perf_counter() - t0
    flops = done * 4.0 * 64 * wl.N * wl.d
    desc = f"{done} query tiles of 64 rows from {len(heads)} heads of '{wl.name}' (pool+route+attend)"
    return dt, flops, desc


def cores_used() -> int:
    n = len(os.sched_getaffinity(0))
    omp = os.environ.get("OMP_NUM_THREADS")
    return min(n, int(omp)) if omp else n


def calibrated_tiles(wl, beta, q, k, v, seconds: float) -> int:
    """Number of query tiles the oracle processes in about ``seconds`` on this host."""
    dt, _, _ = oracle_sample(wl, beta, q, k, v, 16, seed=1234)
    per_tile = max(dt / 16, 1e-4)
    return int(max(4, min(wl.B * wl.H * wl.nq, round(seconds / per_tile))))


def run_reference(args, wl):
    """The oracle arm: the CPU oracle as it stands, on rank 0 only, each step a bounded sample
    (sized so that all steps together take about --ref-seconds)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    q, k, v = inputs.gen_workload(wl)
    tiles = calibrated_tiles(wl, args.beta, q, k, v, args.ref_seconds / max(1, args.steps))
    for _ in range(args.warmup):
        oracle_sample(wl, args.beta, q, k, v, max(2, tiles // 4), seed=99)
    times, flops = [], []
    desc = ""
    for s in range(args.steps):
        dt, fl, desc = oracle_sample(wl, args.beta, q, k, v, tiles, seed=s)
        times.append(dt)
        flops.append(fl)
    value = sum(flops) / sum(times) / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(wl, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores_used(), "kind": "oracle",
                         "sample": f"each step: {desc}"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------ GPU arm

METRIC = "sparse attn fwd ms/call, dense-equiv TFLOP/s, % B200 BF16 tensor peak"
UNIT = "TFLOP/s (dense-equivalent)"


def config_of(wl, args):
    return {"workload": wl.name, "B": wl.B, "H": wl.H, "N": wl.N, "d": wl.d, "grid": list(wl.grid),
            "beta": args.beta, "tile": 64,
            "l2": "flushed before every timed step (256 MiB write)",
            "parallelism": ("single GPU" if args.gpus == 1 else
                            f"head-sharded x{args.gpus}, outputs all-gathered" if args.shard == "heads"
                            else f"replicas x{args.gpus}")}


def timed_fwd(fn, flush, stream, steps: int) -> float:
    """Mean device time (ms) of ``fn`` over ``steps`` calls, L2 flushed before each."""
    import torch
    ts = []
    for _ in range(steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        ts.append((a, b))
    torch.cuda.synchronize()
    return float(np.mean([a.elapsed_time(b) for a, b in ts]))


def beta_point(sol, wl, tq, tk, tv, ws, out, dens, beta, flush, stream, steps, dense):
    """One (workload, beta) point: the kernel's own mask for the flop count, then the timed fwd."""
    import torch
    B, H, N, d = tq.shape
    Nq = wl.nq
    m = torch.empty((B * H, Nq, Nq), dtype=torch.uint8, device=tq.device)
    st = sol.sol_attn_fwd_debug(tq, tk, tv, beta, ws, out, dens, None, m, None)
    if st != 0:
        raise RuntimeError(f"debug forward failed: {sol.STATUS.get(st)}")
    fc = mask_flop_counts(m, N, d)
    del m
    ms = timed_fwd(lambda: sol.sol_attn_fwd(tq, tk, tv, beta, ws, out, dens), flush, stream, steps)
    return {"beta": beta, "density": round(fc["density"], 4),
            "density_tokens": round(fc["density_tokens"], 4), "fwd_ms": round(ms, 4),
            "dense_equiv_tflops": round(dense / (ms * 1e-3) / 1e12, 1),
            "computed_tile_frac": round(fc["kept"] / (ms * 1e-3) / 1e12 / PEAK_BF16, 4),
            "computed_tile_frac_sustained": round(fc["kept"] / (ms * 1e-3) / 1e12 / PEAK_BF16_SUST, 4),
            "roofline_frac": round((fc["kept"] + fc["corr"]) / (ms * 1e-3) / 1e12 / PEAK_BF16, 4)}


def dense_regime(sol, dev, flush, stream, steps: int, d: int):
    """The Wan2.1- and HunyuanVideo-shaped workloads at beta = 0.25 and 0 (block density 0.3 and
    0.4, the regime of the tensor-peak target), each point timed (fwd only, L2 flushed) with its
    own clock record."""
    import torch
    res = []
    for name in ("wan", "hunyuan"):
        wl = dataclasses.replace(inputs.WORKLOADS[name], d=d)
        q, k, v = inputs.gen_workload(wl)
        to_dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
        tq, tk, tv = to_dev(q), to_dev(k), to_dev(v)
        del q, k, v
        B, H, N, _ = tq.shape
        ws = torch.zeros(sol.sol_attn_workspace_bytes(B, H, N, d), dtype=torch.uint8, device=dev)
        out = torch.empty_like(tq)
        dens = torch.empty((B, H, wl.nq), dtype=torch.int32, device=dev)
        sol.sol_attn_pool(tk, tv, ws)
        for beta in (0.25, 0.0):
            for _ in range(2):
                sol.sol_attn_fwd(tq, tk, tv, beta, ws, out, dens)
            sampler = ClockSampler(dev)
            with sampler:
                pt = beta_point(sol, wl, tq, tk, tv, ws, out, dens, beta, flush, stream, steps,
                                wl.dense_flops())
            clk = sampler.summary()
            res.append({"workload": name, **pt, "clocks": {k2: clk.get(k2) for k2 in ("sm_mhz", "reasons")}})
        st, where = sol.sol_attn_read_status(ws)
        if st != 0:
            raise RuntimeError(f"device status {sol.STATUS.get(st)} at wait site {where}")
        del tq, tk, tv, ws, out, dens
        torch.cuda.empty_cache()
    return res


def run_ours(args, wl):
    import torch
    import torch.distributed as dist
    import free_sparse_attention_block_b200 as sol

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    sol.load_library()

    shard = args.shard == "heads"
    t_gen = time.perf_counter()
    if shard:
        # this rank's contiguous head range; the outputs are all-gathered inside every step
        from free_sparse_attention_block_b200.sharded import gather_heads, head_range
        h0, h1 = head_range(wl.H, rank, world)
        if h1 == h0:
            raise SystemExit(f"--shard heads: {wl.H} heads over {world} ranks leaves rank {rank} idle")
        q, k, v = inputs.gen_workload(wl, heads=[(b, h) for b in range(wl.B) for h in range(h0, h1)])
        q, k, v = (np.ascontiguousarray(x[:, h0:h1]) for x in (q, k, v))
        hq, hk, hv = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for x in (q, k, v))
    else:
        # generated straight into pinned host buffers: the end-to-end leg uploads from them
        shape = (wl.B, wl.H, wl.N, wl.d)
        hq, hk, hv = (torch.empty(shape, dtype=torch.int16, pin_memory=True) for _ in range(3))
        q, k, v = (t.numpy().view(np.uint16) for t in (hq, hk, hv))
        inputs.gen_workload(wl, out=(q, k, v))
        hq, hk, hv = (t.view(torch.bfloat16) for t in (hq, hk, hv))
    gen_s = time.perf_counter() - t_gen
    B, H, N, d = q.shape
    Nq = wl.nq
    tq, tk, tv = (t.to(dev) for t in (hq, hk, hv))
    ws = torch.zeros(sol.sol_attn_workspace_bytes(B, H, N, d), dtype=torch.uint8, device=dev)
    out = torch.empty_like(tq)
    dens = torch.empty((B, H, Nq), dtype=torch.int32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    # mask once (outside timing) for the exact algorithmic flop count
    sol.sol_attn_pool(tk, tv, ws)
    mask = torch.empty((B * H, Nq, Nq), dtype=torch.uint8, device=dev)
    st = sol.sol_attn_fwd_debug(tq, tk, tv, args.beta, ws, out, dens, None, mask, None)
    if st != 0:
        raise RuntimeError(f"debug forward failed: {sol.STATUS.get(st)}")
    fc = mask_flop_counts(mask, N, d)
    del mask

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        sol.sol_attn_pool(tk, tv, ws)
        if ev is not None:
            ev[1].record(stream)
        sol.sol_attn_fwd(tq, tk, tv, args.beta, ws, out, dens)
        if ev is not None:
            ev[2].record(stream)
        if shard and world > 1:
            gather_heads(out, wl.H)        # NCCL; the current stream waits for it
            gather_heads(dens, wl.H)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    st, where = sol.sol_attn_read_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {sol.STATUS.get(st)} at wait site {where}")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(dev)
    with sampler:
        for s in range(args.steps):
            flush.zero_()
            step(evs[s])
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    pool_ms = [e[0].elapsed_time(e[1]) for e in evs]
    fwd_ms = [e[1].elapsed_time(e[2]) for e in evs]
    gather_ms = float(np.mean([e[2].elapsed_time(e[3]) for e in evs]))
    step_ms = float(np.mean([e[0].elapsed_time(e[3]) for e in evs]))
    mean_fwd = float(np.mean(fwd_ms))
    mean_pool = float(np.mean(pool_ms))
    st, where = sol.sol_attn_read_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {sol.STATUS.get(st)} at wait site {where}")

    # max over ranks of the device time
    t_max = max_over_ranks(step_ms, dev)
    dense = wl.dense_flops()
    # replicas: every rank runs the whole workload; head-sharded: the ranks split one workload
    value = dense / (t_max * 1e-3) / 1e12 if shard else replica_throughput(dense, world, t_max)

    # ---- e2e through the C ABI on pinned host buffers (copies inside the timed region)
    hout = torch.empty(hq.shape, dtype=torch.bfloat16, pin_memory=True)
    hdens = torch.empty((B, H, Nq), dtype=torch.int32, pin_memory=True)
    e2e_steps = max(3, min(args.steps, 20))
    for _ in range(2):
        sol.sol_attn_fwd_host(hq, hk, hv, args.beta, tq, tk, tv, ws, out, hout, dens, hdens)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        sol.sol_attn_fwd_host(hq, hk, hv, args.beta, tq, tk, tv, ws, out, hout, dens, hdens)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dev)
    e2e_value = dense / (e2e_ms * 1e-3) / 1e12 if shard else replica_throughput(dense, world, e2e_ms)
    assert bool(torch.isfinite(hout[0, 0].float()).all()) and bool(torch.isfinite(hout[-1, -1].float()).all())
    h2d = 3 * B * H * N * d * 2
    d2h = B * H * N * d * 2 + B * H * Nq * 4
    del hout

    # ---- beta sweep (fwd only, same inputs), for the record
    sweep = []
    if args.sweep:
        # the workload's beta sweep, plus 0.25 and 0.0 so that densities of 0.3 and above are covered
        for beta in sorted(set(wl.betas) | {0.0, 0.25}):
            sweep.append(beta_point(sol, wl, tq, tk, tv, ws, out, dens, beta, flush, stream,
                                    max(3, args.steps // 2), dense))

    # ---- routing rules at matched density (threshold, per-head beta, top-k, top-p), for the record
    routes = None
    if args.route_compare:
        routes = compare_routes(sol, tq, tk, tv, ws, out, dens, flush, stream, args.beta,
                                max(3, args.steps // 2))

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    # ---- the density >= 0.3 regime on the Wan2.1 / Hunyuan shapes (rank 0, N = 1 only)
    dense_block = None
    if world == 1 and not args.no_dense_block and wl.name in ("long", "wan", "hunyuan"):
        del tq, tk, tv, out
        torch.cuda.empty_cache()
        dense_block = dense_regime(sol, dev, flush, stream, max(3, args.steps // 5), d)

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N = 1 only)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        nt = calibrated_tiles(wl, args.beta, q, k, v, args.cpu_seconds)
        dt, fl, desc = oracle_sample(wl, args.beta, q, k, v, nt)
        cpu = {"value": fl / dt / 1e12, "unit": UNIT, "cores": cores_used(), "kind": "oracle",
               "sample": desc, "seconds": round(dt, 2)}

    achieved = (fc["kept"] + fc["corr"]) / (mean_fwd * 1e-3) / 1e12
    peak, peak_src = roofline_peak(step_ms * args.steps * 1e-3)
    kh = kernel_hash()
    tr = NCU_TRAFFIC.get((wl.name.split("_")[0], wl.d, args.beta))
    traffic = tr["bytes_per_head"] * B * H if tr and tr["kernel"] == kh else None
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_max, "higher_is_better": True,
        "scaling": "strong" if shard else "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_of(wl, args) | {"seed": wl.seed},
        "fwd_ms": mean_fwd, "pool_ms": mean_pool,
        "gather_ms": gather_ms if shard and world > 1 else None,
        "heads_this_rank": int(H),
        "pool_gbs": (2 * B * H * N * d * 2 + B * H * Nq * d * 12) / (mean_pool * 1e-3) / 1e9,
        "density": fc["density"],
        "density_tokens": fc["density_tokens"],
        "computed_tile_frac": fc["kept"] / (mean_fwd * 1e-3) / 1e12 / PEAK_BF16,
        "computed_tile_frac_sustained": fc["kept"] / (mean_fwd * 1e-3) / 1e12 / PEAK_BF16_SUST,
        "executed_mma_tflops": fc["executed"] / (mean_fwd * 1e-3) / 1e12,
        "union_waste": 1.0 - (fc["kept"] + fc["corr"]) / fc["executed"],
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic, "peak_source": peak_src,
                     "frac_of_burst": achieved / PEAK_BF16, "frac_of_sustained": achieved / PEAK_BF16_SUST,
                     "kernel": "sol_fwd_kernel", "algorithmic_flops_per_launch": fc["kept"] + fc["corr"]},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT, "ms": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "api": "sol_attn_fwd_host (pinned host buffers)"},
        "gpu_launches": 2 * args.steps,
        "clocks": sampler.summary(),
        "workspace_bytes": sol.sol_attn_workspace_bytes(B, H, N, d),
        "kernel_sha": kh,
        "input_gen_s": round(gen_s, 2),
    }
    if dense_block:
        line["density_ge_0.3"] = dense_block
    if sweep:
        line["sweep"] = sweep
    if routes:
        line["routing_compare"] = routes
    print(json.dumps(line), flush=True)


PEAKS, PEAK_SRC = load_peaks()
PEAK_BF16 = float(PEAKS.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"]))
PEAK_BF16_SUST = float(PEAKS.get("bf16_tflops_sustained", PEAKS_FALLBACK["bf16_tflops_sustained"]))


def roofline_peak(timed_s: float):
    """Denominator of the roofline: the measured burst bf16 peak for a kernel timed alone, the
    sustained one (a seconds-long GEMM loop under the power cap) when the timed region itself
    runs for more than a second.  Returns (TFLOP/s, description)."""
    if timed_s > 1.0:
        return PEAK_BF16_SUST, f"bf16_tflops_sustained ({PEAK_SRC}): the timed region runs {timed_s:.1f} s"
    return PEAK_BF16, f"bf16_tflops ({PEAK_SRC}; burst): the timed region runs {timed_s:.2f} s"


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--shard", choices=["none", "heads"], default="none",
                    help="with N > 1: split the workload's heads over the ranks and all-gather the "
                         "outputs (strong scaling) instead of N independent replicas (weak)")
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long", choices=sorted(inputs.WORKLOADS),
                    help="default: the long-video stress shape, the largest single-GPU workload")
    ap.add_argument("--beta", type=float, default=None,
                    help="routing offset (default: the first of the workload's beta sweep)")
    ap.add_argument("--heads", type=int, default=None,
                    help="run only the first this many heads of the workload (small profiling cases)")
    ap.add_argument("--sweep", action="store_true", help="also time fwd over the workload's beta sweep")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU-baseline sample time")
    ap.add_argument("--ref-seconds", type=float, default=90.0, help="target total time of the oracle arm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense-block", action="store_true",
                    help="skip the Wan2.1/Hunyuan timings at beta 0.25 and 0 (density >= 0.3)")
    ap.add_argument("--route-compare", action="store_true",
                    help="also compare the routing rules at matched density (threshold, per-head "
                         "beta, top-k, top-p)")
    ap.add_argument("--head-dim", type=int, choices=[64, 128], default=None,
                    help="generate the workload with this head dimension instead of its own")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    wl = inputs.WORKLOADS[args.workload]
    if args.beta is None:
        args.beta = wl.betas[0]
    if args.head_dim is not None and args.head_dim != wl.d:
        wl = dataclasses.replace(wl, d=args.head_dim, name=f"{wl.name}_d{args.head_dim}")
    if args.heads is not None and args.heads < wl.H:
        wl = dataclasses.replace(wl, H=args.heads, name=f"{wl.name}_h{args.heads}")
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()
