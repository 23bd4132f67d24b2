"""Host-side logic of bench.py (no GPU): the flop accounting from a block mask, and the multi-GPU
replica timing (slowest rank over a 2-rank gloo process group)."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def test_flop_counts_hand_computed():
    # one head, N = 64*3 + 16 -> blocks of 64, 64, 64, 16; 4 query tiles (last one 16 rows)
    N = 208
    mask = np.zeros((1, 4, 4), np.uint8)
    mask[0, 0, 0] = 1                       # tile 0 keeps block 0
    mask[0, 3, 3] = 1                       # the 16-row tile keeps the 16-token block
    mask[0, 1, :] = 1                       # tile 1 keeps everything
    fc = bench.flop_counts(mask, N, d=128)
    n = np.array([64, 64, 64, 16], float)
    kept = 4 * 128 * (64 * 64 + 16 * 16 + 64 * n.sum())
    corr = 4 * 128 * (64 * 3 + 16 * 3 + 64 * 4)   # skipped pairs: tile0 3, tile3 3, tile2 4
    assert fc["kept"] == kept and fc["corr"] == corr
    assert fc["density"] == mask.mean()
    # tile pairs (0,1) and (2,3): unions of 4 and 1 kept blocks; one correction chunk each
    # (tile 0 and tile 2 skip blocks) -> 7 MMA iterations of 128 x 64 keys
    assert fc["executed"] == 4 * 128 * 128 * 64 * (4 + 1 + 2)
    # token-weighted density: computed (query, key) pairs over N^2
    pairs = 64 * 64 + 16 * 16 + 64 * 208
    assert abs(fc["density_tokens"] - pairs / 208 ** 2) < 1e-15
    # d scales every flop count but no density
    fc64 = bench.flop_counts(mask, N, d=64)
    assert fc64["kept"] == kept / 2 and fc64["density_tokens"] == fc["density_tokens"]


def test_replica_throughput():
    assert bench.replica_throughput(1e12, 1, 1.0) == 1000.0
    assert bench.replica_throughput(1e12, 4, 2.0) == 2000.0


def _worker(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out[rank] = bench.max_over_ranks(times[rank], "cpu")
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    times = [1.25, 3.5]
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_worker, args=(2, port, times, out), nprocs=2, start_method="spawn", join=True)
    assert out[0] == out[1] == 3.5
    assert bench.max_over_ranks(2.0) == 2.0        # no process group: unchanged


def test_density_spread_hand_computed():
    # 2 heads x 3 tiles over Nk = 4 blocks: head 0 keeps 1,2,3 blocks, head 1 keeps 2,2,2
    dens = np.array([[[1, 2, 3], [2, 2, 2]]], np.int32)
    s = bench.density_spread(dens, 4)
    tiles = np.array([1, 2, 3, 2, 2, 2]) / 4
    assert abs(s["density"] - 0.5) < 1e-15
    assert abs(s["tile_density_std"] - tiles.std()) < 1e-15
    assert s["head_density_std"] == 0.0          # both heads average 0.5


def test_mask_flop_counts_matches_flop_counts():
    """The torch form used on full-size device masks equals the numpy definition above."""
    rng = np.random.default_rng(3)
    for N, BH in [(208, 1), (64 * 9, 2), (64 * 70 + 5, 3), (1, 1)]:
        Nk = (N + 63) // 64
        for p in (0.0, 0.3, 1.0):
            mask = (rng.random((BH, Nk, Nk)) < p).astype(np.uint8)
            a = bench.flop_counts(mask, N, d=128)
            b = bench.mask_flop_counts(torch.from_numpy(mask), N, d=128)
            for key in ("kept", "corr", "executed"):
                assert a[key] == b[key], (N, p, key)
            assert abs(a["density"] - b["density"]) < 1e-15
            assert abs(a["density_tokens"] - b["density_tokens"]) < 1e-15


def test_roofline_peak_follows_the_timed_region_length():
    burst, src = bench.roofline_peak(0.05)            # e.g. 20 steps of 2.5 ms
    assert burst == bench.PEAK_BF16 and "burst" in src
    sust, src = bench.roofline_peak(3.2)              # e.g. 30 steps of 107 ms
    assert sust == bench.PEAK_BF16_SUST and "sustained" in src
    assert sust < burst
