"""ctypes wrapper around the C oracle in sol_ref.c.  TEST INFRASTRUCTURE ONLY.

Only tests/, the package smoke check and the benchmark's CPU-baseline leg may import this module.
It builds ``libsolref.so`` next to this file with gcc (-O2 -fopenmp -ffp-contract=off) on first
use.  The arithmetic lives in sol_ref.c; this file only marshals numpy arrays.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "sol_ref.c")
LIB = os.path.join(HERE, "libsolref.so")
TILE = 64

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into oracle/libsolref.so (plain gcc, no fast-math)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-fPIC", "-shared", "-Wall", "-o", tmp, SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = C.CDLL(LIB)
            i64, p = C.c_int64, C.c_void_p
            lib.sol_ref_pool.argtypes = [p, i64, i64, i64, p]
            lib.sol_ref_route.argtypes = [p, p, i64, i64, i64, C.c_float, p, i64, p, p, p, p]
            lib.sol_ref_attend.argtypes = [p, p, p, p, p, i64, i64, i64, p, i64, p, p]
            for f in (lib.sol_ref_pool, lib.sol_ref_route, lib.sol_ref_attend):
                f.restype = C.c_int
            _lib = lib
    return _lib


def _ptr(a):
    return a.ctypes.data_as(C.c_void_p) if a is not None else None


def _bh(x):
    x = np.ascontiguousarray(x, dtype=np.uint16)
    return x.reshape(-1, x.shape[-2], x.shape[-1])


def nblocks(N: int) -> int:
    return (N + TILE - 1) // TILE


def pool(x) -> np.ndarray:
    """Block means of bf16 bit patterns [..., N, d] -> float32 [BH, Nk, d]."""
    x = _bh(x)
    BH, N, d = x.shape
    out = np.empty((BH, nblocks(N), d), np.float32)
    rc = _load().sol_ref_pool(_ptr(x), BH, N, d, _ptr(out))
    if rc:
        raise RuntimeError("sol_ref_pool failed")
    return out


def route(q, kbar, beta: float, units=None):
    """Routing for query tiles ``units`` (bh*Nq + i; default all).

    Returns dict(proxy [U,Nk] f32, mu, sigma, tau [U] f64, mask [U,Nk] u8, count [U] i32, units).
    """
    q = _bh(q)
    BH, N, d = q.shape
    Nk = nblocks(N)
    kbar = np.ascontiguousarray(kbar, dtype=np.float32).reshape(BH, Nk, d)
    units = np.arange(BH * Nk, dtype=np.int64) if units is None else np.ascontiguousarray(units, np.int64)
    U = units.shape[0]
    proxy = np.empty((U, Nk), np.float32)
    stats = np.empty((U, 3), np.float64)
    mask = np.empty((U, Nk), np.uint8)
    count = np.empty((U,), np.int32)
    rc = _load().sol_ref_route(_ptr(q), _ptr(kbar), BH, N, d, C.c_float(beta), _ptr(units), U,
                               _ptr(proxy), _ptr(stats), _ptr(mask), _ptr(count))
    if rc:
        raise RuntimeError("sol_ref_route failed")
    return dict(proxy=proxy, mu=stats[:, 0], sigma=stats[:, 1], tau=stats[:, 2], mask=mask,
                count=count, units=units)


def attend(q, k, v, kbar, vbar, units, mask) -> np.ndarray:
    """Output rows of query tiles ``units`` under ``mask`` [U, Nk] -> float64 [U, 64, d]."""
    q, k, v = _bh(q), _bh(k), _bh(v)
    BH, N, d = q.shape
    Nk = nblocks(N)
    kbar = np.ascontiguousarray(kbar, dtype=np.float32).reshape(BH, Nk, d)
    vbar = np.ascontiguousarray(vbar, dtype=np.float32).reshape(BH, Nk, d)
    units = np.ascontiguousarray(units, np.int64)
    mask = np.ascontiguousarray(mask, np.uint8).reshape(units.shape[0], Nk)
    out = np.zeros((units.shape[0], TILE, d), np.float64)
    rc = _load().sol_ref_attend(_ptr(q), _ptr(k), _ptr(v), _ptr(kbar), _ptr(vbar), BH, N, d,
                                _ptr(units), units.shape[0], _ptr(mask), _ptr(out))
    if rc:
        raise RuntimeError("sol_ref_attend failed")
    return out


def forward(q, k, v, beta: float, units=None, mask_override=None):
    """Whole oracle forward for the chosen query tiles.

    Returns the routing dict plus ``out`` [U, 64, d] float64 (rows past N are zero) and the
    pooled ``kbar``/``vbar``.  ``mask_override`` replaces the oracle's own mask (used to take the
    GPU's decision on near-tie blocks, whose proxy lies within the tie band of tau).
    """
    kbar, vbar = pool(k), pool(v)
    r = route(q, kbar, beta, units)
    m = r["mask"] if mask_override is None else mask_override
    r["out"] = attend(q, k, v, kbar, vbar, r["units"], m)
    r["kbar"], r["vbar"] = kbar, vbar
    return r

