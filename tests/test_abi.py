"""The C-ABI library loads, exports every entry point include/sol_attn.h declares, and rejects
bad arguments on the host before any CUDA call (no GPU needed)."""
import ctypes as C
import math
import os
import re

import pytest

import free_sparse_attention_block_b200 as sol
from free_sparse_attention_block_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return sol.load_library()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "sol_attn.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sol_attn_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("sol_attn_workspace_bytes", "sol_attn_pool", "sol_attn_fwd",
                     "sol_attn_fwd_debug", "sol_attn_error_string"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_workspace_bytes(lib):
    B, H, N = 1, 12, 16384
    Nk = N // 64
    n = B * H * Nk * 128
    got = sol.sol_attn_workspace_bytes(B, H, N, 128)
    up = lambda x: (x + 255) & ~255

    def layout(BH, Nk, d):
        # 1 KB header; float32 k_bar, v_bar; bf16 k_bar, v_bar; then the partial rows of up to
        # 128 split tile pairs: [pairs][2 halves][128 rows][d + 4] float32
        e = BH * Nk * d
        pooled = up(up(up(up(1024 + 4 * e) + 4 * e) + 2 * e) + 2 * e)
        cap = min(BH * ((Nk + 1) // 2), 128)
        return up(pooled + cap * 2 * 128 * (d + 4) * 4)

    assert got == layout(B * H, Nk, 128) and got % 256 == 0
    assert got >= 1024 + n * (4 + 4 + 2 + 2) + 128 * 2 * 128 * 132 * 4       # 1536 pairs: cap 128
    assert sol.sol_attn_workspace_bytes(1, 1, 100, 128) == layout(1, 2, 128)  # one pair: cap 1
    assert sol.sol_attn_workspace_bytes(1, 1, 100, 96) == 0       # d not 64/128: unsupported
    assert sol.sol_attn_workspace_bytes(1, 1, 100, 256) == 0
    # d = 64: the same layout with 64-channel rows
    assert sol.sol_attn_workspace_bytes(1, 1, 100, 64) == layout(1, 2, 64)
    assert sol.sol_attn_workspace_bytes(2, 3, 64 * 5 + 1, 64) == layout(6, 6, 64)
    assert sol.sol_attn_workspace_bytes(0, 1, 100, 128) == 0
    assert sol.sol_attn_workspace_bytes(1, 1, 524288 + 1, 128) == 0


def test_error_strings(lib):
    for code in range(6):
        assert sol.sol_attn_error_string(code)
    assert "unknown" in sol.sol_attn_error_string(99)


A = 0x10000          # a 256-byte aligned fake device address (never dereferenced)
MIS = 0x10008        # 8-byte aligned only


def fwd(lib, q=A, k=A, v=A, B=1, H=1, N=128, d=128, beta=0.5, ws=A, out=A, dens=None):
    return lib.sol_attn_fwd(q, k, v, B, H, N, d, C.c_float(beta), ws, out, dens, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(q=None), 1), (dict(out=None), 1), (dict(ws=None), 1),
    (dict(N=0), 1), (dict(B=-1), 1), (dict(d=96), 2), (dict(d=256), 2), (dict(N=524288 + 64), 2),
    (dict(beta=math.nan), 1), (dict(k=MIS), 3), (dict(ws=A + 16), 3), (dict(dens=A + 2), 3),
])
def test_fwd_rejects_bad_arguments_on_host(lib, kw, expect):
    assert fwd(lib, **kw) == expect


def test_pool_rejects_bad_arguments_on_host(lib):
    assert lib.sol_attn_pool(None, A, 1, 1, 128, 128, A, None) == 1
    assert lib.sol_attn_pool(A, A, 1, 1, 128, 96, A, None) == 2
    assert lib.sol_attn_pool(A, MIS, 1, 1, 128, 128, A, None) == 3
    assert lib.sol_attn_pool(A, A, 1, 1, 128, 128, A + 128, None) == 3


def test_host_entry_rejects_bad_arguments_on_host(lib):
    f = lib.sol_attn_fwd_host
    assert f(None, A, A, 1, 1, 128, 128, C.c_float(0.5), A, A, A, A, A, None, A, None, None) == 1
    assert f(A, A, A, 1, 1, 128, 128, C.c_float(0.5), A, A, A, A, A, A, A, None, None) == 1
    assert f(A, A, A, 1, 1, 128, 128, C.c_float(math.nan), A, A, A, A, A, None, A, None, None) == 1
    assert f(A, A, A, 1, 1, 128, 128, C.c_float(0.5), MIS, A, A, A, A, None, A, None, None) == 3


def test_rank_rules_reject_bad_parameters_before_launch(lib):
    """Negative or fractional k, NaN p and unknown rules fail on the host (no GPU needed)."""
    f = lib.sol_attn_fwd_topk
    assert f(A, A, A, 1, 1, 128, 128, -1, A, A, None, None) == 1
    assert f(A, A, A, 1, 1, 128, 96, 3, A, A, None, None) == 2
    g = lib.sol_attn_fwd_topp
    assert g(A, A, A, 1, 1, 128, 128, C.c_float(math.nan), A, A, None, None) == 1
    assert g(None, A, A, 1, 1, 128, 128, C.c_float(0.5), A, A, None, None) == 1
    h = lib.sol_attn_fwd_debug_route
    assert h(A, A, A, 1, 1, 128, 128, 3, C.c_float(1.0), A, A, None, None, None, None, None) == 1
    assert h(A, A, A, 1, 1, 128, 128, 1, C.c_float(2.5), A, A, None, None, None, None, None) == 1
    assert h(A, A, A, 1, 1, 128, 128, 1, C.c_float(-1.0), A, A, None, None, None, None, None) == 1
    assert h(A, A, A, 1, 1, 128, 128, 2, C.c_float(math.nan), A, A, None, None, None, None, None) == 1
    assert h(A, A, A, 1, 1, 128, 128, 0, C.c_float(math.nan), A, A, None, None, None, None, None) == 1
    assert h(A, A, A, 1, 1, 128, 128, 2, C.c_float(0.5), A, A, None, MIS, None, None, None) == 3
