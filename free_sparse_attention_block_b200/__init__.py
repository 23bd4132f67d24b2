"""Sol-Attn block-sparse attention forward for NVIDIA B200 (sm_100a).

Python binding of the C ABI in include/sol_attn.h.  It only marshals arguments: tensors are
passed as device pointers with their sizes, and every step of the computation runs in the CUDA
kernels of ``libsolattn.so``.  There is no CPU or PyTorch fallback; if the library is missing the
first call raises.

    import torch, free_sparse_attention_block_b200 as sol
    out, density = sol.forward(q, k, v, beta=0.5)      # q, k, v: bf16 [B, H, N, d] on cuda, d = 64 or 128

The functions named ``sol_attn_*`` mirror the C entry points one to one.
"""
from __future__ import annotations

import ctypes as C
import os
import threading

__all__ = [
    "SolError", "load_library", "LIB_PATH", "HEAD_DIM", "HEAD_DIMS", "TILE", "STATUS",
    "sol_attn_workspace_bytes", "sol_attn_pool", "sol_attn_fwd", "sol_attn_fwd_debug",
    "sol_attn_read_status", "sol_attn_fwd_host", "sol_attn_error_string", "forward",
    "workspace_views", "sol_attn_fwd_noalloc", "NOALLOC_MAX_BYTES", "sol_attn_fwd_betas",
    "sol_attn_fwd_topk", "sol_attn_fwd_topp", "sol_attn_fwd_debug_route", "ROUTE",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsolattn.so")
HEAD_DIM = 128              # default head dimension; HEAD_DIMS lists every compiled one
HEAD_DIMS = (64, 128)
TILE = 64
STATUS = {0: "SOL_OK", 1: "SOL_ERR_INVALID_ARG", 2: "SOL_ERR_UNSUPPORTED", 3: "SOL_ERR_ALIGNMENT",
          4: "SOL_ERR_CUDA", 5: "SOL_ERR_TIMEOUT", 6: "SOL_ERR_SCRATCH_LIMIT"}
NOALLOC_MAX_BYTES = 16 * 1024 * 1024
ROUTE = {"threshold": 0, "topk": 1, "topp": 2}     # sol_route

_lock = threading.Lock()
_lib = None


class SolError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({sol_attn_error_string(status)})")


def load_library(path: str | None = None):
    """Load libsolattn.so (built by ``python -m free_sparse_attention_block_b200.build``)."""
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise ImportError(f"CUDA library {p} is not built; run "
                              "`python -m free_sparse_attention_block_b200.build`")
        lib = C.CDLL(p)
        vp, i, f = C.c_void_p, C.c_int, C.c_float
        lib.sol_attn_workspace_bytes.argtypes = [i, i, i, i]
        lib.sol_attn_workspace_bytes.restype = C.c_size_t
        lib.sol_attn_pool.argtypes = [vp, vp, i, i, i, i, vp, vp]
        lib.sol_attn_fwd.argtypes = [vp, vp, vp, i, i, i, i, f, vp, vp, vp, vp]
        lib.sol_attn_fwd_debug.argtypes = [vp, vp, vp, i, i, i, i, f, vp, vp, vp, vp, vp, vp, i, i, vp]
        lib.sol_attn_read_status.argtypes = [vp, C.POINTER(C.c_int), vp]
        lib.sol_attn_fwd_host.argtypes = [vp, vp, vp, i, i, i, i, f, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        lib.sol_attn_fwd_noalloc.argtypes = [vp, vp, vp, i, i, i, i, f, vp, vp, vp]
        lib.sol_attn_fwd_betas.argtypes = [vp, vp, vp, i, i, i, i, vp, vp, vp, vp, vp]
        lib.sol_attn_fwd_topk.argtypes = [vp, vp, vp, i, i, i, i, i, vp, vp, vp, vp]
        lib.sol_attn_fwd_topp.argtypes = [vp, vp, vp, i, i, i, i, f, vp, vp, vp, vp]
        lib.sol_attn_fwd_debug_route.argtypes = [vp, vp, vp, i, i, i, i, i, f, vp, vp, vp, vp, vp, vp, vp]
        lib.sol_attn_error_string.argtypes = [i]
        lib.sol_attn_error_string.restype = C.c_char_p
        for name in ("sol_attn_pool", "sol_attn_fwd", "sol_attn_fwd_debug", "sol_attn_read_status",
                     "sol_attn_fwd_host", "sol_attn_fwd_noalloc", "sol_attn_fwd_betas",
                     "sol_attn_fwd_topk", "sol_attn_fwd_topp", "sol_attn_fwd_debug_route"):
            getattr(lib, name).restype = C.c_int
        if path is None:
            _lib = lib
        return lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _shape(t):
    if t.dim() != 4:
        raise ValueError("expected a [B, H, N, d] tensor")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    B, H, N, d = t.shape
    return int(B), int(H), int(N), int(d)


def _arg(name: str, t, dtype, shape=None, numel=None, cuda=True):
    """Checks a tensor argument before its pointer reaches the library, which cannot see sizes:
    dtype, exact shape or minimum element count, contiguity, then (unless cuda is None) the
    device.  None and raw integer pointers pass unchecked (the caller vouches for them)."""
    if t is None or isinstance(t, int):
        return
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if numel is not None and t.numel() < numel:
        raise ValueError(f"{name}: needs at least {numel} elements, has {t.numel()}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if cuda is not None and t.is_cuda != cuda:
        raise ValueError(f"{name}: must be a {'CUDA' if cuda else 'host'} tensor")


def _args(q, tensors: dict, workspace=None, density=None, host: dict | None = None,
          host_density=None, debug: dict | None = None):
    """Validates one call's tensors against q's [B, H, N, d]: every shape, dtype and size first,
    then every device; returns (B, H, N, d)."""
    import torch
    B, H, N, d = _shape(q)
    shp = (B, H, N, d)
    Nq = (N + TILE - 1) // TILE
    checks = [(name, t, torch.bfloat16, shp, None, True) for name, t in tensors.items()]
    checks += [(name, t, torch.bfloat16, shp, None, False) for name, t in (host or {}).items()]
    need = sol_attn_workspace_bytes(B, H, N, d)
    if need:                     # 0: an unsupported shape, which the library itself reports
        checks.append(("workspace", workspace, torch.uint8, None, need, True))
    checks.append(("density", density, torch.int32, None, B * H * Nq, True))
    checks.append(("host density", host_density, torch.int32, None, B * H * Nq, False))
    if debug:
        checks.append(("proxy_out", debug.get("proxy"), torch.float32, None, B * H * Nq * Nq, True))
        checks.append(("mask_out", debug.get("mask"), torch.uint8, None, B * H * Nq * Nq, True))
        checks.append(("stats_out", debug.get("stats"), torch.float32, None, B * H * Nq * 3, True))
    for name, t, dtype, shape, numel, _ in checks:
        _arg(name, t, dtype, shape=shape, numel=numel, cuda=None)
    for name, t, dtype, shape, numel, cuda in checks:
        _arg(name, t, dtype, shape=shape, numel=numel, cuda=cuda)
    return shp


def _check(status: int, where: str):
    if status != 0:
        raise SolError(status, where)


def sol_attn_error_string(status: int) -> str:
    return load_library().sol_attn_error_string(int(status)).decode()


def sol_attn_workspace_bytes(B: int, H: int, N: int, d: int = HEAD_DIM) -> int:
    return int(load_library().sol_attn_workspace_bytes(B, H, N, d))


def sol_attn_pool(k, v, workspace, stream=None, check: bool = True) -> int:
    B, H, N, d = _args(k, {"k": k, "v": v}, workspace)
    st = load_library().sol_attn_pool(_ptr(k), _ptr(v), B, H, N, d, _ptr(workspace), _stream(stream))
    if check:
        _check(st, "sol_attn_pool")
    return st


def sol_attn_fwd(q, k, v, beta: float, workspace, out, density_out=None, stream=None,
                 check: bool = True) -> int:
    B, H, N, d = _args(q, {"q": q, "k": k, "v": v, "out": out}, workspace, density_out)
    st = load_library().sol_attn_fwd(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, float(beta),
                                     _ptr(workspace), _ptr(out), _ptr(density_out), _stream(stream))
    if check:
        _check(st, "sol_attn_fwd")
    return st


def sol_attn_fwd_betas(q, k, v, beta_per_head, workspace, out, density_out=None, stream=None,
                       check: bool = True) -> int:
    """sol_attn_fwd with one beta per head: beta_per_head is a float32 device tensor of B*H."""
    B, H, N, d = _args(q, {"q": q, "k": k, "v": v, "out": out}, workspace, density_out)
    if beta_per_head.numel() != B * H:
        raise ValueError("beta_per_head must hold B*H values")
    import torch
    _arg("beta_per_head", beta_per_head, torch.float32, numel=B * H)
    st = load_library().sol_attn_fwd_betas(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, _ptr(beta_per_head),
                                           _ptr(workspace), _ptr(out), _ptr(density_out),
                                           _stream(stream))
    if check:
        _check(st, "sol_attn_fwd_betas")
    return st


def sol_attn_fwd_topk(q, k, v, k_blocks: int, workspace, out, density_out=None, stream=None,
                      check: bool = True) -> int:
    """Forward with the top-k rule: the k_blocks highest-scoring blocks per query tile."""
    B, H, N, d = _args(q, {"q": q, "k": k, "v": v, "out": out}, workspace, density_out)
    st = load_library().sol_attn_fwd_topk(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, int(k_blocks),
                                          _ptr(workspace), _ptr(out), _ptr(density_out),
                                          _stream(stream))
    if check:
        _check(st, "sol_attn_fwd_topk")
    return st


def sol_attn_fwd_topp(q, k, v, p: float, workspace, out, density_out=None, stream=None,
                      check: bool = True) -> int:
    """Forward with the top-p rule: the shortest highest-first prefix of blocks whose softmax
    probability over the proxy row reaches p."""
    B, H, N, d = _args(q, {"q": q, "k": k, "v": v, "out": out}, workspace, density_out)
    st = load_library().sol_attn_fwd_topp(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, float(p),
                                          _ptr(workspace), _ptr(out), _ptr(density_out),
                                          _stream(stream))
    if check:
        _check(st, "sol_attn_fwd_topp")
    return st


def sol_attn_fwd_debug_route(q, k, v, route, param: float, workspace, out, density_out=None,
                             proxy_out=None, mask_out=None, stats_out=None, stream=None) -> int:
    """Debug forward for any rule (``route``: a ROUTE name or code).  Returns the status code."""
    B, H, N, d = _args(q, {"q": q, "k": k, "v": v, "out": out}, workspace, density_out,
                       debug={"proxy": proxy_out, "mask": mask_out, "stats": stats_out})
    code = ROUTE[route] if isinstance(route, str) else int(route)
    return load_library().sol_attn_fwd_debug_route(
        _ptr(q), _ptr(k), _ptr(v), B, H, N, d, code, float(param), _ptr(workspace), _ptr(out),
        _ptr(density_out), _ptr(proxy_out), _ptr(mask_out), _ptr(stats_out), _stream(stream))


def sol_attn_fwd_debug(q, k, v, beta: float, workspace, out, density_out=None, proxy_out=None,
                       mask_out=None, stats_out=None, fault_flags: int = 0, timeout_ms: int = 0,
                       stream=None) -> int:
    """Returns the status code (it is not raised: tests inspect SOL_ERR_TIMEOUT)."""
    B, H, N, d = _args(q, {"q": q, "k": k, "v": v, "out": out}, workspace, density_out,
                       debug={"proxy": proxy_out, "mask": mask_out, "stats": stats_out})
    return load_library().sol_attn_fwd_debug(
        _ptr(q), _ptr(k), _ptr(v), B, H, N, d, float(beta), _ptr(workspace), _ptr(out),
        _ptr(density_out), _ptr(proxy_out), _ptr(mask_out), _ptr(stats_out), int(fault_flags),
        int(timeout_ms), _stream(stream))


def sol_attn_read_status(workspace, stream=None):
    """Synchronise the stream, read and clear the device status words: (status code, wait site).
    workspace None reads the status of sol_attn_fwd_noalloc's built-in scratch on this device."""
    where = C.c_int(0)
    st = load_library().sol_attn_read_status(_ptr(workspace), C.byref(where), _stream(stream))
    return st, where.value


def sol_attn_fwd_host(h_q, h_k, h_v, beta: float, d_q, d_k, d_v, workspace, d_out, h_out,
                      d_density=None, h_density=None, stream=None, check: bool = True) -> int:
    B, H, N, d = _args(d_q, {"d_q": d_q, "d_k": d_k, "d_v": d_v, "d_out": d_out}, workspace, d_density,
                       host={"h_q": h_q, "h_k": h_k, "h_v": h_v, "h_out": h_out}, host_density=h_density)
    st = load_library().sol_attn_fwd_host(
        _ptr(h_q), _ptr(h_k), _ptr(h_v), B, H, N, d, float(beta), _ptr(d_q), _ptr(d_k), _ptr(d_v),
        _ptr(workspace), _ptr(d_out), _ptr(d_density), _ptr(h_out), _ptr(h_density), _stream(stream))
    if check:
        _check(st, "sol_attn_fwd_host")
    return st


def sol_attn_fwd_noalloc(q, k, v, beta: float, out, density_out=None, stream=None,
                         check: bool = True) -> int:
    """Pool + forward without a caller workspace: the library's built-in scratch (at most
    NOALLOC_MAX_BYTES) holds the pooled keys/values.  For callers that cannot allocate device
    memory.  Calls that overlap on the GPU share that scratch and race; serialise them."""
    B, H, N, d = _args(q, {"q": q, "k": k, "v": v, "out": out}, density=density_out)
    st = load_library().sol_attn_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, float(beta),
                                             _ptr(out), _ptr(density_out), _stream(stream))
    if check:
        _check(st, "sol_attn_fwd_noalloc")
    return st


def workspace_views(workspace, B: int, H: int, N: int, d: int = HEAD_DIM):
    """Views of the pooled arrays inside a workspace tensor (uint8, device): (kbar32, vbar32,
    kbar16, vbar16) shaped [B, H, Nk, d]; the layout mirrors the C library's."""
    import torch
    Nk = (N + TILE - 1) // TILE
    n = B * H * Nk * d
    up = lambda x: (x + 255) & ~255
    o_k32 = 1024                       # after the header (status words, split counters)
    o_v32 = up(o_k32 + 4 * n)
    o_k16 = up(o_v32 + 4 * n)
    o_v16 = up(o_k16 + 2 * n)
    shp = (B, H, Nk, d)
    k32 = workspace[o_k32:o_k32 + 4 * n].view(torch.float32).view(shp)
    v32 = workspace[o_v32:o_v32 + 4 * n].view(torch.float32).view(shp)
    k16 = workspace[o_k16:o_k16 + 2 * n].view(torch.bfloat16).view(shp)
    v16 = workspace[o_v16:o_v16 + 2 * n].view(torch.bfloat16).view(shp)
    return k32, v32, k16, v16


def _torch_stream(stream, device):
    """`stream` (a torch stream or a raw cudaStream_t handle) as a torch stream object."""
    import torch
    if isinstance(stream, torch.cuda.Stream):
        return stream
    return torch.cuda.ExternalStream(int(stream), device=device)


def forward(q, k, v, beta: float, stream=None):
    """Pool + fused forward on device tensors.  Allocates the workspace, output and density with
    torch (the library itself allocates nothing).  Returns (out bf16 [B,H,N,d], density int32
    [B,H,Nq]).  With a `stream` other than the current one, the kernels run on it after the work
    already queued on the current stream; the results are ready when that stream reaches them
    (the caller synchronises before using them elsewhere), and the caching allocator keeps the
    workspace, freed on return, until the stream's kernels are done."""
    import torch
    B, H, N, d = _shape(q)
    ws = torch.empty(sol_attn_workspace_bytes(B, H, N, d), dtype=torch.uint8, device=q.device)
    out = torch.empty_like(q)
    dens = torch.empty((B, H, (N + TILE - 1) // TILE), dtype=torch.int32, device=q.device)
    if stream is not None:
        s = _torch_stream(stream, q.device)
        if s != torch.cuda.current_stream(q.device):
            s.wait_stream(torch.cuda.current_stream(q.device))
            for t in (ws, out, dens):
                t.record_stream(s)
    sol_attn_pool(k, v, ws, stream)
    sol_attn_fwd(q, k, v, beta, ws, out, dens, stream)
    return out, dens
