"""In-context Sparse Attention (ISA) forward pass for NVIDIA B200 (sm_100a).

Python binding of the C-ABI library ``libisa.so`` (declared in
``include/isa.h``). The binding only marshals arguments: every step of the
pass runs in the library's CUDA kernels. PyTorch provides device memory and
streams. There is no CPU fallback; if the library is missing this module
raises on first use.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

__all__ = [
    "IsaError",
    "ISA_BF16",
    "ISA_F32",
    "lib",
    "lib_path",
    "plan",
    "plan_ns",
    "workspace_bytes",
    "launch_count",
    "forward",
    "forward_into",
    "forward_host",
    "forward_varlen",
    "varlen_workspace_bytes",
    "forward_train",
    "backward",
    "select_context_noalloc",
    "select_context_noalloc_status",
    "device_status",
    "debug_pooled",
    "selftest_wait_timeout",
    "set_stage_events",
    "STAGES",
    "last_error",
    "EXPORTS",
]

ISA_BF16 = 0
ISA_F32 = 1

ERROR_NAMES = {
    0: "ISA_OK",
    -1: "ISA_ERR_ARG",
    -2: "ISA_ERR_SHAPE",
    -3: "ISA_ERR_UNSUPPORTED",
    -4: "ISA_ERR_WORKSPACE",
    -5: "ISA_ERR_CUDA",
    -6: "ISA_ERR_TIMEOUT",
}

# Every function declared in include/isa.h.
EXPORTS = (
    "isa_plan",
    "isa_workspace_bytes",
    "isa_forward_ex",
    "isa_forward",
    "isa_forward_host",
    "isa_device_status",
    "isa_debug_pooled",
    "isa_launch_count",
    "isa_selftest_wait_timeout",
    "isa_selftest_exp2",
    "isa_set_stage_events",
    "isa_select_context_noalloc",
    "isa_select_context_noalloc_status",
    "isa_forward_host_ns",
    "isa_workspace_bytes_varlen",
    "isa_forward_varlen",
    "isa_forward_train",
    "isa_backward_workspace_bytes",
    "isa_backward",
    "isa_plan_ns",
    "isa_workspace_bytes_ns",
    "isa_forward_ns",
    "isa_launch_count_ns",
    "isa_last_error",
)

_HERE = os.path.dirname(os.path.abspath(__file__))


class IsaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{ERROR_NAMES.get(code, code)}: {msg}")
        self.code = code


def lib_path() -> str:
    return os.path.join(_HERE, "libisa.so")


_LIB = None


def lib() -> ctypes.CDLL:
    """Load libisa.so (built in-tree by ``python -m block_sparse_attention_isa_b200.build``)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = os.environ.get("ISA_LIBRARY_PATH") or lib_path()
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m block_sparse_attention_isa_b200.build`")
    L = ctypes.CDLL(path)
    c_int, c_float, c_size, vp = ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p
    i32p = ctypes.POINTER(ctypes.c_int32)
    fp = ctypes.POINTER(ctypes.c_float)
    L.isa_plan.argtypes = [c_int] * 6 + [c_float, c_float, i32p, i32p, i32p]
    L.isa_plan.restype = c_int
    L.isa_workspace_bytes.argtypes = [c_int] * 6 + [c_float, c_int]
    L.isa_workspace_bytes.restype = c_size
    L.isa_forward_ex.argtypes = [vp, vp, vp] + [c_int] * 6 + [c_float, c_float, c_int, vp, vp, vp, vp, c_size, vp]
    L.isa_forward_ex.restype = c_int
    L.isa_forward.argtypes = [vp, vp, vp] + [c_int] * 6 + [c_float, c_float, vp, vp, vp]
    L.isa_forward.restype = c_int
    L.isa_forward_host.argtypes = [vp, vp, vp] + [c_int] * 6 + [c_float, c_float, c_int, vp, vp, vp]
    L.isa_forward_host.restype = c_int
    L.isa_device_status.argtypes = [vp, vp]
    L.isa_device_status.restype = c_int
    L.isa_debug_pooled.argtypes = [c_int] * 6 + [c_float, c_int, vp, vp, vp, vp, vp, vp, vp]
    L.isa_debug_pooled.restype = c_int
    L.isa_launch_count.argtypes = [c_int] * 6 + [c_float, c_float, c_int]
    L.isa_launch_count.restype = c_int
    L.isa_selftest_wait_timeout.argtypes = [vp, c_int, vp]
    L.isa_selftest_wait_timeout.restype = c_int
    L.isa_selftest_exp2.argtypes = [vp, vp, vp, c_int, vp]
    L.isa_selftest_exp2.restype = c_int
    L.isa_set_stage_events.argtypes = [vp, c_int]
    L.isa_set_stage_events.restype = c_int
    L.isa_select_context_noalloc.argtypes = [vp, vp, vp] + [c_int] * 6 + [c_float, c_int, vp, vp, vp]
    L.isa_select_context_noalloc.restype = c_int
    L.isa_select_context_noalloc_status.argtypes = [vp]
    L.isa_select_context_noalloc_status.restype = c_int
    L.isa_forward_host_ns.argtypes = [vp, vp, vp] + [c_int] * 6 + [c_float, c_float, c_float, c_int, vp, vp, vp]
    L.isa_forward_host_ns.restype = c_int
    L.isa_workspace_bytes_varlen.argtypes = [c_int, c_int, vp, vp, c_int, c_int, c_float, c_int]
    L.isa_workspace_bytes_varlen.restype = c_size
    L.isa_forward_varlen.argtypes = [vp, vp, vp, c_int, c_int, vp, vp, c_int, c_int, c_float, c_float, c_int, vp, vp,
                                     vp, vp, c_size, vp]
    L.isa_forward_varlen.restype = c_int
    L.isa_forward_train.argtypes = [vp, vp, vp] + [c_int] * 6 + [c_float, c_float, c_int, vp, vp, vp, c_size, vp]
    L.isa_forward_train.restype = c_int
    L.isa_backward_workspace_bytes.argtypes = [c_int] * 6 + [c_float, c_int]
    L.isa_backward_workspace_bytes.restype = c_size
    L.isa_backward.argtypes = [vp] * 6 + [c_int] * 6 + [c_float, c_float, c_int, vp, vp, vp, vp, c_size, vp, c_size,
                                                          vp]
    L.isa_backward.restype = c_int
    L.isa_plan_ns.argtypes = [c_int] * 6 + [c_float, c_float, c_float, i32p, i32p, i32p, i32p]
    L.isa_plan_ns.restype = c_int
    L.isa_workspace_bytes_ns.argtypes = [c_int] * 6 + [c_float, c_float, c_int]
    L.isa_workspace_bytes_ns.restype = c_size
    L.isa_forward_ns.argtypes = [vp, vp, vp] + [c_int] * 6 + [c_float, c_float, c_float, c_int, vp, vp, vp, vp, vp,
                                                              c_size, vp]
    L.isa_forward_ns.restype = c_int
    L.isa_launch_count_ns.argtypes = [c_int] * 6 + [c_float, c_float, c_float, c_int]
    L.isa_launch_count_ns.restype = c_int
    L.isa_last_error.argtypes = []
    L.isa_last_error.restype = ctypes.c_char_p
    _LIB = L
    return L


def last_error() -> str:
    return lib().isa_last_error().decode()


def _check(rc: int):
    if rc != 0:
        raise IsaError(rc, last_error())


def plan(B, H, L_src, L_ctx, D, b, alpha_s, alpha_f) -> Tuple[int, int, int]:
    """(n_q, k, n_flat) for these sizes: query blocks, kept context blocks, Taylor blocks."""
    n_q, k, n_flat = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _check(lib().isa_plan(B, H, L_src, L_ctx, D, b, alpha_s, alpha_f, ctypes.byref(n_q), ctypes.byref(k),
                          ctypes.byref(n_flat)))
    return n_q.value, k.value, n_flat.value


def plan_ns(B, H, L_src, L_ctx, D, b, alpha_s, alpha_f, alpha_ns) -> Tuple[int, int, int, int]:
    """(n_q, k, n_flat, k_ns): plan() plus the exact key blocks per Taylor query block."""
    n_q, k, n_flat, k_ns = (ctypes.c_int32() for _ in range(4))
    _check(lib().isa_plan_ns(B, H, L_src, L_ctx, D, b, alpha_s, alpha_f, alpha_ns, ctypes.byref(n_q),
                             ctypes.byref(k), ctypes.byref(n_flat), ctypes.byref(k_ns)))
    return n_q.value, k.value, n_flat.value, k_ns.value


def workspace_bytes(B, H, L_src, L_ctx, D, b, alpha_s, dtype=ISA_BF16, alpha_ns: float = 0.0) -> int:
    if alpha_ns:
        n = lib().isa_workspace_bytes_ns(B, H, L_src, L_ctx, D, b, alpha_s, alpha_ns, dtype)
    else:
        n = lib().isa_workspace_bytes(B, H, L_src, L_ctx, D, b, alpha_s, dtype)
    if n == 0:
        raise IsaError(-1, last_error())
    return n


def launch_count(B, H, L_src, L_ctx, D, b, alpha_s, alpha_f, dtype=ISA_BF16, alpha_ns: float = 0.0) -> int:
    if alpha_ns:
        return lib().isa_launch_count_ns(B, H, L_src, L_ctx, D, b, alpha_s, alpha_f, alpha_ns, dtype)
    return lib().isa_launch_count(B, H, L_src, L_ctx, D, b, alpha_s, alpha_f, dtype)


def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return ISA_BF16
    if t.dtype == torch.float32:
        return ISA_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


_WS_CACHE = {}


def _workspace(device, nbytes: int):
    torch = _torch()
    key = (device.index if device.index is not None else torch.cuda.current_device())
    ws = _WS_CACHE.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
        _WS_CACHE[key] = ws
    return ws


def forward_into(q, k, v, out, L_src: int, L_ctx: int, b: int, alpha_s: float, alpha_f: float,
                 dbg_sel=None, dbg_route=None, workspace=None, stream=None, alpha_ns: float = 0.0, dbg_ns=None):
    """Enqueue the pass on ``stream`` (default: torch's current stream) writing ``out``.

    All tensors are CUDA tensors; q, k, v, out are contiguous [B, H, N, D] of one
    dtype (bfloat16 or float32); dbg_sel int32 [B, H, k] and dbg_route int32
    [B, H, n_q] are optional. With ``alpha_ns`` > 0 (bfloat16 only) the Taylor
    query blocks compute their k_ns best K_new blocks exactly (isa_forward_ns);
    dbg_ns int32 [B, H, n_q, k_ns] then receives those blocks. Asynchronous;
    returns the workspace used.
    """
    torch = _torch()
    for t in (q, k, v, out):
        if not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError("q, k, v and out must be contiguous 4-D CUDA tensors [B, H, N, D]")
    B, H, N, D = q.shape
    dt = _dtype_code(q)
    if workspace is None:
        workspace = _workspace(q.device, workspace_bytes(B, H, L_src, L_ctx, D, b, alpha_s, dt, alpha_ns))
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    s = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    if alpha_ns or dbg_ns is not None:
        _check(lib().isa_forward_ns(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, L_src, L_ctx, D, b, alpha_s, alpha_f, alpha_ns, dt,
            out.data_ptr(), dbg_sel.data_ptr() if dbg_sel is not None else None,
            dbg_route.data_ptr() if dbg_route is not None else None,
            dbg_ns.data_ptr() if dbg_ns is not None else None, workspace.data_ptr(), workspace.numel(), s))
        return workspace
    rc = lib().isa_forward_ex(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, L_src, L_ctx, D, b, alpha_s, alpha_f, dt, out.data_ptr(),
        dbg_sel.data_ptr() if dbg_sel is not None else None, dbg_route.data_ptr() if dbg_route is not None else None,
        workspace.data_ptr(), workspace.numel(), s)
    _check(rc)
    return workspace


def forward(q, k, v, L_src: int, L_ctx: int, b: int, alpha_s: float, alpha_f: float, debug: bool = False,
            stream=None, alpha_ns: float = 0.0):
    """ISA forward pass on CUDA tensors; returns out, or (out, sel, route) when ``debug``
    ((out, sel, route, ns) with ``alpha_ns`` > 0, ns int32 [B, H, n_q, k_ns])."""
    torch = _torch()
    out = torch.empty_like(q)
    sel = route = ns = None
    if debug:
        B, H, N, D = q.shape
        n_q, kk, _, k_ns = plan_ns(B, H, L_src, L_ctx, D, b, alpha_s, alpha_f, alpha_ns)
        sel = torch.empty((B, H, kk), dtype=torch.int32, device=q.device)
        route = torch.empty((B, H, n_q), dtype=torch.int32, device=q.device)
        if alpha_ns:
            ns = torch.empty((B, H, n_q, k_ns), dtype=torch.int32, device=q.device)
    forward_into(q, k, v, out, L_src, L_ctx, b, alpha_s, alpha_f, sel, route, stream=stream, alpha_ns=alpha_ns,
                 dbg_ns=ns)
    if not debug:
        return out
    return (out, sel, route, ns) if alpha_ns else (out, sel, route)


def device_status(workspace=None, stream=None):
    """Synchronise and raise IsaError(ISA_ERR_TIMEOUT) if a kernel wait gave up."""
    torch = _torch()
    if workspace is None:
        dev = torch.cuda.current_device()
        workspace = _WS_CACHE.get(dev)
        if workspace is None:
            return
    if stream is None:
        stream = torch.cuda.current_stream(workspace.device)
    s = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    _check(lib().isa_device_status(workspace.data_ptr(), s))


STAGES = ("pool_score_topk", "gather", "route", "attention")


def set_stage_events(events):
    """Record these 5 torch.cuda.Event objects around the 4 kernels of the next calls (None to stop)."""
    if events is None:
        _check(lib().isa_set_stage_events(None, 0))
        return
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    _check(lib().isa_set_stage_events(arr, len(events)))


def selftest_wait_timeout(workspace, timeout_ms: int = 100, stream=None):
    """Enqueue a kernel whose wait can never complete; its bounded wait gives up and flags ``workspace``."""
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream(workspace.device)
    s = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    _check(lib().isa_selftest_wait_timeout(workspace.data_ptr(), timeout_ms, s))


def debug_pooled(B, H, L_src, L_ctx, D, b, alpha_s, dtype=ISA_BF16, workspace=None, stream=None):
    """Intermediates of the last call made with ``workspace``: dict of Qc, Kc, Vc, colscore, sharp."""
    torch = _torch()
    n_ctx = -(-L_ctx // b)                  # the last block of each part may be short
    n_q = -(-L_src // b) + n_ctx
    dev = torch.cuda.current_device() if workspace is None else workspace.device
    if workspace is None:
        workspace = _WS_CACHE[dev]
    f = dict(device=workspace.device, dtype=torch.float32)
    res = dict(qc=torch.empty((B, H, n_q, D), **f), kc=torch.empty((B, H, n_q, D), **f),
               vc=torch.empty((B, H, n_q, D), **f), colscore=torch.empty((B, H, n_ctx), **f),
               sharp=torch.empty((B, H, n_q), **f))
    if stream is None:
        stream = torch.cuda.current_stream(workspace.device)
    s = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    _check(lib().isa_debug_pooled(B, H, L_src, L_ctx, D, b, alpha_s, dtype, workspace.data_ptr(),
                                  res["qc"].data_ptr(), res["kc"].data_ptr(), res["vc"].data_ptr(),
                                  res["colscore"].data_ptr(), res["sharp"].data_ptr(), s))
    return res


def _i32_array(xs):
    arr = (ctypes.c_int32 * len(xs))(*[int(x) for x in xs])
    return arr


def varlen_workspace_bytes(H, L_src, L_ctx, D, b, alpha_s, dtype=ISA_BF16) -> int:
    """Workspace of isa_forward_varlen for the per-element length lists L_src, L_ctx."""
    B = len(L_src)
    if len(L_ctx) != B:
        raise ValueError("L_src and L_ctx must have one entry per batch element")
    n = lib().isa_workspace_bytes_varlen(B, H, _i32_array(L_src), _i32_array(L_ctx), D, b, alpha_s, dtype)
    if n == 0:
        raise IsaError(-1, last_error())
    return n


def forward_varlen(q, k, v, H: int, L_src, L_ctx, b: int, alpha_s: float, alpha_f: float, out=None,
                   debug: bool = False, workspace=None, stream=None):
    """The pass over a variable-length batch (isa_forward_varlen).

    q, k, v: contiguous CUDA tensors holding the elements one after another, element i a
    [H, L_src[i] + L_ctx[i], D] block (at least 2-D; the last dimension is D). Returns out
    (same shape), or (out, sel, route) with ``debug``: sel and route are 1-D int32 tensors holding
    each element's [H, k_i] and [H, n_q_i] lists one after another.
    """
    torch = _torch()
    for t in (q, k, v):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k and v must be contiguous CUDA tensors")
    if q.dim() < 2:
        raise ValueError("q, k and v must be at least 2-D with D as the last dimension")
    B, D = len(L_src), q.shape[-1]
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty_like(q)
    sel = route = None
    if debug:
        n_sel = n_route = 0
        for ls, lc in zip(L_src, L_ctx):
            n_q, kk, _ = plan(1, H, ls, lc, D, b, alpha_s, alpha_f)
            n_sel += H * kk
            n_route += H * n_q
        sel = torch.empty(max(n_sel, 1), dtype=torch.int32, device=q.device)[:n_sel]
        route = torch.empty(n_route, dtype=torch.int32, device=q.device)
    if workspace is None:
        workspace = _workspace(q.device, varlen_workspace_bytes(H, L_src, L_ctx, D, b, alpha_s, dt))
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    s = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    _check(lib().isa_forward_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, _i32_array(L_src),
                                    _i32_array(L_ctx), D, b, alpha_s, alpha_f, dt, out.data_ptr(),
                                    sel.data_ptr() if debug and sel.numel() else None,
                                    route.data_ptr() if debug else None, workspace.data_ptr(), workspace.numel(), s))
    return (out, sel, route) if debug else out


def forward_train(q, k, v, L_src: int, L_ctx: int, b: int, alpha_s: float, alpha_f: float, stream=None):
    """Training forward (isa_forward_train): returns (out, lse, workspace).

    lse float32 [B, H, N] is each row's log softmax denominator; the workspace (a fresh tensor,
    not the module's shared one) holds the call's decisions and must be passed to ``backward``."""
    torch = _torch()
    B, H, N, D = q.shape
    dt = _dtype_code(q)
    out = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    ws = torch.empty(workspace_bytes(B, H, L_src, L_ctx, D, b, alpha_s, dt), dtype=torch.uint8, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    s = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    _check(lib().isa_forward_train(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, L_src, L_ctx, D, b, alpha_s,
                                   alpha_f, dt, out.data_ptr(), lse.data_ptr(), ws.data_ptr(), ws.numel(), s))
    return out, lse, ws


def backward(q, k, v, out, lse, dout, workspace, L_src: int, L_ctx: int, b: int, alpha_s: float, alpha_f: float,
             stream=None, bwd_workspace=None):
    """Gradients (dq, dk, dv) of sum(out * dout), from a forward_train call's tensors and workspace."""
    torch = _torch()
    B, H, N, D = q.shape
    dt = _dtype_code(q)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    nb = lib().isa_backward_workspace_bytes(B, H, L_src, L_ctx, D, b, alpha_s, dt)
    if nb == 0:
        raise IsaError(-1, last_error())
    if bwd_workspace is None or bwd_workspace.numel() < nb:
        bwd_workspace = torch.empty(nb, dtype=torch.uint8, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    s = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    _check(lib().isa_backward(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                              dout.data_ptr(), B, H, L_src, L_ctx, D, b, alpha_s, alpha_f, dt, dq.data_ptr(),
                              dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(), workspace.numel(),
                              bwd_workspace.data_ptr(), bwd_workspace.numel(), s))
    return dq, dk, dv


def select_context_noalloc(q, k, v, L_src: int, L_ctx: int, b: int, alpha_s: float, sel, colscore, stream=None):
    """Stages 1-2 through the allocation-free entry point (scratch in the library's fixed array).

    Enqueues only; call ``select_context_noalloc_status`` before the next call to learn whether
    the kernel's bounded waits gave up."""
    torch = _torch()
    B, H, N, D = q.shape
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    s = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    _check(lib().isa_select_context_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, L_src, L_ctx, D, b,
                                            alpha_s, _dtype_code(q), sel.data_ptr(), colscore.data_ptr(), s))


def select_context_noalloc_status(stream=None):
    """Synchronise and raise IsaError(ISA_ERR_TIMEOUT) if the last allocation-free call's wait gave up."""
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    s = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    _check(lib().isa_select_context_noalloc_status(s))


def forward_host(q, k, v, L_src: int, L_ctx: int, b: int, alpha_s: float, alpha_f: float, out=None,
                 dbg_sel=None, dbg_route=None, dtype: Optional[int] = None, alpha_ns: float = 0.0):
    """The pass on HOST buffers (numpy arrays or CPU tensors, pinned or not): copies in, runs, copies out.

    For bfloat16, pass uint16 numpy arrays holding the bit patterns, or bfloat16 CPU tensors.
    With ``alpha_ns`` > 0 the Taylor query blocks keep their k_ns best K_new blocks exact
    (isa_forward_host_ns).
    """
    import numpy as np

    def ptr(a):
        if a is None:
            return None
        if isinstance(a, np.ndarray):
            if not a.flags["C_CONTIGUOUS"]:
                raise ValueError("host arrays must be C-contiguous")
            return a.ctypes.data
        if not a.is_contiguous() or a.is_cuda:
            raise ValueError("host tensors must be contiguous CPU tensors")
        return a.data_ptr()

    B, H, N, D = q.shape
    if dtype is None:
        if isinstance(q, np.ndarray):
            dtype = ISA_F32 if q.dtype == np.float32 else ISA_BF16
        else:
            dtype = _dtype_code(q)
    if out is None:
        out = np.empty_like(q) if isinstance(q, np.ndarray) else _torch().empty_like(q)
    if alpha_ns:
        _check(lib().isa_forward_host_ns(ptr(q), ptr(k), ptr(v), B, H, L_src, L_ctx, D, b, alpha_s, alpha_f,
                                         alpha_ns, dtype, ptr(out), ptr(dbg_sel), ptr(dbg_route)))
        return out
    _check(lib().isa_forward_host(ptr(q), ptr(k), ptr(v), B, H, L_src, L_ctx, D, b, alpha_s, alpha_f, dtype,
                                  ptr(out), ptr(dbg_sel), ptr(dbg_route)))
    return out
