"""B200 (sm_100a) Newton-Schulz msign: thin PyTorch binding of the C ABI.

Each function marshals tensors into the pointer/size arguments of the C entry
point of the same name (include/msign_b200.h) and enqueues it on the current
CUDA stream.  Every step of the computation runs in the library's kernels;
PyTorch only supplies device memory and the stream.  There is no CPU path:
calling these without the built library or without a CUDA tensor raises.
"""

from __future__ import annotations

import ctypes
import math

from . import _lib
from ._lib import BF16, FP16, FP32, MsignError, check, make_coeffs

__all__ = [
    "MsignError", "msign_ns", "msign_ns_workspace_size", "msign_ns_route", "msign_ns_host",
    "msign_ns_host_workspace_size", "msign_ns_noalloc", "msign_ns_noalloc_max_bytes",
    "gram_xxt", "gram_xxt_workspace_size", "gram_ns",
    "gram_ns_workspace_size", "muon_step", "muon_step_workspace_size", "muon_step_route", "mousse_inv_root",
    "mousse_direction",
    "sync_status", "selftest_timeout", "set_chaining", "library_path",
]


def library_path() -> str:
    return _lib.LIB_PATH


def _torch():
    import torch

    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    m = {torch.bfloat16: BF16, torch.float16: FP16, torch.float32: FP32}
    if t.dtype not in m:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return m[t.dtype]


def _compute_code(name) -> int:
    return {"bf16": BF16, "fp16": FP16, "fp32": FP32}[name]


def _stream(stream, device=None) -> int:
    """The raw cudaStream_t: the given stream, else the current stream of
    ``device`` (of the current device when None)."""
    torch = _torch()
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _need_cuda(t, name):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _batch_layout(t, name):
    """(batch, rows, cols, stride) of a CUDA tensor whose last two dims are a
    dense row-major matrix and whose leading dims step through memory with
    one stride (any view of that form, e.g. ``big[:, 0]``); stride 0 means
    back to back."""
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if t.dim() < 2:
        raise ValueError(f"{name} needs at least two dims")
    rows, cols = t.shape[-2], t.shape[-1]
    if rows * cols == 0:  # empty matrices have no layout to check
        return math.prod(t.shape[:-2]), rows, cols, 0
    if (cols > 1 and t.stride(-1) != 1) or (rows > 1 and t.stride(-2) != cols):
        raise ValueError(f"{name}: each matrix (the last two dims) must be dense row-major")
    lead = [(t.shape[d], t.stride(d)) for d in range(t.dim() - 2) if t.shape[d] != 1]
    batch = math.prod(sz for sz, _ in lead)
    if batch <= 1:
        return batch, rows, cols, 0
    stride = lead[-1][1]
    for (sz_o, st_o), (sz_i, st_i) in zip(lead[:-1], lead[1:]):
        if st_o != st_i * sz_i:
            raise ValueError(f"{name}: the batch dims must step through memory with one stride")
    if stride < rows * cols:
        raise ValueError(f"{name}: matrices of the batch overlap (stride {stride} < {rows * cols})")
    return batch, rows, cols, (0 if stride == rows * cols else stride)


def _same_device(t, device, name):
    """The C side works on the current device: every tensor of a call must
    live on the device the call runs on."""
    if t is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, the call runs on {device}")


def _workspace(nbytes, device, workspace):
    torch = _torch()
    if workspace is not None:
        _same_device(workspace, device, "workspace")
    if nbytes == 0:
        return workspace, (0 if workspace is None else workspace.numel() * workspace.element_size())
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return workspace, workspace.numel() * workspace.element_size()


def _ptr(t):
    return None if t is None else t.data_ptr()


def sync_status(stream=None, device=None) -> None:
    """Waits for the stream (default: the current stream of ``device``, or of
    the current device) and raises MsignError if a kernel's bounded wait on
    that device ran out."""
    torch = _torch()
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        check(_lib.lib().msign_sync_status(_stream(stream, device)), "msign_sync_status")


# ---------------------------------------------------------------- msign_ns

def msign_ns_workspace_size(batch: int, rows: int, cols: int, compute: str = "bf16") -> int:
    return int(_lib.lib().msign_ns_workspace_size(batch, rows, cols, _compute_code(compute)))


_METHODS = {"standard": 0, "auto": 1}


def msign_ns_route(batch: int, rows: int, cols: int, compute: str = "bf16", *, method: str = "auto", coeffs=None,
                   improved_init=False) -> str:
    """The iteration ``msign_ns`` runs for these arguments: "standard" or "gram" (host only)."""
    c, keep = make_coeffs(coeffs, None, 1 if improved_init else 0, _METHODS[method])
    r = _lib.lib().msign_ns_route(batch, rows, cols, _compute_code(compute), ctypes.byref(c) if c is not None else None)
    del keep
    if r < 0:
        check(-r, "msign_ns_route")
    return "gram" if r == 1 else "standard"


def msign_ns(x, out=None, *, compute: str = "bf16", coeffs=None, eps=None, improved_init=False, method="standard",
             workspace=None, stream=None):
    """Newton-Schulz msign of the last two dims of ``x`` (bf16/fp16/fp32 CUDA tensor).

    ``x`` and ``out`` may be batched views whose matrices are dense but not
    back to back (e.g. ``big[:, 0]``): their batch strides are passed on.
    ``improved_init``: the sharper step-0 normalisation (msign_coeffs.init = 1).
    ``method``: "standard" (standard NS) or "auto" (Gram NS where ``msign_ns_route``
    picks it, msign_coeffs.method = 1)."""
    torch = _torch()
    batch, rows, cols, in_stride = _batch_layout(x, "x")
    if out is None:
        out = torch.empty(x.shape, dtype=x.dtype, device=x.device)
    _same_device(out, x.device, "out")
    if out.shape != x.shape or out.dtype != x.dtype:
        raise ValueError("out must match x in shape and dtype")
    _, _, _, out_stride = _batch_layout(out, "out")
    with torch.cuda.device(x.device):
        ws, wsb = _workspace(msign_ns_workspace_size(batch, rows, cols, compute), x.device, workspace)
        c, keep = make_coeffs(coeffs, eps, 1 if improved_init else 0, _METHODS[method])
        st = _lib.lib().msign_ns(x.data_ptr(), out.data_ptr(), _dtype_code(x), _compute_code(compute), batch, rows,
                                 cols, in_stride, out_stride, ctypes.byref(c) if c is not None else None, _ptr(ws),
                                 wsb, _stream(stream, x.device))
        del keep
    check(st, "msign_ns")
    return out


def msign_ns_host_workspace_size(batch: int, rows: int, cols: int, io: str = "bf16", compute: str = "bf16") -> int:
    return int(_lib.lib().msign_ns_host_workspace_size(batch, rows, cols, _compute_code(io), _compute_code(compute)))


def msign_ns_host(x, out=None, *, compute: str = "bf16", coeffs=None, eps=None, improved_init=False,
                  method="standard", workspace=None, stream=None, device=None):
    """msign_ns of HOST matrices (``x``: a CPU tensor, dense, bf16/fp16/fp32;
    page-locked for asynchronous copies): the call enqueues the copy in, the
    iteration and the copy out on ``stream`` (default: the current stream of
    ``device``, default the current device) and returns ``out`` (a CPU
    tensor, page-locked when allocated here) BEFORE the result is there:
    synchronize the stream before reading it.  ``workspace``: a device uint8
    tensor of at least msign_ns_host_workspace_size() bytes."""
    torch = _torch()
    if x.is_cuda or out is not None and out.is_cuda:
        raise ValueError("msign_ns_host takes host (CPU) tensors; use msign_ns for device tensors")
    if not x.is_contiguous():
        raise ValueError("x must be contiguous")
    if x.dim() < 2:
        raise ValueError("x needs at least two dims")
    rows, cols = x.shape[-2], x.shape[-1]
    batch = x.numel() // max(rows * cols, 1) if rows * cols else 0
    if out is None:
        out = torch.empty(x.shape, dtype=x.dtype).pin_memory()
    if out.shape != x.shape or out.dtype != x.dtype or not out.is_contiguous():
        raise ValueError("out must be a contiguous CPU tensor matching x in shape and dtype")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    io = _dtype_code(x)
    with torch.cuda.device(dev):
        need = int(_lib.lib().msign_ns_host_workspace_size(batch, rows, cols, io, _compute_code(compute)))
        ws, wsb = _workspace(need, dev, workspace)
        c, keep = make_coeffs(coeffs, eps, 1 if improved_init else 0, _METHODS[method])
        st = _lib.lib().msign_ns_host(x.data_ptr(), out.data_ptr(), io, _compute_code(compute), batch, rows, cols,
                                      ctypes.byref(c) if c is not None else None, _ptr(ws), wsb, _stream(stream, dev))
        del keep
    check(st, "msign_ns_host")
    return out


def msign_ns_noalloc_max_bytes() -> int:
    """Size of the scratch array built into the library (the largest
    msign_ns_workspace_size() that msign_ns_noalloc accepts)."""
    return int(_lib.lib().msign_ns_noalloc_max_bytes())


def msign_ns_noalloc(x, out, *, coeffs=None, eps=None, improved_init=False, method="standard", stream=None):
    """msign_ns (bf16 arithmetic) in the library's built-in scratch array: no
    workspace and no device allocation.  ``x`` and ``out`` are the caller's
    dense CUDA tensors of one shape and dtype.  Calls on one device share the
    scratch array: order them on one stream.  Raises MsignError with status
    ERR_WORKSPACE, before anything is enqueued, when the problem needs more
    than msign_ns_noalloc_max_bytes() of workspace."""
    torch = _torch()
    _need_cuda(x, "x")
    _need_cuda(out, "out")
    _same_device(out, x.device, "out")
    if x.dim() < 2:
        raise ValueError("x needs at least two dims")
    if out.shape != x.shape or out.dtype != x.dtype:
        raise ValueError("out must match x in shape and dtype")
    rows, cols = x.shape[-2], x.shape[-1]
    batch = math.prod(x.shape[:-2])
    c, keep = make_coeffs(coeffs, eps, 1 if improved_init else 0, _METHODS[method])
    with torch.cuda.device(x.device):
        st = _lib.lib().msign_ns_noalloc(x.data_ptr(), out.data_ptr(), _dtype_code(x), batch, rows, cols,
                                         ctypes.byref(c) if c is not None else None, _stream(stream, x.device))
    del keep
    check(st, "msign_ns_noalloc")
    return out


# ---------------------------------------------------------------- gram_xxt

def gram_xxt_workspace_size(x) -> int:
    n, m = x.shape[-2], x.shape[-1]
    batch = math.prod(x.shape[:-2])
    return int(_lib.lib().gram_xxt_workspace_size(batch, n, m, _dtype_code(x), x.data_ptr()))


def gram_xxt(x, out=None, *, out_dtype=None, workspace=None, stream=None):
    """A = X X^T over the last two dims of ``x`` (bf16 or fp16), exactly symmetric."""
    torch = _torch()
    _need_cuda(x, "x")
    n, m = x.shape[-2], x.shape[-1]
    batch = math.prod(x.shape[:-2])
    if out is None:
        out = torch.empty(*x.shape[:-2], n, n, dtype=out_dtype or x.dtype, device=x.device)
    _need_cuda(out, "out")
    _same_device(out, x.device, "out")
    if tuple(out.shape) != tuple(x.shape[:-2]) + (n, n):
        raise ValueError("out must be (..., n, n)")
    with torch.cuda.device(x.device):
        ws, wsb = _workspace(gram_xxt_workspace_size(x), x.device, workspace)
        st = _lib.lib().gram_xxt(x.data_ptr(), _dtype_code(x), out.data_ptr(), _dtype_code(out), batch, n, m,
                                 _ptr(ws), wsb, _stream(stream, x.device))
    check(st, "gram_xxt")
    return out


# ---------------------------------------------------------------- gram_ns

def gram_ns_workspace_size(batch: int, rows: int, cols: int) -> int:
    return int(_lib.lib().gram_ns_workspace_size(batch, rows, cols))


def gram_ns(x, out=None, *, coeffs=None, eps=None, restart_after=(2,), workspace=None, stream=None):
    """Stabilized Gram Newton-Schulz (fp16 inner iteration) of the last two dims of ``x``
    (batched views with one batch stride accepted, as for ``msign_ns``)."""
    torch = _torch()
    batch, rows, cols, in_stride = _batch_layout(x, "x")
    if out is None:
        out = torch.empty(x.shape, dtype=x.dtype, device=x.device)
    _same_device(out, x.device, "out")
    if out.shape != x.shape or out.dtype != x.dtype:
        raise ValueError("out must match x in shape and dtype")
    _, _, _, out_stride = _batch_layout(out, "out")
    c, keep = make_coeffs(coeffs, eps)
    if restart_after is None:
        rbuf, nr = None, -1
    else:
        r = [int(v) for v in restart_after]
        rbuf, nr = (ctypes.c_int * max(1, len(r)))(*r), len(r)
    with torch.cuda.device(x.device):
        ws, wsb = _workspace(gram_ns_workspace_size(batch, rows, cols), x.device, workspace)
        st = _lib.lib().gram_ns(x.data_ptr(), out.data_ptr(), _dtype_code(x), batch, rows, cols, in_stride,
                                out_stride, ctypes.byref(c) if c is not None else None,
                                ctypes.cast(rbuf, ctypes.POINTER(ctypes.c_int)) if rbuf is not None else None, nr,
                                _ptr(ws), wsb, _stream(stream, x.device))
    del keep
    check(st, "gram_ns")
    return out


# ---------------------------------------------------------------- muon_step

def _i64_array(vals):
    return (ctypes.c_int64 * len(vals))(*[int(v) for v in vals])


def muon_step_route(rows: int, cols: int, *, coeffs=None, improved_init=False, method="auto") -> str:
    """The iteration ``muon_step`` runs for one rows x cols matrix: "standard" or "gram" (host only)."""
    c, keep = make_coeffs(coeffs, None, 1 if improved_init else 0, _METHODS[method])
    r = _lib.lib().muon_step_route(rows, cols, ctypes.byref(c) if c is not None else None)
    del keep
    if r < 0:
        check(-r, "muon_step_route")
    return "gram" if r == 1 else "standard"


def muon_step_workspace_size(shapes) -> int:
    rows = _i64_array([s[0] for s in shapes])
    cols = _i64_array([s[1] for s in shapes])
    return int(_lib.lib().muon_step_workspace_size(len(shapes), rows, cols))


def muon_step(weights, momenta, grads, *, momentum: float = 0.95, lr: float = 0.02, coeffs=None, eps=None,
              improved_init=False, method="standard", workspace=None, stream=None):
    """In-place Muon update of lists of weights (bf16/fp32), fp32 momenta and grads (bf16/fp32).

    ``method="auto"``: the matrices ``muon_step_route`` gives to Gram NS take it
    (msign_coeffs.method = 1)."""
    torch = _torch()
    num = len(weights)
    if not (len(momenta) == num and len(grads) == num):
        raise ValueError("weights, momenta and grads must have the same length")
    if num == 0:
        return
    device = weights[0].device
    for w, m, g in zip(weights, momenta, grads):
        for t, nm in ((w, "weight"), (m, "momentum"), (g, "grad")):
            _need_cuda(t, nm)
            _same_device(t, device, nm)
        if w.dim() != 2 or w.shape != m.shape or w.shape != g.shape:
            raise ValueError("each weight, momentum and grad must be the same 2-D shape")
        if m.dtype != torch.float32:
            raise TypeError("momenta must be float32")
    wdt = {_dtype_code(w) for w in weights}
    gdt = {_dtype_code(g) for g in grads}
    if len(wdt) != 1 or len(gdt) != 1:
        raise TypeError("all weights (and all grads) must share one dtype")
    shapes = [tuple(w.shape) for w in weights]
    W = (ctypes.c_void_p * num)(*[w.data_ptr() for w in weights])
    M = (ctypes.c_void_p * num)(*[m.data_ptr() for m in momenta])
    G = (ctypes.c_void_p * num)(*[g.data_ptr() for g in grads])
    rows = _i64_array([s[0] for s in shapes])
    cols = _i64_array([s[1] for s in shapes])
    c, keep = make_coeffs(coeffs, eps, 1 if improved_init else 0, _METHODS[method])
    with torch.cuda.device(device):
        ws, wsb = _workspace(muon_step_workspace_size(shapes), device, workspace)
        st = _lib.lib().muon_step(num, W, M, G, rows, cols, wdt.pop(), gdt.pop(), float(momentum), float(lr),
                                  ctypes.byref(c) if c is not None else None, _ptr(ws), wsb,
                                  _stream(stream, device))
    del keep
    check(st, "muon_step")


# ---------------------------------------------------------------- Mousse

def mousse_inv_root(a, out=None, *, eps: float = 0.0, iters: int = 0, workspace=None, stream=None):
    """(A + eps I)^(-1/4) of symmetric positive semidefinite fp32 matrices (the
    last two dims of ``a``), exactly symmetric, by the coupled Newton
    iteration in fp32-accurate arithmetic (``iters`` 0: the library default)."""
    torch = _torch()
    _need_cuda(a, "a")
    if a.dtype != torch.float32 or a.dim() < 2 or a.shape[-1] != a.shape[-2]:
        raise ValueError("a must be float32 (..., n, n)")
    n = a.shape[-1]
    batch = math.prod(a.shape[:-2])
    if out is None:
        out = torch.empty_like(a)
    _need_cuda(out, "out")
    _same_device(out, a.device, "out")
    if out.shape != a.shape or out.dtype != torch.float32:
        raise ValueError("out must match a")
    with torch.cuda.device(a.device):
        ws, wsb = _workspace(int(_lib.lib().mousse_inv_root_workspace_size(batch, n)), a.device, workspace)
        st = _lib.lib().mousse_inv_root(a.data_ptr(), out.data_ptr(), batch, n, float(eps), int(iters), _ptr(ws), wsb,
                                        _stream(stream, a.device))
    check(st, "mousse_inv_root")
    return out


def mousse_direction(g, l_root, r_root, out=None, *, coeffs=None, eps=None, improved_init=False, workspace=None,
                     stream=None):
    """L^(-1/4) msign(L^(-1/4) G R^(-1/4)) R^(-1/4) of the last two dims of ``g``,
    given ``l_root`` = L^(-1/4) (..., rows, rows) and ``r_root`` = R^(-1/4)
    (..., cols, cols) as float32 (e.g. from ``mousse_inv_root``)."""
    torch = _torch()
    for t, nm in ((g, "g"), (l_root, "l_root"), (r_root, "r_root")):
        _need_cuda(t, nm)
        _same_device(t, g.device, nm)
    if g.dim() < 2:
        raise ValueError("g needs at least two dims")
    rows, cols = g.shape[-2], g.shape[-1]
    lead = tuple(g.shape[:-2])
    if (l_root.dtype != torch.float32 or r_root.dtype != torch.float32 or tuple(l_root.shape) != lead + (rows, rows)
            or tuple(r_root.shape) != lead + (cols, cols)):
        raise ValueError("l_root and r_root must be float32 (..., rows, rows) and (..., cols, cols)")
    batch = math.prod(lead)
    if out is None:
        out = torch.empty_like(g)
    _need_cuda(out, "out")
    _same_device(out, g.device, "out")
    if out.shape != g.shape or out.dtype != g.dtype:
        raise ValueError("out must match g")
    c, keep = make_coeffs(coeffs, eps, 1 if improved_init else 0, 0)
    with torch.cuda.device(g.device):
        ws, wsb = _workspace(int(_lib.lib().mousse_direction_workspace_size(batch, rows, cols)), g.device, workspace)
        st = _lib.lib().mousse_direction(g.data_ptr(), out.data_ptr(), _dtype_code(g), batch, rows, cols,
                                         l_root.data_ptr(), r_root.data_ptr(),
                                         ctypes.byref(c) if c is not None else None, _ptr(ws), wsb,
                                         _stream(stream, g.device))
    del keep
    check(st, "mousse_direction")
    return out


# ---------------------------------------------------------------- launch records

PROFILE_KINDS = {"gemm": 0, "norm": 1, "ingest": 2, "elementwise": 3}


def selftest_timeout(limit_ns: int = 50_000_000, stream=None) -> None:
    """Makes the library's bounded waits expire on purpose (see
    msign_selftest_timeout): the next sync_status() raises MsignError with
    status ERR_TIMEOUT, and the GPU context stays usable."""
    check(_lib.lib().msign_selftest_timeout(int(limit_ns), _stream(stream)), "msign_selftest_timeout")


def set_chaining(enable: bool) -> bool:
    """Diagnostics (msign_set_chaining): False runs each product of a
    standard-route iteration step as a launch of its own, for profiling the
    phases apart; True (the default) chains them.  Returns the previous
    setting."""
    return bool(_lib.lib().msign_set_chaining(1 if enable else 0))


def profile_enable(enable: bool = True) -> None:
    check(_lib.lib().msign_profile_enable(1 if enable else 0), "msign_profile_enable")


def profile_reset() -> None:
    check(_lib.lib().msign_profile_reset(), "msign_profile_reset")


def profile_read(kind: str) -> dict:
    """{'launches', 'ms', 'flops', 'bytes'} summed over the recorded launches of one kind."""
    n = ctypes.c_int()
    ms, fl, by = ctypes.c_double(), ctypes.c_double(), ctypes.c_double()
    check(_lib.lib().msign_profile_read(PROFILE_KINDS[kind], ctypes.byref(n), ctypes.byref(ms), ctypes.byref(fl),
                                        ctypes.byref(by)), "msign_profile_read")
    return {"launches": n.value, "ms": ms.value, "flops": fl.value, "bytes": by.value}
