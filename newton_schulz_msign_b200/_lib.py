"""ctypes declarations of the C ABI in include/msign_b200.h.

Loading fails loudly when the shared library has not been built; there is no
fallback implementation.
"""

from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmsign_b200.so")

# msign_status
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT = range(6)
# msign_dtype
BF16, FP16, FP32 = 0, 1, 2

EXPORTS = (
    "msign_abi_version", "msign_status_string", "msign_sync_status",
    "msign_ns_workspace_size", "msign_ns", "msign_ns_route", "muon_step_route",
    "gram_xxt_workspace_size", "gram_xxt",
    "gram_ns_workspace_size", "gram_ns",
    "muon_step_workspace_size", "muon_step",
    "msign_profile_enable", "msign_profile_read", "msign_profile_reset",
    "msign_ns_noalloc_max_bytes", "msign_ns_noalloc",
    "msign_selftest_timeout", "msign_set_chaining", "msign_ns_host_workspace_size", "msign_ns_host",
    "mousse_inv_root_workspace_size", "mousse_inv_root", "mousse_direction_workspace_size", "mousse_direction",
)


class MsignCoeffs(ctypes.Structure):
    _fields_ = [("steps", ctypes.c_int), ("abc", ctypes.POINTER(ctypes.c_float)), ("eps", ctypes.c_float),
                ("init", ctypes.c_int), ("method", ctypes.c_int)]


class MsignError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


_lib = None

P = ctypes.c_void_p
I64 = ctypes.c_int64
SZ = ctypes.c_size_t
I32 = ctypes.c_int
F32 = ctypes.c_float


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m newton_schulz_msign_b200.build` "
                "(this package has no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        L.msign_abi_version.restype = I32
        L.msign_abi_version.argtypes = []
        L.msign_status_string.restype = ctypes.c_char_p
        L.msign_status_string.argtypes = [I32]
        L.msign_sync_status.restype = I32
        L.msign_sync_status.argtypes = [P]
        L.msign_ns_workspace_size.restype = SZ
        L.msign_ns_workspace_size.argtypes = [I64, I64, I64, I32]
        L.msign_ns.restype = I32
        L.msign_ns.argtypes = [P, P, I32, I32, I64, I64, I64, I64, I64, ctypes.POINTER(MsignCoeffs), P, SZ, P]
        L.msign_ns_host_workspace_size.restype = SZ
        L.msign_ns_host_workspace_size.argtypes = [I64, I64, I64, I32, I32]
        L.msign_ns_host.restype = I32
        L.msign_ns_host.argtypes = [P, P, I32, I32, I64, I64, I64, ctypes.POINTER(MsignCoeffs), P, SZ, P]
        L.msign_ns_route.restype = I32
        L.msign_ns_route.argtypes = [I64, I64, I64, I32, ctypes.POINTER(MsignCoeffs)]
        L.muon_step_route.restype = I32
        L.muon_step_route.argtypes = [I64, I64, ctypes.POINTER(MsignCoeffs)]
        L.gram_xxt_workspace_size.restype = SZ
        L.gram_xxt_workspace_size.argtypes = [I64, I64, I64, I32, P]
        L.gram_xxt.restype = I32
        L.gram_xxt.argtypes = [P, I32, P, I32, I64, I64, I64, P, SZ, P]
        L.gram_ns_workspace_size.restype = SZ
        L.gram_ns_workspace_size.argtypes = [I64, I64, I64]
        L.gram_ns.restype = I32
        L.gram_ns.argtypes = [P, P, I32, I64, I64, I64, I64, I64, ctypes.POINTER(MsignCoeffs),
                              ctypes.POINTER(I32), I32, P, SZ, P]
        L.muon_step_workspace_size.restype = SZ
        L.muon_step_workspace_size.argtypes = [I32, ctypes.POINTER(I64), ctypes.POINTER(I64)]
        L.muon_step.restype = I32
        L.muon_step.argtypes = [I32, ctypes.POINTER(P), ctypes.POINTER(P), ctypes.POINTER(P),
                                ctypes.POINTER(I64), ctypes.POINTER(I64), I32, I32, F32, F32,
                                ctypes.POINTER(MsignCoeffs), P, SZ, P]
        L.msign_profile_enable.restype = I32
        L.msign_profile_enable.argtypes = [I32]
        L.msign_profile_read.restype = I32
        L.msign_profile_read.argtypes = [I32, ctypes.POINTER(I32), ctypes.POINTER(ctypes.c_double),
                                         ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)]
        L.msign_profile_reset.restype = I32
        L.msign_profile_reset.argtypes = []
        L.msign_ns_noalloc_max_bytes.restype = SZ
        L.msign_ns_noalloc_max_bytes.argtypes = []
        L.msign_selftest_timeout.restype = I32
        L.msign_selftest_timeout.argtypes = [ctypes.c_uint64, P]
        L.msign_set_chaining.restype = I32
        L.msign_set_chaining.argtypes = [I32]
        L.msign_ns_noalloc.restype = I32
        L.msign_ns_noalloc.argtypes = [P, P, I32, I64, I64, I64, ctypes.POINTER(MsignCoeffs), P]
        L.mousse_inv_root_workspace_size.restype = SZ
        L.mousse_inv_root_workspace_size.argtypes = [I64, I64]
        L.mousse_inv_root.restype = I32
        L.mousse_inv_root.argtypes = [P, P, I64, I64, F32, I32, P, SZ, P]
        L.mousse_direction_workspace_size.restype = SZ
        L.mousse_direction_workspace_size.argtypes = [I64, I64, I64]
        L.mousse_direction.restype = I32
        L.mousse_direction.argtypes = [P, P, I32, I64, I64, I64, P, P, ctypes.POINTER(MsignCoeffs), P, SZ, P]
        _lib = L
    return _lib


def status_string(status: int) -> str:
    try:
        return lib().msign_status_string(int(status)).decode()
    except RuntimeError:
        return "library not loaded"


def check(status: int, what: str) -> None:
    if status != OK:
        raise MsignError(status, what)


def make_coeffs(schedule=None, eps=None, init=0, method=0):
    """(MsignCoeffs, keep-alive buffer) for a list of (a, b, c) triples."""
    if schedule is None and eps is None and not init and not method:
        return None, None
    c = MsignCoeffs()
    c.eps = -1.0 if eps is None else float(eps)
    c.init = int(init)
    c.method = int(method)
    if schedule is None:
        c.steps = 0
        c.abc = None
        return c, None
    flat = [float(v) for abc in schedule for v in abc]
    buf = (ctypes.c_float * len(flat))(*flat)
    c.steps = len(flat) // 3
    c.abc = ctypes.cast(buf, ctypes.POINTER(ctypes.c_float))
    return c, buf
