"""C-ABI checks that need no GPU: the library builds and loads, exports every
function the header declares, and rejects bad arguments on the host before
touching CUDA."""

import ctypes
import os
import re

import pytest

from conftest import ROOT
from newton_schulz_msign_b200 import _lib, build

HEADER = os.path.join(ROOT, "include", "msign_b200.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.lib()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w \*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "sizeof")))


def test_header_declares_the_boundary():
    assert header_functions() == sorted(_lib.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    for name in header_functions():
        assert hasattr(L, name), name


def test_exported_symbols_match_nm(L):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for name in header_functions():
        assert name in exported


def test_abi_version_and_status_strings(L):
    assert L.msign_abi_version() == 106
    assert L.msign_status_string(_lib.OK) == b"ok"
    assert b"timed out" in L.msign_status_string(_lib.ERR_TIMEOUT)
    assert L.msign_status_string(99) == b"unknown status"


def test_workspace_queries_are_host_only(L):
    assert L.msign_ns_workspace_size(0, 16, 16, _lib.BF16) == 0
    a = L.msign_ns_workspace_size(1, 256, 512, _lib.BF16)
    b = L.msign_ns_workspace_size(1, 512, 256, _lib.BF16)
    assert a == b > 0  # the tall case is oriented to the wide one
    # two X operand copies + A + B (bf16) + fp32 X, 4096 x 4096
    big = L.msign_ns_workspace_size(1, 4096, 4096, _lib.BF16)
    assert 4096 * 4096 * (2 + 2 + 4 + 2 + 2) <= big < 4096 * 4096 * 12 + 2 ** 20
    assert L.gram_ns_workspace_size(2, 1024, 4096) > 0
    rows = (ctypes.c_int64 * 3)(4096, 1024, 14336)
    cols = (ctypes.c_int64 * 3)(4096, 4096, 4096)
    assert L.muon_step_workspace_size(3, rows, cols) > L.msign_ns_workspace_size(1, 4096, 14336, _lib.BF16)
    # aligned X with m % 8 == 0 needs no staging workspace
    assert L.gram_xxt_workspace_size(1, 100, 64, _lib.BF16, 1 << 20) == 0
    assert L.gram_xxt_workspace_size(1, 100, 63, _lib.BF16, 1 << 20) > 0
    # host buffers: the device copy of the matrices (256-byte rounded) ahead of msign_ns's workspace
    for io, es in ((_lib.BF16, 2), (_lib.FP32, 4)):
        h = L.msign_ns_host_workspace_size(3, 100, 70, io, _lib.BF16)
        assert h == -(-3 * 100 * 70 * es // 256) * 256 + L.msign_ns_workspace_size(3, 100, 70, _lib.BF16)
    assert L.msign_ns_host_workspace_size(0, 100, 70, _lib.BF16, _lib.BF16) == 0


def test_host_buffer_call_checks_before_any_copy(L):
    # argument errors of msign_ns_host come back before anything is enqueued
    # (no device is touched: these run without a GPU)
    buf = (ctypes.c_uint16 * 16)()
    p = ctypes.addressof(buf)
    assert L.msign_ns_host(p, p, 7, _lib.BF16, 1, 4, 4, None, None, 0, None) == _lib.ERR_INVALID_ARG
    assert L.msign_ns_host(p, p, _lib.BF16, _lib.BF16, -1, 4, 4, None, None, 0, None) == _lib.ERR_INVALID_ARG
    assert L.msign_ns_host(None, None, _lib.BF16, _lib.BF16, 0, 4, 4, None, None, 0, None) == _lib.OK
    assert L.msign_ns_host(None, p, _lib.BF16, _lib.BF16, 1, 4, 4, None, None, 0, None) == _lib.ERR_INVALID_ARG
    assert L.msign_ns_host(p, p, _lib.BF16, _lib.BF16, 65536, 4, 4, None, None, 0, None) == _lib.ERR_UNSUPPORTED
    assert L.msign_ns_host(p, p, _lib.BF16, _lib.BF16, 1, 4, 4, None, None, 0, None) == _lib.ERR_WORKSPACE


def test_invalid_arguments_rejected_on_host(L):
    # negative sizes and bad dtypes fail before any CUDA call
    assert L.msign_ns(None, None, _lib.BF16, _lib.BF16, -1, 4, 4, 0, 0, None, None, 0, None) == _lib.ERR_INVALID_ARG
    assert L.msign_ns(None, None, 7, _lib.BF16, 1, 4, 4, 0, 0, None, None, 0, None) == _lib.ERR_INVALID_ARG
    # empty problems are a no-op
    assert L.msign_ns(None, None, _lib.BF16, _lib.BF16, 0, 4, 4, 0, 0, None, None, 0, None) == _lib.OK
    assert L.msign_ns(None, None, _lib.BF16, _lib.BF16, 3, 0, 4, 0, 0, None, None, 0, None) == _lib.OK
    # null data pointers with a non-empty problem
    assert L.msign_ns(None, None, _lib.BF16, _lib.BF16, 1, 4, 4, 0, 0, None, None, 0, None) == _lib.ERR_INVALID_ARG
    # a coefficient table needs a positive step count
    c = _lib.MsignCoeffs()
    buf = (ctypes.c_float * 3)(1.0, 0.0, 0.0)
    c.steps, c.abc, c.eps = 0, ctypes.cast(buf, ctypes.POINTER(ctypes.c_float)), -1.0
    assert L.msign_ns(None, None, _lib.BF16, _lib.BF16, 1, 4, 4, 0, 0, ctypes.byref(c), None, 0, None) == \
        _lib.ERR_INVALID_ARG
    c.steps = 100  # beyond the built maximum
    assert L.msign_ns(None, None, _lib.BF16, _lib.BF16, 1, 4, 4, 0, 0, ctypes.byref(c), None, 0, None) == \
        _lib.ERR_UNSUPPORTED
    # workspace missing for a real problem (pointer values are never dereferenced on this path)
    assert L.msign_ns(16, 16, _lib.BF16, _lib.BF16, 1, 4, 4, 0, 0, None, None, 0, None) == _lib.ERR_WORKSPACE
    assert L.msign_ns(16, 16, _lib.BF16, _lib.FP32, 1, 4, 4, 0, 0, None, None, 0, None) == _lib.ERR_WORKSPACE
    # the fp32-accurate path keeps two fp32 planes per operand: larger workspace
    assert L.msign_ns_workspace_size(1, 512, 512, _lib.FP32) > L.msign_ns_workspace_size(1, 512, 512, _lib.BF16)


def test_init_option_validation(L):
    # msign_coeffs.init: 0 or 1; the sharper normalisation needs 16-bit
    # operands and is a standard-NS option
    c = _lib.MsignCoeffs()
    c.steps, c.abc, c.eps, c.init = 0, None, -1.0, 2
    assert L.msign_ns(16, 16, _lib.BF16, _lib.BF16, 1, 4, 4, 0, 0, ctypes.byref(c), None, 0, None) == _lib.ERR_INVALID_ARG
    c.init = 1
    assert L.msign_ns(16, 16, _lib.BF16, _lib.FP32, 1, 4, 4, 0, 0, ctypes.byref(c), None, 0, None) == _lib.ERR_UNSUPPORTED
    assert L.gram_ns(16, 16, _lib.BF16, 1, 4, 8, 0, 0, ctypes.byref(c), None, 0, None, 0, None) == _lib.ERR_UNSUPPORTED
    # bf16 with init = 1 passes the argument checks (fails only on the missing workspace)
    assert L.msign_ns(16, 16, _lib.BF16, _lib.BF16, 1, 4, 4, 0, 0, ctypes.byref(c), None, 0, None) == _lib.ERR_WORKSPACE


def _route(L, batch, rows, cols, compute=_lib.BF16, method=1, init=0, steps=0):
    c = _lib.MsignCoeffs()
    c.steps, c.abc, c.eps, c.init, c.method = steps, None, -1.0, init, method
    return L.msign_ns_route(batch, rows, cols, compute, ctypes.byref(c))


def test_route_rule(L):
    # the automatic route takes Gram NS only for 16-bit problems with
    # n >= 512 and m - n >= 3072 (>= 2048 where n <= 2048), in either
    # orientation, whose Gram-NS workspace fits in msign_ns's
    assert _route(L, 1, 1024, 16384) == 1
    assert _route(L, 1, 16384, 1024) == 1
    assert _route(L, 3, 512, 4608) == 1
    assert _route(L, 1, 4096, 8192) == 1
    assert _route(L, 4, 4096, 11008) == 1
    assert _route(L, 1, 14336, 4096) == 1
    assert _route(L, 1, 1024, 16384, compute=_lib.FP16) == 1
    assert _route(L, 1, 1024, 4096) == 1
    assert _route(L, 1, 4096, 1024) == 1
    assert _route(L, 1, 512, 2560) == 1     # m - n = 2048 at n <= 2048
    assert _route(L, 4, 2048, 4096) == 1
    assert _route(L, 1, 3072, 6144) == 1    # m - n = 3072 at n > 2048
    assert _route(L, 1, 4096, 7168) == 1
    assert _route(L, 1, 512, 2559) == 0     # m - n < 2048
    assert _route(L, 1, 1024, 3071) == 0
    assert _route(L, 1, 4096, 6144) == 0    # m - n < 3072 at n > 2048
    assert _route(L, 1, 3072, 5119) == 0
    assert _route(L, 1, 2048, 4096) == 0    # Gram NS's workspace would not fit
    assert L.gram_ns_workspace_size(1, 2048, 4096) > L.msign_ns_workspace_size(1, 2048, 4096, _lib.BF16)
    assert _route(L, 1, 511, 8192) == 0     # n < 512
    assert _route(L, 1, 4096, 4096) == 0
    assert _route(L, 1, 1024, 16384, compute=_lib.FP32) == 0   # fp32-accurate stays standard
    assert _route(L, 1, 1024, 16384, init=1) == 0              # sharper init is standard-only
    assert _route(L, 1, 1024, 16384, method=0) == 0
    assert L.msign_ns_route(1, 1024, 16384, _lib.BF16, None) == 0  # NULL coeffs: standard
    # arguments msign_ns rejects come back negated
    assert _route(L, 1, 1024, 16384, method=2) == -_lib.ERR_INVALID_ARG
    assert _route(L, 1, 1024, 16384, compute=_lib.FP32, init=1) == -_lib.ERR_UNSUPPORTED
    assert _route(L, 1, 1024, 16384, steps=100) == -_lib.ERR_UNSUPPORTED
    assert L.msign_ns_route(-1, 4, 4, _lib.BF16, None) == -_lib.ERR_INVALID_ARG


def test_muon_route_rule(L):
    # muon_step takes Gram NS only where msign_ns's route does and m - n >= 4096
    c = _lib.MsignCoeffs()
    c.steps, c.abc, c.eps, c.init, c.method = 0, None, -1.0, 0, 1
    assert L.muon_step_route(4096, 14336, ctypes.byref(c)) == 1
    assert L.muon_step_route(14336, 4096, ctypes.byref(c)) == 1
    assert L.muon_step_route(4096, 11008, ctypes.byref(c)) == 1
    assert L.muon_step_route(600, 5000, ctypes.byref(c)) == 1
    assert _route(L, 1, 1024, 4096) == 1 and L.muon_step_route(1024, 4096, ctypes.byref(c)) == 0
    assert L.muon_step_route(4096, 4096, ctypes.byref(c)) == 0
    assert L.muon_step_route(0, 4096, ctypes.byref(c)) == 0
    assert L.muon_step_route(4096, 14336, None) == 0  # NULL coeffs: standard
    c.init = 1
    assert L.muon_step_route(4096, 14336, ctypes.byref(c)) == 0  # the sharper init is standard-only
    c.init, c.method = 0, 2
    assert L.muon_step_route(4096, 14336, ctypes.byref(c)) == -_lib.ERR_INVALID_ARG
    assert L.muon_step_route(-1, 4, None) == -_lib.ERR_INVALID_ARG
    # every matrix the Muon route takes is one msign_ns's route takes
    c.method = 1
    for n in (256, 512, 1024, 2048, 3072, 4096):
        for m in (n + 2048, n + 3072, n + 4096, 2 * n, 4 * n):
            if L.muon_step_route(n, m, ctypes.byref(c)) == 1:
                assert _route(L, 1, n, m) == 1 and m - n >= 4096


def test_route_workspace_fits(L):
    # wherever the route picks Gram NS, its workspace fits in msign_ns's
    # (the one query a caller makes)
    routed = 0
    for batch in (1, 2, 8):
        for n in (512, 640, 1024, 1536, 2048, 3072, 4096, 8192, 16384):
            for m in (n + 2048, n + 3072, n + 4096, n + 5000, 2 * n, 3 * n, 4 * n, 8 * n, 16 * n):
                if _route(L, batch, n, m) == 1:
                    routed += 1
                    assert L.gram_ns_workspace_size(batch, n, m) <= L.msign_ns_workspace_size(batch, n, m, _lib.BF16)
    assert routed > 100


def test_method_field_validation(L):
    c = _lib.MsignCoeffs()
    c.steps, c.abc, c.eps, c.init, c.method = 0, None, -1.0, 0, 1
    assert L.gram_ns(16, 16, _lib.BF16, 1, 4, 8, 0, 0, ctypes.byref(c), None, -1, 16, 1 << 20, None) == \
        _lib.ERR_INVALID_ARG
    one = (ctypes.c_void_p * 1)(16)
    rows = (ctypes.c_int64 * 1)(8)
    cols = (ctypes.c_int64 * 1)(8)
    # muon_step takes the route too: these arguments pass the checks and
    # fail only on the missing workspace
    assert L.muon_step(1, one, one, one, rows, cols, _lib.BF16, _lib.BF16, 0.95, 0.02, ctypes.byref(c), None, 0,
                       None) == _lib.ERR_WORKSPACE
    c.method = 3
    assert L.muon_step(1, one, one, one, rows, cols, _lib.BF16, _lib.BF16, 0.95, 0.02, ctypes.byref(c), None, 0,
                       None) == _lib.ERR_INVALID_ARG
    assert L.msign_ns(16, 16, _lib.BF16, _lib.BF16, 1, 4, 4, 0, 0, ctypes.byref(c), None, 0, None) == \
        _lib.ERR_INVALID_ARG


def test_selftest_timeout_validation(L):
    assert L.msign_selftest_timeout(0, None) == _lib.ERR_INVALID_ARG
    assert L.msign_selftest_timeout(2_000_000_000, None) == _lib.ERR_INVALID_ARG


def test_gram_ns_restart_validation(L):
    r = (ctypes.c_int * 1)(5)  # must lie in 1..T-1
    assert L.gram_ns(16, 16, _lib.BF16, 1, 4, 8, 0, 0, None, ctypes.cast(r, ctypes.POINTER(ctypes.c_int)), 1, None, 0,
                     None) == _lib.ERR_INVALID_ARG
    assert L.gram_ns(16, 16, _lib.BF16, 1, 4, 8, 0, 0, None, None, 2, None, 0, None) == _lib.ERR_INVALID_ARG
    assert L.gram_ns(16, 16, _lib.BF16, 1, 4, 8, 0, 0, None, None, -1, None, 0, None) == _lib.ERR_WORKSPACE


def test_muon_step_validation(L):
    assert L.muon_step(0, None, None, None, None, None, _lib.BF16, _lib.BF16, 0.95, 0.02, None, None, 0,
                       None) == _lib.OK
    assert L.muon_step(-1, None, None, None, None, None, _lib.BF16, _lib.BF16, 0.95, 0.02, None, None, 0,
                       None) == _lib.ERR_INVALID_ARG
    one = (ctypes.c_void_p * 1)(16)
    rows = (ctypes.c_int64 * 1)(8)
    cols = (ctypes.c_int64 * 1)(8)
    assert L.muon_step(1, one, one, one, rows, cols, _lib.FP16, _lib.BF16, 0.95, 0.02, None, None, 0,
                       None) == _lib.ERR_UNSUPPORTED
    assert L.muon_step(1, one, one, one, rows, cols, _lib.BF16, _lib.BF16, float("nan"), 0.02, None, None, 0,
                       None) == _lib.ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors():
    import torch
    import newton_schulz_msign_b200 as msb
    with pytest.raises(ValueError, match="CUDA"):
        msb.msign_ns(torch.zeros(4, 4))


def test_binding_noalloc_checks_on_host():
    # the no-allocation binding takes the caller's CUDA tensors only, and
    # reports the built-in scratch size without a GPU
    import torch
    import newton_schulz_msign_b200 as msb
    build.build()
    assert msb.msign_ns_noalloc_max_bytes() == 32 << 20
    with pytest.raises(ValueError, match="CUDA"):
        msb.msign_ns_noalloc(torch.zeros(4, 4), torch.zeros(4, 4))


def test_binding_route_query():
    # the Python binding's route query is host-only as well
    import newton_schulz_msign_b200 as msb
    build.build()
    assert msb.msign_ns_route(1, 1024, 16384) == "gram"
    assert msb.msign_ns_route(1, 1024, 16384, method="standard") == "standard"
    assert msb.msign_ns_route(1, 1024, 16384, "fp32") == "standard"
    assert msb.msign_ns_route(1, 1024, 16384, improved_init=True) == "standard"
    assert msb.msign_ns_route(4, 4096, 11008) == "gram"
    assert msb.msign_ns_route(8, 4096, 4096) == "standard"
    assert msb.muon_step_route(4096, 14336) == "gram"
    assert msb.muon_step_route(1024, 4096) == "standard"
    assert msb.muon_step_route(4096, 14336, method="standard") == "standard"
    with pytest.raises(msb.MsignError):
        msb.msign_ns_route(1, 1024, 16384, coeffs=[(1.0, 0.0, 0.0)] * 100)


def test_binding_rejects_tensors_on_another_device():
    # every tensor of a call must live on the device the call runs on
    import torch

    import newton_schulz_msign_b200 as msb

    with pytest.raises(ValueError):
        msb._same_device(torch.empty(1), torch.device("cuda", 0), "out")
    msb._same_device(torch.empty(1), torch.device("cpu"), "out")
    msb._same_device(None, torch.device("cuda", 0), "workspace")


def test_batch_strides_validated_on_host(L):
    # a stride is 0 (back to back) or at least one matrix; overlapping
    # matrices are rejected before anything else is looked at
    assert L.msign_ns(16, 16, _lib.BF16, _lib.BF16, 2, 4, 4, 15, 0, None, None, 0, None) == _lib.ERR_INVALID_ARG
    assert L.msign_ns(16, 16, _lib.BF16, _lib.BF16, 2, 4, 4, 0, -1, None, None, 0, None) == _lib.ERR_INVALID_ARG
    assert L.gram_ns(16, 16, _lib.BF16, 2, 4, 8, 31, 0, None, None, -1, None, 0, None) == _lib.ERR_INVALID_ARG
    # valid strides pass the checks (and fail only on the missing workspace)
    assert L.msign_ns(16, 16, _lib.BF16, _lib.BF16, 2, 4, 4, 16, 48, None, None, 0, None) == _lib.ERR_WORKSPACE
    assert L.gram_ns(16, 16, _lib.BF16, 2, 4, 8, 64, 32, None, None, -1, None, 0, None) == _lib.ERR_WORKSPACE


def test_binding_batch_layout():
    import torch

    import newton_schulz_msign_b200 as msb

    class FakeCuda:
        """Shape and strides of a tensor, posing as a CUDA tensor."""

        is_cuda = True

        def __init__(self, t):
            self.t = t
            self.shape = t.shape

        def dim(self):
            return self.t.dim()

        def stride(self, d):
            return self.t.stride(d)

    big = torch.empty(5, 3, 7, 9)
    assert msb._batch_layout(FakeCuda(big), "x") == (15, 7, 9, 0)
    assert msb._batch_layout(FakeCuda(big[:, 1]), "x") == (5, 7, 9, 3 * 63)
    assert msb._batch_layout(FakeCuda(big[1:4:2, 2]), "x") == (2, 7, 9, 2 * 3 * 63)
    with pytest.raises(ValueError):
        msb._batch_layout(FakeCuda(big[1:4:2]), "x")  # leading dims without one common stride
    with pytest.raises(ValueError):
        msb._batch_layout(FakeCuda(big[..., ::2]), "x")  # matrix not dense
    assert msb._batch_layout(FakeCuda(big[0, 0]), "x") == (1, 7, 9, 0)
    # empty batches and empty matrices pass whatever strides torch gave them
    assert msb._batch_layout(FakeCuda(torch.empty(0, 64, 96)), "x") == (0, 64, 96, 0)
    assert msb._batch_layout(FakeCuda(torch.empty(5, 0, 8)), "x") == (5, 0, 8, 0)
    assert msb._batch_layout(FakeCuda(torch.empty(4, 16, 0)), "x") == (4, 16, 0, 0)


def test_mousse_arguments_validated_on_host(L):
    F32 = ctypes.c_float
    # inverse root: eps must be finite and >= 0, iters in [2, 1000] (0: default)
    assert L.mousse_inv_root(16, 16, 1, 8, F32(-1.0), 0, None, 0, None) == _lib.ERR_INVALID_ARG
    assert L.mousse_inv_root(16, 16, 1, 8, F32(0.1), 1, None, 0, None) == _lib.ERR_INVALID_ARG
    assert L.mousse_inv_root(16, 16, 1, 8, F32(0.1), 1001, None, 0, None) == _lib.ERR_INVALID_ARG
    assert L.mousse_inv_root(None, None, 0, 8, F32(0.1), 0, None, 0, None) == _lib.OK
    assert L.mousse_inv_root(None, 16, 1, 8, F32(0.1), 0, None, 0, None) == _lib.ERR_INVALID_ARG
    assert L.mousse_inv_root(16, 16, 1, 8, F32(0.1), 0, None, 0, None) == _lib.ERR_WORKSPACE
    assert L.mousse_inv_root_workspace_size(1, 8) > 0
    # direction: every matrix pointer is needed; method must be 0
    assert L.mousse_direction(16, 16, _lib.BF16, 1, 8, 16, None, 16, None, None, 0, None) == _lib.ERR_INVALID_ARG
    c = _lib.MsignCoeffs()
    c.steps, c.abc, c.eps, c.init, c.method = 0, None, -1.0, 0, 1
    assert L.mousse_direction(16, 16, _lib.BF16, 1, 8, 16, 16, 16, ctypes.byref(c), None, 0, None) == \
        _lib.ERR_INVALID_ARG
    assert L.mousse_direction(16, 16, _lib.BF16, 1, 8, 16, 16, 16, None, None, 0, None) == _lib.ERR_WORKSPACE
    assert L.mousse_direction_workspace_size(1, 8, 16) > L.msign_ns_workspace_size(1, 8, 16, _lib.BF16)
