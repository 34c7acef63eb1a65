"""msign_ns_noalloc: the entry point for callers that cannot allocate device
memory where they call msign (plugins whose host framework owns every byte of
GPU memory through its own pool, loops that forbid allocation after
start-up).  It runs msign_ns in a scratch array built into the library, so
it must give exactly what msign_ns gives with a caller workspace, call after
call, and must not allocate.

Kept in a file of its own that pytest collects last."""

import ctypes

import pytest
import torch

import newton_schulz_msign_b200 as msb
from newton_schulz_msign_b200 import _lib, synth
from oracle import ns_oracle as O

from helpers import TOL_BF16, rel_fro, to_np

pytestmark = pytest.mark.gpu


def noalloc(x, out, coeffs=None):
    L = _lib.lib()
    stream = torch.cuda.current_stream().cuda_stream
    rows, cols = x.shape[-2], x.shape[-1]
    batch = x.numel() // (rows * cols)
    code = {torch.bfloat16: _lib.BF16, torch.float16: _lib.FP16, torch.float32: _lib.FP32}[x.dtype]
    return L.msign_ns_noalloc(x.data_ptr(), out.data_ptr(), code, batch, rows, cols,
                              ctypes.byref(coeffs) if coeffs is not None else None, stream)


def free_device_bytes():
    """Free bytes on the current device (cudaMemGetInfo)."""
    return torch.cuda.mem_get_info()[0]


def test_noalloc_matches_msign_ns_on_two_calls_in_a_row():
    xs = [torch.from_numpy(synth.gaussian((384, 640), seed=s)).to(torch.bfloat16).cuda() for s in (71, 72)]
    outs = [torch.empty_like(x) for x in xs]
    # allocate everything first, then run the two no-allocation calls back to back
    refs = [msb.msign_ns(x) for x in xs]
    torch.cuda.synchronize()
    for x, out in zip(xs, outs):
        assert noalloc(x, out) == _lib.OK
    msb.sync_status()
    for out, ref in zip(outs, refs):
        # the same kernels on the same values: bit for bit the same result
        assert torch.equal(out, ref)
    # and the first against the fp64 oracle, as every msign_ns result is
    assert rel_fro(to_np(outs[0]), O.msign_ns(to_np(xs[0]), input_cast="bf16")) < TOL_BF16


def test_noalloc_tall_fp32_batch_matches_msign_ns():
    x = torch.from_numpy(synth.gaussian((2, 520, 200), seed=73)).cuda()
    ref = msb.msign_ns(x)
    out = torch.empty_like(x)
    torch.cuda.synchronize()
    for _ in range(2):
        out.zero_()
        assert noalloc(x, out) == _lib.OK
        msb.sync_status()
        assert torch.equal(out, ref)
    assert rel_fro(to_np(out), O.msign_ns(to_np(x), input_cast="bf16")) < TOL_BF16


def test_noalloc_allocates_nothing():
    x = torch.from_numpy(synth.gaussian((256, 1024), seed=74)).to(torch.bfloat16).cuda()
    out = torch.empty_like(x)
    assert noalloc(x, out) == _lib.OK  # the first call on the device does the set-up
    torch.cuda.synchronize()
    torch_bytes = torch.cuda.memory_allocated()
    free = free_device_bytes()
    for _ in range(2):
        assert noalloc(x, out) == _lib.OK
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == torch_bytes
    assert free_device_bytes() == free
    msb.sync_status()
    assert torch.equal(out, msb.msign_ns(x))


def test_noalloc_rejects_problems_beyond_the_builtin_scratch():
    L = _lib.lib()
    assert L.msign_ns_noalloc_max_bytes() == 32 << 20
    assert msb.msign_ns_workspace_size(1, 2048, 2048) > L.msign_ns_noalloc_max_bytes()
    x = torch.zeros(2048, 2048, dtype=torch.bfloat16, device="cuda")
    out = torch.full_like(x, 7.0)
    assert noalloc(x, out) == _lib.ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())  # nothing was enqueued


def test_noalloc_binding_matches_msign_ns():
    # the Python binding of the same name: same result, and the size check
    # raises before anything is enqueued
    x = torch.from_numpy(synth.gaussian((3, 200, 330), seed=75)).to(torch.float16).cuda()
    ref = msb.msign_ns(x)
    out = torch.empty_like(x)
    torch.cuda.synchronize()
    assert msb.msign_ns_noalloc(x, out) is out
    msb.sync_status()
    assert torch.equal(out, ref)
    big = torch.zeros(2048, 2048, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(msb.MsignError) as e:
        msb.msign_ns_noalloc(big, torch.empty_like(big))
    assert e.value.status == _lib.ERR_WORKSPACE


def test_noalloc_follows_the_automatic_route():
    # msign_coeffs.method = 1 through the no-allocation entry point: a shape
    # the route sends to Gram NS fits the built-in scratch too
    x = torch.from_numpy(synth.gaussian((512, 4608), seed=73)).to(torch.bfloat16).cuda()
    assert msb.msign_ns_route(1, 512, 4608, method="auto") == "gram"
    ref = msb.msign_ns(x, method="auto")
    out = torch.empty_like(x)
    c = _lib.MsignCoeffs()
    c.steps, c.abc, c.eps, c.init, c.method = 0, None, -1.0, 0, 1
    assert noalloc(x, out, c) == _lib.OK
    msb.sync_status()
    assert torch.equal(out, ref)
    assert rel_fro(to_np(out), O.gram_ns(to_np(x))) < TOL_BF16
