"""msign_ns_noalloc: the entry point for callers that cannot allocate device
memory (graph capture, framework-owned memory pools, allocation-free loops).
It runs msign_ns in a scratch array built into the library, so it must give
the same answers as msign_ns with a caller workspace, call after call.

Kept in a file of its own that pytest collects last."""

import numpy as np
import pytest
import torch

import newton_schulz_msign_b200 as msb
from newton_schulz_msign_b200 import _lib, synth

from helpers import TOL_BF16, rel_fro, to_np

pytestmark = pytest.mark.gpu


def noalloc(x, out):
    L = _lib.lib()
    stream = torch.cuda.current_stream().cuda_stream
    rows, cols = x.shape[-2], x.shape[-1]
    batch = x.numel() // (rows * cols)
    code = {torch.bfloat16: _lib.BF16, torch.float16: _lib.FP16, torch.float32: _lib.FP32}[x.dtype]
    return L.msign_ns_noalloc(x.data_ptr(), out.data_ptr(), code, batch, rows, cols, None, stream)


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
        assert torch.isfinite(out).all()
        assert rel_fro(to_np(out), to_np(ref)) < TOL_BF16


def test_noalloc_tall_fp32_batch_matches_msign_ns():
    x = torch.from_numpy(synth.gaussian((2, 520, 200), seed=73)).cuda()
    ref = msb.msign_ns(x)
    out = torch.empty_like(x)
    torch.cuda.synchronize()
    for _ in range(2):
        out.zero_()
        assert noalloc(x, out) == _lib.OK
        msb.sync_status()
        assert rel_fro(to_np(out), to_np(ref)) < TOL_BF16


def test_noalloc_rejects_problems_beyond_the_builtin_scratch():
    L = _lib.lib()
    assert L.msign_ns_noalloc_max_bytes() == 32 << 20
    assert msb.msign_ns_workspace_size(1, 2048, 2048) > L.msign_ns_noalloc_max_bytes()
    x = torch.zeros(2048, 2048, dtype=torch.bfloat16, device="cuda")
    out = torch.full_like(x, 7.0)
    assert noalloc(x, out) == _lib.ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())  # nothing was enqueued


def test_noalloc_follows_the_automatic_route():
    # msign_coeffs.method = 1 through the no-allocation entry point: a shape
    # the route sends to Gram NS fits the built-in scratch too
    x = torch.from_numpy(synth.gaussian((512, 4608), seed=73)).to(torch.bfloat16).cuda()
    assert msb.msign_ns_route(1, 512, 4608, method="auto") == "gram"
    ref = msb.msign_ns(x, method="auto")
    out = torch.empty_like(x)
    c = _lib.MsignCoeffs()
    c.steps, c.abc, c.eps, c.init, c.method = 0, None, -1.0, 0, 1
    L = _lib.lib()
    stream = torch.cuda.current_stream().cuda_stream
    assert L.msign_ns_noalloc(x.data_ptr(), out.data_ptr(), _lib.BF16, 1, 512, 4608, c, stream) == _lib.OK
    msb.sync_status()
    assert torch.equal(out, ref)
