"""muon_step on the GPU against the fp64 oracle."""

import math

import numpy as np
import pytest
import torch

import newton_schulz_msign_b200 as msb
from newton_schulz_msign_b200 import synth
from oracle import ns_oracle as O

from helpers import TOL_BF16, rel_fro, to_np

pytestmark = pytest.mark.gpu


def make(shapes, wdt, gdt, seed):
    W, M, G = [], [], []
    for i, (r, c) in enumerate(shapes):
        W.append(synth.gaussian_torch((r, c), seed=seed + 3 * i, device="cuda", std=0.02).to(wdt))
        M.append(synth.gaussian_torch((r, c), seed=seed + 3 * i + 1, device="cuda", std=1e-3))
        G.append(synth.gaussian_torch((r, c), seed=seed + 3 * i + 2, device="cuda", std=1e-4).to(gdt))
    return W, M, G


def check_matrix(W0, M0, G, W1, M1, lr, mu=0.95):
    r, c = W0.shape
    Wr, Mr, Or = O.muon_step(to_np(W0), to_np(M0), to_np(G), momentum=mu, lr=lr, input_cast="bf16")
    # momentum: fp32 fused multiply-add of exact inputs
    assert rel_fro(to_np(M1), Mr) < 1e-6
    scale = math.sqrt(max(1.0, r / c))
    dW_ref = Wr - to_np(W0)
    w1 = to_np(W1)
    if W1.dtype == torch.float32:
        excess = np.abs(w1 - Wr)
    else:
        # bf16 weights: W1 is the bf16 rounding of W0 + dW_gpu, so
        # |W1 - Wr| <= half a bf16 ulp of W1 + |dW_gpu - dW_ref| per element.
        # Removing the half ulp leaves (at most) the update's own error.
        half_ulp = np.ldexp(1.0, np.frexp(np.abs(w1))[1] - 9)
        excess = np.maximum(np.abs(w1 - Wr) - half_ulp, 0.0)
    # the update's error within the bf16-path tolerance of the exact update,
    # in Frobenius norm ...
    assert np.linalg.norm(excess) <= TOL_BF16 * np.linalg.norm(dW_ref)
    # ... and element by element within a fifth of the update's RMS entry:
    # rounding noise of relative size ~1e-2 stays far below that, while one
    # wrong element (a mask or index slip) is of the size of the entry itself
    rms = lr * scale * np.sqrt(np.mean(Or * Or))
    assert float(excess.max()) <= 0.2 * rms


@pytest.mark.parametrize("wdt,gdt", [(torch.float32, torch.float32), (torch.float32, torch.bfloat16),
                                     (torch.bfloat16, torch.bfloat16)])
def test_muon_small_mixed_shapes(wdt, gdt):
    # ragged shapes of both orientations; 33 x 257 (a small, flat, very wide
    # Gaussian spectrum) is the hardest case for bf16 operands
    shapes = [(64, 128), (128, 64), (96, 96), (200, 72), (64, 128), (33, 257), (80, 240)]
    W, M, G = make(shapes, wdt, gdt, seed=100)
    W0 = [w.clone() for w in W]
    M0 = [m.clone() for m in M]
    msb.muon_step(W, M, G, momentum=0.95, lr=0.02)
    msb.sync_status()
    for i in range(len(shapes)):
        check_matrix(W0[i], M0[i], G[i], W[i], M[i], 0.02)


def test_muon_many_shape_classes():
    # seven distinct oriented shapes: more classes than one chained launch
    # holds, so every step runs phase by phase
    shapes = [(64, 128), (96, 96), (200, 72), (80, 240), (48, 160), (32, 96), (120, 130)]
    W, M, G = make(shapes, torch.float32, torch.float32, seed=500)
    W0 = [w.clone() for w in W]
    M0 = [m.clone() for m in M]
    msb.muon_step(W, M, G, momentum=0.95, lr=0.02)
    msb.sync_status()
    for i in range(len(shapes)):
        check_matrix(W0[i], M0[i], G[i], W[i], M[i], 0.02)


def test_muon_equals_msign_composition():
    # the fused step equals momentum + msign_ns + scaled update done by hand
    shapes = [(256, 128), (128, 384)]
    W, M, G = make(shapes, torch.float32, torch.float32, seed=200)
    W0 = [w.clone() for w in W]
    M0 = [m.clone() for m in M]
    msb.muon_step(W, M, G, momentum=0.9, lr=0.05)
    msb.sync_status()
    for i, (r, c) in enumerate(shapes):
        Mn = 0.9 * M0[i] + G[i]
        assert torch.allclose(M[i], Mn, rtol=1e-6, atol=1e-9)
        O_ = msb.msign_ns(Mn)
        Wn = W0[i] - 0.05 * math.sqrt(max(1.0, r / c)) * O_
        assert torch.allclose(W[i], Wn, rtol=1e-5, atol=1e-6)


def test_muon_small_workspace_processes_in_groups():
    shapes = [(128, 256), (256, 128), (128, 256), (64, 64)]
    W, M, G = make(shapes, torch.float32, torch.float32, seed=300)
    Wb, Mb = [w.clone() for w in W], [m.clone() for m in M]
    msb.muon_step(W, M, G)
    need_one = max(msb.muon_step_workspace_size([s]) for s in shapes)
    ws = torch.empty(need_one, dtype=torch.uint8, device="cuda")
    msb.muon_step(Wb, Mb, G, workspace=ws)
    msb.sync_status()
    for a, b in zip(W, Wb):
        assert torch.equal(a, b)
    for a, b in zip(M, Mb):
        assert torch.equal(a, b)


def test_muon_llama_layer_full_size():
    # one Llama-3-8B decoder layer (q, k, v, o, gate, up, down) at full size,
    # bf16 weights, fp32 momentum, G ~ N(0, 1e-4^2); all seven matrices are
    # checked against the oracle (gate and up are the tall ones, which run
    # transposed on ingest and are stored back transposed)
    shapes = [(r, c) for _, r, c in synth.llama3_8b_layer_shapes()]
    W, M, G = make(shapes, torch.bfloat16, torch.bfloat16, seed=400)
    for m in M:
        m.zero_()
    W0 = [w.clone() for w in W]
    M0 = [m.clone() for m in M]
    msb.muon_step(W, M, G, momentum=0.95, lr=0.02)
    msb.sync_status()
    for w in W:
        assert torch.isfinite(w).all()
    for i in range(len(shapes)):
        check_matrix(W0[i], M0[i], G[i], W[i], M[i], 0.02)


def test_muon_improved_init():
    # the sharper step-0 normalisation inside the Muon update
    shapes = [(128, 256), (256, 128), (96, 96)]
    W, M, G = make(shapes, torch.float32, torch.float32, seed=600)
    W0 = [w.clone() for w in W]
    M0 = [m.clone() for m in M]
    msb.muon_step(W, M, G, momentum=0.95, lr=0.02, improved_init=True)
    msb.sync_status()
    for i, (r, c) in enumerate(shapes):
        Mr = 0.95 * to_np(M0[i]) + to_np(G[i])
        O_ref = O.msign_ns_improved_init(Mr, input_cast="bf16")
        dW_ref = -0.02 * math.sqrt(max(1.0, r / c)) * O_ref
        assert rel_fro(to_np(W[i]) - to_np(W0[i]), dW_ref) < TOL_BF16


def test_muon_auto_route_mixed():
    # method="auto": the wide matrices (m - n >= 4096, n >= 512) run Gram NS,
    # the others standard NS, in one call; each against its fp64 oracle.
    # 1024 x 3072 is one msign_ns's route gives to Gram NS and muon_step's
    # keeps in the standard group.
    shapes = [(600, 5000), (256, 384), (5000, 600), (512, 512), (1024, 3072)]
    gram_shapes = {(600, 5000), (5000, 600)}
    for r, c in shapes:
        want = "gram" if (r, c) in gram_shapes else "standard"
        assert msb.muon_step_route(r, c, method="auto") == want
    assert msb.msign_ns_route(1, 1024, 3072, method="auto") == "gram"
    W, M, G = make(shapes, torch.bfloat16, torch.bfloat16, seed=900)
    W0 = [w.clone() for w in W]
    M0 = [m.clone() for m in M]
    msb.muon_step(W, M, G, momentum=0.95, lr=0.02, method="auto")
    msb.sync_status()
    for i, (r, c) in enumerate(shapes):
        if (r, c) not in gram_shapes:
            check_matrix(W0[i], M0[i], G[i], W[i], M[i], 0.02)
            continue
        m_ref = 0.95 * to_np(M0[i]).astype(np.float64) + to_np(G[i]).astype(np.float64)
        assert rel_fro(to_np(M[i]), m_ref) < 1e-6
        # O from Gram NS of the fp32 momentum (fp16 inside), as the GPU gets it
        o_ref = O.gram_ns(to_np(M[i]))
        w_ref = to_np(W0[i]) - 0.02 * math.sqrt(max(1.0, r / c)) * o_ref
        dW_ref = w_ref - to_np(W0[i])
        w1 = to_np(W[i])
        half_ulp = np.ldexp(1.0, np.frexp(np.abs(w1))[1] - 9)
        excess = np.maximum(np.abs(w1 - w_ref) - half_ulp, 0.0)
        assert np.linalg.norm(excess) <= TOL_BF16 * np.linalg.norm(dW_ref)
        assert float(excess.max()) <= 0.2 * 0.02 * math.sqrt(max(1.0, r / c)) * np.sqrt(np.mean(o_ref * o_ref))
        # and the standard-NS update agrees within the same tolerance
        w_std, _, _ = O.muon_step(to_np(W0[i]), to_np(M0[i]), to_np(G[i]), momentum=0.95, lr=0.02, input_cast="bf16")
        assert rel_fro(w_ref - to_np(W0[i]), w_std - to_np(W0[i])) < TOL_BF16


def test_muon_llama_stack_one_step():
    # the whole 32-layer Llama-3-8B stack (224 matrices, ~7e9 parameters) in
    # one call, as the Muon workload runs it: bf16 weights, fp32 momenta from
    # zero, bf16 G ~ N(0, 1e-4^2).  After the step every matrix is finite and
    # one matrix of each distinct shape -- q (4096^2), k (1024x4096), gate
    # (14336x4096, tall) and down (4096x14336) -- matches the oracle; the
    # spot checks sit in different layers of the stack.
    layer = [(r, c) for _, r, c in synth.llama3_8b_layer_shapes()]
    shapes = layer * synth.LLAMA3_8B_LAYERS
    W = [synth.gaussian_torch(s, seed=7000 + i, device="cuda", std=0.02, dtype=torch.bfloat16)
         for i, s in enumerate(shapes)]
    M = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in shapes]
    G = [synth.gaussian_torch(s, seed=9000 + i, device="cuda", std=1e-4, dtype=torch.bfloat16)
         for i, s in enumerate(shapes)]
    picks = [7 * 3 + 0, 7 * 11 + 1, 7 * 20 + 4, 7 * 31 + 6]  # q, k, gate, down in layers 3, 11, 20, 31
    W0 = {i: W[i].clone() for i in picks}
    # the automatic route: q, k, v, o run standard NS, gate, up and down
    # Gram NS (batched by shape), all in one call
    assert [msb.muon_step_route(r, c) for r, c in layer] == ["standard"] * 4 + ["gram"] * 3
    method = "auto"
    msb.muon_step(W, M, G, momentum=0.95, lr=0.02, method=method)
    msb.sync_status()
    for w in W:
        assert torch.isfinite(w).all()
    for i in picks:
        r, c = shapes[i]
        if method == "auto" and msb.muon_step_route(r, c, method="auto") == "gram":
            # Gram NS (fp16 inside) on the momentum M = G; the update against
            # its own oracle and within the acceptance bound of standard NS
            o_ref = O.gram_ns(to_np(M[i]))
            dW_ref = -0.02 * math.sqrt(max(1.0, r / c)) * o_ref
            w1 = to_np(W[i])
            half_ulp = np.ldexp(1.0, np.frexp(np.abs(w1))[1] - 9)
            excess = np.maximum(np.abs(w1 - (to_np(W0[i]) + dW_ref)) - half_ulp, 0.0)
            assert np.linalg.norm(excess) <= TOL_BF16 * np.linalg.norm(dW_ref)
        else:
            check_matrix(W0[i], torch.zeros(shapes[i], device="cuda"), G[i], W[i], M[i], 0.02)
