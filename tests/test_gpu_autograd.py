"""The differentiable loss (linear_cross_entropy / linear_cross_entropy_quantized):
values and gradients against torch autograd on materialised logits.

bf16 inputs: the fused backward rounds dZ to bf16 (relative 2^-9) and the
gradients come back as bf16, so the bar is a relative Frobenius error below
1e-2 against an fp32 reference on the same bf16 values (the element-wise
derived bounds are tested against the oracle elsewhere).  fp32 inputs run the
three-product split, so against an fp64 reference the bar is 1e-4.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_bf16_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_cross_entropy_bf16_b200 import build
    build.build()
    oracle.build()


def rel(a, b):
    a, b = a.double(), b.double()
    return float((a - b).norm() / max(b.norm(), 1e-30))


def reference(H, W, y, reduction, upstream, dtype):
    Hr = H.detach().to(dtype).requires_grad_(True)
    Wr = W.detach().to(dtype).requires_grad_(True)
    loss = torch.nn.functional.cross_entropy(Hr @ Wr.T, y, reduction=reduction)
    (loss * upstream).sum().backward()
    return loss.detach(), Hr.grad, Wr.grad


@pytest.mark.parametrize("reduction", ["mean", "sum", "none"])
def test_bf16_loss_and_gradients(reduction):
    import linear_cross_entropy_bf16_b200 as flce
    N, V, D = 300, 5000, 128
    H, W, y = synth.random_inputs(N, V, D, seed=91)
    Hd = torch.from_numpy(H).view(torch.bfloat16).cuda().requires_grad_(True)
    Wd = torch.from_numpy(W).view(torch.bfloat16).cuda().requires_grad_(True)
    yd = torch.from_numpy(y).cuda()
    upstream = (torch.rand(N, device="cuda") + 0.5) if reduction == "none" else torch.tensor(1.7, device="cuda")
    loss = flce.linear_cross_entropy(Hd, Wd, yd, reduction=reduction)
    (loss * upstream).sum().backward()
    ref_loss, ref_dH, ref_dW = reference(Hd, Wd, yd, reduction, upstream, torch.float32)
    assert Hd.grad.dtype == torch.bfloat16 and Wd.grad.dtype == torch.bfloat16
    assert float((loss.detach().float() - ref_loss).abs().max()) <= 1e-3 * (N if reduction == "sum" else 1)
    assert rel(Hd.grad, ref_dH) < 1e-2 and rel(Wd.grad, ref_dW) < 1e-2


def test_fp32_gradients_match_fp64_reference():
    import linear_cross_entropy_bf16_b200 as flce
    N, V, D = 200, 3000, 72
    H, W, y = synth.random_inputs(N, V, D, seed=92, dtype="fp32")
    Hd = torch.from_numpy(H).cuda().requires_grad_(True)
    Wd = torch.from_numpy(W).cuda().requires_grad_(True)
    yd = torch.from_numpy(y).cuda()
    loss = flce.linear_cross_entropy(Hd, Wd, yd)
    loss.backward()
    ref_loss, ref_dH, ref_dW = reference(Hd, Wd, yd, "mean", torch.tensor(1.0, device="cuda"),
                                         torch.float64)
    assert abs(loss.item() - ref_loss.item()) <= 1e-5 * abs(ref_loss.item())
    assert rel(Hd.grad, ref_dH) < 1e-4 and rel(Wd.grad, ref_dW) < 1e-4


def test_frozen_head_gets_no_gradient():
    import linear_cross_entropy_bf16_b200 as flce
    N, V, D = 130, 2000, 64
    H, W, y = synth.random_inputs(N, V, D, seed=93)
    Hd = torch.from_numpy(H).view(torch.bfloat16).cuda().requires_grad_(True)
    Wd = torch.from_numpy(W).view(torch.bfloat16).cuda()
    flce.linear_cross_entropy(Hd, Wd, torch.from_numpy(y).cuda()).backward()
    assert Hd.grad is not None and Wd.grad is None


def test_quantized_head_gradient_for_H():
    import linear_cross_entropy_bf16_b200 as flce
    N, V, D, bits, G = 256, 4000, 128, 4, 64
    H, Wf, y = synth.random_inputs(N, V, D, seed=94, dtype="fp32")
    H = synth.round_to_bf16_bits(H)
    wq, sc, bi = synth.quantize_affine(Wf, bits, G)
    Wdq = torch.from_numpy(oracle.dequantize(wq, sc, bi, bits, G)).cuda()   # fp64 reference head
    Hd = torch.from_numpy(H).view(torch.bfloat16).cuda().requires_grad_(True)
    yd = torch.from_numpy(y).cuda()
    args = (torch.from_numpy(wq.view(np.int32)).cuda(), torch.from_numpy(sc).view(torch.bfloat16).cuda(),
            torch.from_numpy(bi).view(torch.bfloat16).cuda())
    loss = flce.linear_cross_entropy_quantized(Hd, *args, yd, bits, G)
    loss.backward()
    Hr = Hd.detach().double().requires_grad_(True)
    ref = torch.nn.functional.cross_entropy(Hr @ Wdq.T, yd)
    ref.backward()
    assert abs(loss.item() - ref.item()) <= 1e-5 * abs(ref.item())
    assert rel(Hd.grad, Hr.grad) < 1e-2


def test_int32_targets_and_strided_inputs():
    """int32 targets and a row-strided H (a slice of a wider activation) go through."""
    import linear_cross_entropy_bf16_b200 as flce
    N, V, D = 200, 3000, 64
    H, W, y = synth.random_inputs(N, V, D + 32, seed=95)
    Hwide = torch.from_numpy(H).view(torch.bfloat16).cuda().requires_grad_(True)
    Wd = torch.from_numpy(W).view(torch.bfloat16).cuda()[:, :D].contiguous().requires_grad_(True)
    y32 = torch.from_numpy(y).cuda().to(torch.int32)
    Hs = Hwide[:, 16:16 + D]                      # strided rows
    loss = flce.linear_cross_entropy(Hs, Wd, y32)
    loss.backward()
    ref_loss, ref_dH, ref_dW = reference(Hs, Wd, y32.long(), "mean", torch.tensor(1.0, device="cuda"),
                                         torch.float32)
    assert abs(loss.item() - ref_loss.item()) <= 1e-3
    assert Hwide.grad is not None and not Hwide.grad[:, :16].float().abs().any()
    assert rel(Hwide.grad[:, 16:16 + D], ref_dH) < 1e-2 and rel(Wd.grad, ref_dW) < 1e-2
