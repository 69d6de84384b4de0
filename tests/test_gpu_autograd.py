"""The autograd wiring of the student's simulated quantization.

FakeQuantSTE: its forward equals oracle.fake_quant bit for bit in every scale
mode (including a 3-D input, which is quantized along its last dimension),
and its backward is the straight-through estimator: dx = dy exactly, also on
elements that the quantizer saturated (Nemotron 3.5 Lightning NVFP4 article,
"QAD的工作原理": the student's forward runs through simulated quantization
and is trained through it).
"""
import numpy as np
import pytest
import torch

import oracle as O
import nvfp4_quantization_aware_b200 as Q
from nvfp4_quantization_aware_b200 import synthetic as S

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _oracle_fq_bits(x: torch.Tensor, mode, s_g=None, s_b=None) -> np.ndarray:
    x2 = x.reshape(-1, x.shape[-1]).float().cpu().numpy()
    _, bits, _, _ = O.fake_quant(x2, mode, s_g=s_g, s_b=s_b)
    return bits.reshape(x.shape)


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("mode", ["dynamic", "frozen_global", "frozen_all"])
def test_fake_quant_ste_forward_and_backward(mode):
    x = S.channel_scaled_activations(96, 512, seed=21, device=DEV).reshape(4, 24, 512)
    x.requires_grad_(True)
    if mode == "dynamic":
        args, ref = (Q.DYNAMIC,), _oracle_fq_bits(x.detach(), O.DYNAMIC)
    elif mode == "frozen_global":
        # a tensor scale far below amax / 2688: most blocks saturate at +-6 d
        sg = float(x.detach().abs().max()) / 2688.0 / 64.0
        ts = torch.tensor([sg], dtype=torch.float32, device=DEV)
        args, ref = (Q.FROZEN_GLOBAL, ts), _oracle_fq_bits(x.detach(), O.FROZEN_GLOBAL, s_g=float(ts[0]))
    else:
        x2 = x.detach().reshape(-1, 512).float().cpu().numpy()
        _, sb, sg = O.quantize(x2, O.DYNAMIC)
        sb = (sb // 2).astype(np.uint8)  # smaller block scales than amax gives: saturation again
        ts = torch.tensor([sg], dtype=torch.float32, device=DEV)
        args = (Q.FROZEN_ALL, ts, torch.from_numpy(sb).to(DEV))
        ref = _oracle_fq_bits(x.detach(), O.FROZEN_ALL, s_g=sg, s_b=sb)
    y = Q.fake_quant_ste(x, *args)
    assert y.shape == x.shape and y.dtype == x.dtype
    assert np.array_equal(_bits(y.detach()), ref)
    dy = torch.randn(x.shape, generator=torch.Generator(device=DEV).manual_seed(5), device=DEV).to(x.dtype)
    y.backward(dy)
    assert torch.equal(x.grad, dy)
    if mode != "dynamic":
        # elements the quantizer clipped (|x| / d beyond 6) or rounded down:
        # the straight-through gradient passes dy unchanged there as well
        yf = y.detach().float()
        sat = (x.detach().float().abs() > yf.abs() * 1.0001) & (yf != 0)
        assert int(sat.sum()) > 1000
        assert torch.equal(x.grad[sat], dy[sat])


def test_fake_quant_ste_inside_a_graph_of_ops():
    """Gradients flow through the STE as through the identity: for
    loss = sum(c * fq(w)), d loss / d w = c exactly."""
    w = S.weights(64, 256, seed=4, device=DEV).requires_grad_(True)
    c = torch.randn(64, 256, generator=torch.Generator(device=DEV).manual_seed(1), device=DEV).to(torch.bfloat16)
    (Q.fake_quant_ste(w) * c).float().sum().backward()
    assert torch.equal(w.grad, c)
