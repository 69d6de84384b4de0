"""Autograd wiring of the QAD student step.

* FakeQuantSTE: forward is the library's fake quantization (simulated NVFP4
  quantization of the student's weights and activations, Nemotron 3.5
  Lightning NVFP4 article, "QAD的工作原理"); backward is the straight-through
  estimator, the identity dx = dy, including saturated elements.
* KLDistillLoss: forward computes KL(p_teacher || p_student) and, in the same
  pass over the logits, dLogits w.r.t. the student; backward multiplies the
  stored dLogits by the incoming scalar gradient.
"""
from __future__ import annotations

import torch

from . import binding as B


class FakeQuantSTE(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, mode=B.DYNAMIC, tensor_scale=None, block_scales=None):
        shape = x.shape
        x2 = x.reshape(-1, shape[-1])
        if x2.stride(1) != 1:
            x2 = x2.contiguous()
        y = B.nvfp4_fake_quant(x2, mode=mode, tensor_scale=tensor_scale, block_scales=block_scales)
        return y.reshape(shape)

    @staticmethod
    def backward(ctx, dy):
        return dy, None, None, None


def fake_quant_ste(x, mode=B.DYNAMIC, tensor_scale=None, block_scales=None):
    return FakeQuantSTE.apply(x, mode, tensor_scale, block_scales)


class KLDistillLoss(torch.autograd.Function):
    @staticmethod
    def forward(ctx, student, teacher, temperature=1.0):
        loss, _, grad = B.qad_kl_fwd_bwd(teacher.detach(), student.detach(), temperature=temperature,
                                         want_grad=student.requires_grad)
        ctx.save_for_backward(grad if grad is not None else torch.empty(0, device=student.device))
        return loss[0]

    @staticmethod
    def backward(ctx, dloss):
        (grad,) = ctx.saved_tensors
        if grad.numel() == 0:
            return None, None, None
        return grad * dloss.to(grad.dtype), None, None


def kl_distill_loss(student, teacher, temperature=1.0):
    return KLDistillLoss.apply(student, teacher, temperature)
