"""nvfp4_quantization_aware_b200 -- B200 (sm_100a) hot path of NVFP4
quantization-aware distillation.

The compute lives in ``libnvfp4qad.so`` (hand-written CUDA for sm_100a, C ABI
declared in ``include/nvfp4qad.h``).  This package is the thin Python side:

* ``nvfp4_quantize``, ``nvfp4_fake_quant``, ``nvfp4_dequantize``,
  ``nvfp4_gemm_w4a4``, ``qad_kl_fwd_bwd``, ``nvfp4_gemm_bf16_grouped`` and the
  MoE layer step (``MoeLayerStep`` over ``qad_moe_forward`` /
  ``qad_moe_backward``) -- the C entry points under the
  same names, taking torch tensors and marshalling pointers, sizes and the
  current CUDA stream (nothing is computed in Python);
* ``FakeQuantSTE`` and ``KLDistillLoss`` -- autograd wiring: straight-through
  gradient for fake quantization, stored dLogits for the KL loss.

There is no CPU fallback: if the library is missing or the tensors are not on
a CUDA device, the call raises.
"""
from .binding import (  # noqa: F401
    BF16,
    DYNAMIC,
    F32,
    FROZEN_ALL,
    FROZEN_GLOBAL,
    NVFP4Error,
    SCALES_MMA,
    SCALES_ROWMAJOR,
    lib,
    library_path,
    mma_scales_bytes,
    nvfp4_dequantize,
    nvfp4_device_error,
    nvfp4_fault_inject,
    nvfp4_selftest_timeout,
    nvfp4_fake_quant,
    nvfp4_fake_quant_grouped,
    nvfp4_launch_count,
    nvfp4_quantize_grouped,
    TensorRef,
    nvfp4_gemm_w4a4,
    nvfp4_gemm_w4a4_grouped,
    nvfp4_gemm_bf16_grouped,
    nvfp4_gemm_w4a16,
    nvfp4_probe_fp4_mma,
    nvfp4_scales_to_mma,
    nvfp4_quantize_fake_quant_grouped,
    MoeLayerStep,
    MoeExpertStep,
    MOE_BUFFERS,
    nvfp4_quantize,
    nvfp4_selftest_division,
    qad_kl_fwd_bwd,
    qad_kl_topk_fwd_bwd,
    qad_kl_topp_fwd_bwd,
    nvfp4_calibrate_mse,
    nvfp4_calibrate_mse_grouped,
)
from .autograd import FakeQuantSTE, KLDistillLoss, fake_quant_ste, kl_distill_loss  # noqa: F401
from .hostio import HostGroupedQuantizer  # noqa: F401
