"""Row-sharded NVFP4 quantization and KL loss over several GPUs.

One process per GPU (torch.distributed over NCCL).  The path partitions by
rows; the only data exchanged are scalars:

* dynamic-scale quantization of a tensor whose rows are spread over the
  ranks: each rank takes the max |x| of its rows (nvfp4_tensor_amax_grouped),
  one all-reduce(max) of one float per tensor combines them, every rank
  derives the same s_g = amax / 2688 (nvfp4_global_scale_from_amax) and
  quantizes its rows with that frozen global scale (FROZEN_GLOBAL): codes
  and block scales equal those of a DYNAMIC call on the whole tensor, since
  the block scales depend only on a block and s_g;
* the KL loss over rows spread over the ranks: each rank runs the fused
  kernel on its rows with grad_scale = 1 / (all rows), so its dLogits are
  already those of the global mean, and one all-reduce(sum) of the ranks'
  partial sums gives the loss.

The device operations are passed in (`ops`), defaulting to this package's
CUDA entry points; the collectives go through torch.distributed.  No
arithmetic on tensors happens here beyond the scalar mean.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable

import torch
import torch.distributed as dist


@dataclass
class ShardOps:
    """Device operations used by the sharded helpers."""
    tensor_amax: Callable        # (list of tensors) -> float32 [n] max |x| per tensor
    scale_from_amax: Callable    # (amax [n]) -> float32 [n] s_g
    quantize_frozen_global: Callable  # (list of tensors, s_g [n]) -> (codes list, block scales list)
    kl: Callable                 # (teacher, student, T, grad_scale) -> (row_kl [rows], dlogits)


def cuda_ops() -> ShardOps:
    from . import binding as B

    def tensor_amax(xs):
        n = len(xs)
        dev = xs[0].device
        out = torch.empty(n, dtype=torch.float32, device=dev)
        arr = (B.TensorRef * n)()
        for i, x in enumerate(xs):
            B._cuda2d(x, f"tensor {i}")
            arr[i] = B.TensorRef(x.data_ptr(), x.shape[0], x.shape[1], x.stride(0), None, None, None, 0)
        B._check(B.lib().nvfp4_tensor_amax_grouped(n, arr, B._dtype_code(xs[0]), out.data_ptr(), B._stream(dev)),
                 "nvfp4_tensor_amax_grouped")
        return out

    def scale_from_amax(amax):
        ts = torch.empty_like(amax)
        B._check(B.lib().nvfp4_global_scale_from_amax(amax.data_ptr(), amax.numel(), ts.data_ptr(),
                                                      B._stream(amax.device)), "nvfp4_global_scale_from_amax")
        return ts

    def quantize_frozen_global(xs, ts):
        codes, sbs, _ = B.nvfp4_quantize_grouped(xs, B.FROZEN_GLOBAL, tensor_scales=ts)
        return codes, sbs

    def kl(teacher, student, T, grad_scale):
        _, row_kl, g = B.qad_kl_fwd_bwd(teacher, student, temperature=T, grad_scale=grad_scale, want_row_kl=True)
        return row_kl, g

    return ShardOps(tensor_amax, scale_from_amax, quantize_frozen_global, kl)


def sharded_dynamic_quantize(shards, ops: ShardOps | None = None, group=None):
    """Dynamic-scale quantization of tensors whose rows are split over the
    ranks of `group`: `shards` holds this rank's rows of each tensor.
    Returns (codes list, block scales list, s_g [n]) -- the same on every rank
    for s_g, and for codes/scales equal to the whole-tensor DYNAMIC result
    restricted to this rank's rows."""
    ops = ops or cuda_ops()
    amax = ops.tensor_amax(shards)
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    ts = ops.scale_from_amax(amax)
    codes, sbs = ops.quantize_frozen_global(shards, ts)
    return codes, sbs, ts


def sharded_kl(teacher, student, total_rows: int, T: float = 1.0, ops: ShardOps | None = None, group=None):
    """KL distillation loss over rows split across the ranks: returns (loss of
    all rows, this rank's per-row KL, this rank's dLogits of the global mean)."""
    ops = ops or cuda_ops()
    row_kl, g = ops.kl(teacher, student, T, 1.0 / total_rows)
    part = row_kl.double().sum().reshape(1)
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(part, op=dist.ReduceOp.SUM, group=group)
    return part / total_rows, row_kl, g
