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

* expert parallelism for the MoE layer (experts owned in contiguous blocks,
  rank r holding experts [r E/W, (r+1) E/W)): the routed (token, slot) rows
  travel to the rank that owns their expert and the expert outputs travel
  back, each way one all_to_all_single of the rows (plus one of the row
  counts); the backward pass runs the same two exchanges in reverse.  The
  pages train with expert parallelism (EP 4 and 8).  ExpertParallelMoE runs
  the whole layer step: the exchanges here, the experts' FFNs on the device
  (qad_moe_expert_forward / qad_moe_expert_backward).

The device operations are passed in (`ops`), defaulting to this package's
CUDA entry points; the collectives go through torch.distributed.  Beyond the
collectives, only data movement (row gathers and scatters, the weighted sum
over a token's slots) happens here.
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


# ------------------------------------------------------------------ expert parallelism


def _world(group=None) -> int:
    return dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1


@dataclass
class EpPlan:
    """Bookkeeping of one expert-parallel dispatch, reused by the combine and
    by both backward exchanges."""
    perm: torch.Tensor   # [tokens * topk] int64: (token, slot) pairs in send order
    send_counts: list    # rows sent to each rank
    recv_counts: list    # rows received from each rank
    tokens: int
    topk: int


def _exchange(out_rows: int, rows: torch.Tensor, out_splits, in_splits, group=None) -> torch.Tensor:
    out = rows.new_empty((out_rows,) + tuple(rows.shape[1:]))
    if _world(group) > 1:
        if rows.is_cuda and dist.get_backend(group) == "gloo":
            # gloo moves host memory only: stage the rows through the host
            host = torch.empty(out.shape, dtype=out.dtype)
            dist.all_to_all_single(host, rows.contiguous().cpu(), list(out_splits), list(in_splits), group=group)
            out.copy_(host)
        else:
            dist.all_to_all_single(out, rows.contiguous(), list(out_splits), list(in_splits), group=group)
    else:
        out.copy_(rows)
    return out


def ep_dispatch(x: torch.Tensor, ids: torch.Tensor, experts: int, group=None):
    """Send this rank's routed rows to the ranks that own their experts.

    x [tokens, H]; ids [tokens, topk] expert of each (token, slot).  Returns
    (recv_x [R, H], recv_expert [R] int32 -- the expert's index among the
    receiving rank's experts, plan).  Received rows are grouped by source rank
    (rank order) and, within a source, in (token, slot) order, so the result
    does not depend on timing."""
    world = _world(group)
    if experts % world:
        raise ValueError(f"{experts} experts do not split evenly over {world} ranks")
    per = experts // world
    tokens, topk = ids.shape
    flat = ids.reshape(-1).to(torch.int64)
    if flat.numel() and (int(flat.min()) < 0 or int(flat.max()) >= experts):
        raise ValueError("expert id out of range")
    owner = flat // per
    perm = torch.argsort(owner, stable=True)
    send_counts = torch.bincount(owner, minlength=world).to(torch.int64)
    recv_counts = _exchange(world, send_counts.view(world, 1), [1] * world, [1] * world, group).view(world)
    sc, rc = send_counts.tolist(), recv_counts.tolist()
    recv_x = _exchange(sum(rc), x[perm // topk], rc, sc, group)
    local_e = (flat[perm] - owner[perm] * per).to(torch.int32)
    recv_e = _exchange(sum(rc), local_e, rc, sc, group)
    return recv_x, recv_e, EpPlan(perm, sc, rc, tokens, topk)


def ep_combine(y_recv: torch.Tensor, plan: EpPlan, combine: torch.Tensor, group=None):
    """Return the expert outputs of the received rows to their tokens and sum
    them with the combine weights: y[t] = sum_j combine[t, j] * y_slot[t, j]
    (at least fp32, slots in order).  Returns (y [tokens, H], y_slot [tokens,
    topk, H] in y_recv's dtype -- kept for the backward pass)."""
    back = _exchange(plan.tokens * plan.topk, y_recv, plan.send_counts, plan.recv_counts, group)
    y_slot = torch.empty_like(back)
    y_slot[plan.perm] = back
    y_slot = y_slot.view(plan.tokens, plan.topk, -1)
    acc = torch.promote_types(y_slot.dtype, torch.float32)
    y = torch.zeros(plan.tokens, y_slot.shape[-1], dtype=acc, device=y_slot.device)
    for j in range(plan.topk):
        y += combine[:, j:j + 1].to(acc) * y_slot[:, j].to(acc)
    return y, y_slot


def ep_combine_backward(dy: torch.Tensor, plan: EpPlan, combine: torch.Tensor, y_slot: torch.Tensor, group=None):
    """Backward of ep_combine: d y_slot[t, j] = combine[t, j] * dy[t] goes to
    the expert owners (rows in the order the forward received them);
    d combine[t, j] = <dy[t], y_slot[t, j]> stays here.  Returns
    (dy_recv [R, H], d_combine [tokens, topk] at least fp32)."""
    acc = torch.promote_types(dy.dtype, torch.float32)
    d_slot = (combine.to(acc).unsqueeze(-1) * dy.to(acc).unsqueeze(1)).to(dy.dtype)
    rows = d_slot.reshape(plan.tokens * plan.topk, -1)[plan.perm]
    dy_recv = _exchange(sum(plan.recv_counts), rows, plan.recv_counts, plan.send_counts, group)
    d_combine = (dy.to(acc).unsqueeze(1) * y_slot.to(acc)).sum(-1)
    return dy_recv, d_combine


def ep_dispatch_backward(dx_recv: torch.Tensor, plan: EpPlan, group=None) -> torch.Tensor:
    """Backward of ep_dispatch: the input gradients of the received rows go
    back to their tokens and are summed over the token's slots (at least fp32,
    slots in order).  Returns dx [tokens, H]."""
    back = _exchange(plan.tokens * plan.topk, dx_recv, plan.send_counts, plan.recv_counts, group)
    per_slot = torch.empty_like(back)
    per_slot[plan.perm] = back
    per_slot = per_slot.view(plan.tokens, plan.topk, -1)
    acc = torch.promote_types(per_slot.dtype, torch.float32)
    dx = torch.zeros(plan.tokens, per_slot.shape[-1], dtype=acc, device=per_slot.device)
    for j in range(plan.topk):
        dx += per_slot[:, j].to(acc)
    return dx


class ExpertParallelMoE:
    """The QAD student's MoE layer step with expert parallelism over the ranks
    of `group` (EP 4 / 8 on the pages): rank r owns experts [r E/W, (r+1) E/W).

    forward: ep_dispatch sends each routed (token, slot) row to its expert's
    owner; the owner runs its experts' FFNs on the received rows on the device
    (qad_moe_expert_forward: grouped W4A4 with frozen scales, as in the
    single-GPU step); ep_combine returns the rows and sums them with the
    combine weights; the shared expert runs on each rank's own tokens (the
    same device path with one expert).  backward: the combine-weighted output
    gradients travel to the owners (ep_combine_backward), the owners run the
    straight-through backward of their experts (qad_moe_expert_backward: the
    rows' input gradients and their experts' weight gradients), the input
    gradients return and are summed over the token's slots
    (ep_dispatch_backward); the shared expert's weight gradient is summed over
    the ranks (all-reduce), since every rank computed it on its own tokens.

    local_weights / shared_weights: the qad_moe_weights tensors (as for
    MoeLayerStep) of this rank's E/W experts and of the shared expert alone.
    """

    def __init__(self, hidden: int, ffn: int, experts: int, local_weights: dict, shared_weights: dict, group=None,
                 device="cuda"):
        from .binding import MoeExpertStep

        self.group = group
        self.experts = experts
        self.hidden, self.ffn = hidden, ffn
        world = _world(group)
        if experts % world:
            raise ValueError(f"{experts} experts do not split evenly over {world} ranks")
        self.local = MoeExpertStep(hidden, ffn, experts // world, local_weights, device)
        self.shared = MoeExpertStep(hidden, ffn, 1, shared_weights, device)
        self._ctx = None

    def forward(self, x: torch.Tensor, ids: torch.Tensor, combine: torch.Tensor) -> torch.Tensor:
        """x [tokens, H] bf16 (this rank's tokens), ids / combine [tokens, topk]."""
        recv_x, recv_e, plan = ep_dispatch(x, ids, self.experts, self.group)
        y_recv = self.local.forward(recv_x, recv_e)
        y_routed, y_slot = ep_combine(y_recv, plan, combine, self.group)
        zero = torch.zeros(x.shape[0], dtype=torch.int32, device=x.device)
        y_shared = self.shared.forward(x, zero)
        self._ctx = (plan, combine, y_slot)
        return (y_routed + y_shared.to(y_routed.dtype)).to(x.dtype)

    def backward(self, dy: torch.Tensor):
        """Returns (dx [tokens, H], (dw_gate, dw_up, dw_down) of this rank's
        experts, (dw_gate, dw_up, dw_down) of the shared expert summed over the
        ranks, d_combine [tokens, topk])."""
        plan, combine, y_slot = self._ctx
        dy_recv, d_combine = ep_combine_backward(dy, plan, combine, y_slot, self.group)
        dx_recv, dwg, dwu, dwd = self.local.backward(dy_recv)
        dx_routed = ep_dispatch_backward(dx_recv, plan, self.group)
        dx_sh, sg, su, sd = self.shared.backward(dy)
        dx = (dx_routed + dx_sh.to(dx_routed.dtype)).to(dy.dtype)
        shared_dw = []
        for t in (sg, su, sd):
            acc = t.to(torch.promote_types(t.dtype, torch.float32))  # summed in at least fp32
            if _world(self.group) > 1:
                if acc.is_cuda and dist.get_backend(self.group) == "gloo":
                    host = acc.cpu()
                    dist.all_reduce(host, op=dist.ReduceOp.SUM, group=self.group)
                    acc.copy_(host)
                else:
                    dist.all_reduce(acc, op=dist.ReduceOp.SUM, group=self.group)
            shared_dw.append(acc.to(t.dtype))
        return dx, (dwg, dwu, dwd), tuple(shared_dw), d_combine
