"""Quantization of weights held in pinned host memory (a checkpoint being
converted, weights offloaded to the host), with the transfers overlapped.

HostGroupedQuantizer splits a list of host tensors into chunks and runs every
chunk through three CUDA streams: host -> device copy, the grouped quantize
passes (nvfp4_quantize_grouped), device -> host copy of the codes, block
scales and tensor scales.  While chunk c is quantized, chunk c + 1 is being
copied in and chunk c - 1 copied out, so a run takes about the larger of the
two transfer times instead of their sum.  A tensor is never split: a dynamic
tensor scale needs the whole tensor.  Chunks are formed largest tensor first,
so that the copy-out of a large tensor overlaps the copy-in of the rest.

The kernels and their results are those of nvfp4_quantize_grouped; this
module only orders copies and launches.
"""
from __future__ import annotations

import torch

from . import binding as B


class HostGroupedQuantizer:
    """Quantize host tensors [rows, cols] (bf16 or f32, pinned) to NVFP4.

    passes: the quantize modes run in order on every chunk, the first of which
    must produce the scales (DYNAMIC, or FROZEN_GLOBAL with tensor_scales
    given); a later FROZEN_ALL pass re-encodes with the scales just computed.
    Results land in the pinned host tensors `codes` ([rows, cols / 2] uint8),
    `block_scales` ([rows, cols / 16] uint8, row-major E4M3) and
    `tensor_scales` ([n] float32) after run() has been waited for.
    """

    def __init__(self, host_xs, device, passes=(B.DYNAMIC,), tensor_scales=None,
                 chunk_bytes: int = 64 << 20):
        if not host_xs:
            raise ValueError("no tensors")
        for x in host_xs:
            if x.device.type != "cpu" or not x.is_pinned():
                raise ValueError("host tensors must be pinned CPU tensors")
            if x.dim() != 2 or x.shape[1] % 16 != 0:
                raise ValueError("each tensor must be [rows, cols] with cols a multiple of 16")
        if any(x.dtype != host_xs[0].dtype for x in host_xs):
            raise ValueError("all tensors must share a dtype (one grouped launch per chunk)")
        if not passes:
            raise ValueError("no quantize pass")
        if passes[0] == B.FROZEN_ALL:
            raise ValueError("the first pass must compute the block scales")
        if passes[0] == B.FROZEN_GLOBAL and tensor_scales is None:
            raise ValueError("FROZEN_GLOBAL needs tensor_scales")
        self.device = torch.device(device)
        self.passes = tuple(passes)
        self.host_xs = list(host_xs)
        n = len(self.host_xs)
        dev = self.device
        self.dx = [torch.empty(x.shape, dtype=x.dtype, device=dev) for x in self.host_xs]
        self.d_codes = [torch.empty(x.shape[0], x.shape[1] // 2, dtype=torch.uint8, device=dev) for x in self.host_xs]
        self.d_sb = [torch.empty(x.shape[0], x.shape[1] // 16, dtype=torch.uint8, device=dev) for x in self.host_xs]
        self.d_ts = torch.zeros(n, dtype=torch.float32, device=dev)
        if tensor_scales is not None:
            self.d_ts.copy_(torch.as_tensor(tensor_scales, dtype=torch.float32))
        self.codes = [torch.empty(c.shape, dtype=torch.uint8).pin_memory() for c in self.d_codes]
        self.block_scales = [torch.empty(s.shape, dtype=torch.uint8).pin_memory() for s in self.d_sb]
        self.tensor_scales = torch.empty(n, dtype=torch.float32).pin_memory()
        need = max(int(B.lib().nvfp4_grouped_workspace_size(m)) for m in self.passes)
        self.workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
        # chunks: indices, largest tensor first, each chunk up to chunk_bytes
        order = sorted(range(n), key=lambda i: -self.host_xs[i].numel() * self.host_xs[i].element_size())
        self.chunks = []
        cur, cur_bytes = [], 0
        for i in order:
            b = self.host_xs[i].numel() * self.host_xs[i].element_size()
            if cur and cur_bytes + b > chunk_bytes:
                self.chunks.append(cur)
                cur, cur_bytes = [], 0
            cur.append(i)
            cur_bytes += b
        if cur:
            self.chunks.append(cur)
        self.s_in = torch.cuda.Stream(dev)
        self.s_comp = torch.cuda.Stream(dev)
        self.s_out = torch.cuda.Stream(dev)
        nc = len(self.chunks)
        self.ev_in = [torch.cuda.Event() for _ in range(nc)]
        self.ev_comp = [torch.cuda.Event() for _ in range(nc)]
        # the device buffers are used on the side streams: when they are freed,
        # the caching allocator waits for the work queued there
        for t in [*self.dx, *self.d_codes, *self.d_sb, self.d_ts, self.workspace]:
            for st in (self.s_in, self.s_comp, self.s_out):
                t.record_stream(st)

    @property
    def h2d_bytes(self) -> int:
        return sum(x.numel() * x.element_size() for x in self.host_xs)

    @property
    def d2h_bytes(self) -> int:
        return sum(c.numel() for c in self.codes) + sum(s.numel() for s in self.block_scales) + 4 * len(self.host_xs)

    def run(self, stream=None):
        """Enqueue one pass over all tensors after the work already on
        `stream` (default: the current stream); `stream` then waits for all of
        it, so events recorded on `stream` around run() bracket the whole
        pass, and successive runs do not overlap."""
        caller = stream or torch.cuda.current_stream(self.device)
        start = torch.cuda.Event()
        start.record(caller)
        for s in (self.s_in, self.s_comp, self.s_out):
            s.wait_event(start)
        for c, idx in enumerate(self.chunks):
            with torch.cuda.stream(self.s_in):
                for i in idx:
                    self.dx[i].copy_(self.host_xs[i], non_blocking=True)
                self.ev_in[c].record(self.s_in)
            with torch.cuda.stream(self.s_comp):
                self.s_comp.wait_event(self.ev_in[c])
                xs = [self.dx[i] for i in idx]
                ts = [self.d_ts[i:i + 1] for i in idx]
                sbs = [self.d_sb[i] for i in idx]
                cds = [self.d_codes[i] for i in idx]
                for mode in self.passes:
                    B.nvfp4_quantize_grouped(xs, mode, tensor_scales=ts, block_scales=sbs, codes=cds,
                                             workspace=self.workspace)
                self.ev_comp[c].record(self.s_comp)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(self.ev_comp[c])
                for i in idx:
                    self.codes[i].copy_(self.d_codes[i], non_blocking=True)
                    self.block_scales[i].copy_(self.d_sb[i], non_blocking=True)
        with torch.cuda.stream(self.s_out):  # every chunk's kernels are done (s_comp is in order)
            self.tensor_scales.copy_(self.d_ts, non_blocking=True)
        caller.wait_stream(self.s_in)
        caller.wait_stream(self.s_comp)
        caller.wait_stream(self.s_out)
