"""MoE test cases shared by the oracle pins and the GPU parity tests.

Builds the oracle's Layer from a synthetic layer (host tensors): the frozen
weight scales come from the oracle's own DYNAMIC quantization of the
calibration weights, per group, so nothing here comes from the CUDA path.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
from oracle import moe as OM


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def f32(t: torch.Tensor) -> np.ndarray:
    """Exact float32 copy of a bf16 tensor (half the host memory of f64)."""
    return t.detach().float().cpu().numpy()


def remap_unused(ids: torch.Tensor, unused: int, experts: int) -> torch.Tensor:
    """Reroutes every assignment to expert `unused` to another expert the token
    has not chosen, so that group `unused` receives no token."""
    ids = ids.clone()
    for t in range(ids.shape[0]):
        row = ids[t].tolist()
        for j, e in enumerate(row):
            if e == unused:
                alt = next(c for c in range(experts) if c != unused and c not in row)
                row[j] = alt
        ids[t] = torch.tensor(row, dtype=ids.dtype)
    return ids


def oracle_frozen_weight_scales(w0: torch.Tensor, groups=None):
    """Per group: (tensor scale, block scales) of the oracle's DYNAMIC
    quantization of the calibration weight w0[g]."""
    G = w0.shape[0]
    rows, cols = w0.shape[1], w0.shape[2]
    ts = np.zeros(G, np.float32)
    sb = np.zeros((G, rows, cols // 16), np.uint8)
    for g in (range(G) if groups is None else groups):
        _, s, t = O.quantize(w0[g].float().cpu().numpy(), O.DYNAMIC)
        ts[g], sb[g] = t, s
    return ts, sb


def oracle_layer(d: dict, groups=None) -> OM.Layer:
    """oracle Layer of a synthetic MoE layer (host tensors); with `groups`,
    frozen weight scales only for those groups."""
    scales = {k: oracle_frozen_weight_scales(d["w0_" + k], groups) for k in ("gate", "up", "down")}
    return OM.Layer(
        x=f64(d["x"]), ids=d["ids"].cpu().numpy().astype(np.int64), cw=f64(d["combine"]),
        w_gate=f32(d["w_gate"]), w_up=f32(d["w_up"]), w_down=f32(d["w_down"]),
        gate_ts=scales["gate"][0], up_ts=scales["up"][0], down_ts=scales["down"][0],
        gate_sb=scales["gate"][1], up_sb=scales["up"][1], down_sb=scales["down"][1],
        x_ts=d["x_ts"].cpu().numpy(), a_ts=d["a_ts"].cpu().numpy())
