"""MoE layer step of the QAD student, plain and slow -- TEST INFRASTRUCTURE ONLY.

Only the test suite, the smoke check and bench.py's CPU-baseline legs may
import this module; the product library never does.

The layer (Nemotron-3-Nano-30B NVFP4 article, "Was ist
Nemotron-Nano-3-30B-A3B-NVFP4?": routed experts plus one shared expert, a
few routed experts per token; Qwen3.6-35B-A3B W4A4 tutorial, "2. PTQ":
expert weights and activations NVFP4, W4A4; Nemotron 3.5 Lightning NVFP4
article, "量化尺度处理策略": frozen scales, the weights trained through
simulated quantization):

    y_t = sum_j w_tj E_{e_tj}(x_t) + E_shared(x_t)
    E(x) = Q(a) W^_down^T,   a = silu(h_gate) * h_up,
    h_gate = Q(x) W^_gate^T, h_up = Q(x) W^_up^T,   silu(g) = g / (1 + e^-g)

Q is NVFP4 quantization with frozen scales (weights: tensor and block
scales given; activations: tensor scale given, block scales from the data),
computed by the pinned scalar oracle in nvfp4_oracle.c.  The forward GEMMs
are the oracle's exact W4A4 GEMM (float64 sums of exact products).

Readings where the pages leave the step open:
  * storage precision: h_gate, h_up, a, the expert outputs, y and every
    gradient are bf16 tensors (the model's dtype), each rounded once (RNE)
    from the float64 value; a is rounded to bf16 before it is quantized;
  * backward: straight-through estimator, dQ(v)/dv = identity; gradients
    are float64 products of the bf16 dequantized operands the forward used
    (W^ and X^, A^ as bf16 fake-quant outputs), rounded to bf16;
  * d(combine weight) = <dy_t, y_expert(t)> with y_expert the bf16 output.

Every function takes the parameters in float64 (weights: float32 or
float64) numpy arrays holding exact copies of the bf16 inputs.  `quantized=False, rounded=False` replaces Q by
the identity and skips the bf16 roundings: the smooth layer, whose exact
gradient the straight-through backward must reproduce (pinned by finite
differences in the tests).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import (FROZEN_ALL, FROZEN_GLOBAL, bf16_bits_to_f32, bf16_round, dequantize, fake_quant,
               gemm_w4a4, quantize)


def silu(g: np.ndarray) -> np.ndarray:
    return g / (1.0 + np.exp(-g))


def silu_grad(g: np.ndarray) -> np.ndarray:
    """d silu / dg = s (1 + g (1 - s)), s = sigmoid(g)."""
    s = 1.0 / (1.0 + np.exp(-g))
    return s * (1.0 + g * (1.0 - s))


def to_bf16(v: np.ndarray) -> np.ndarray:
    """float64 -> nearest bf16 value (RNE), as float64."""
    return bf16_bits_to_f32(bf16_round(v)).astype(np.float64)


@dataclass
class Layer:
    """Inputs of one layer step (group g < E routed expert g, g = E shared)."""
    x: np.ndarray            # [T, H]
    ids: np.ndarray          # int [T, k]
    cw: np.ndarray           # [T, k] combine weights
    w_gate: np.ndarray       # [G, F, H]
    w_up: np.ndarray         # [G, F, H]
    w_down: np.ndarray       # [G, H, F]
    gate_ts: np.ndarray      # [G] frozen tensor scales
    up_ts: np.ndarray
    down_ts: np.ndarray
    gate_sb: np.ndarray      # uint8 [G, F, H/16] frozen block scales
    up_sb: np.ndarray
    down_sb: np.ndarray      # uint8 [G, H, F/16]
    x_ts: np.ndarray         # [G] frozen tensor scale of x per group
    a_ts: np.ndarray         # [G] frozen tensor scale of a per group
    _wq: dict = field(default_factory=dict, repr=False)

    @property
    def experts(self) -> int:
        return self.w_gate.shape[0] - 1

    def forget_quantized_weights(self) -> None:
        """Drop the cached weight quantizations (after changing a weight)."""
        self._wq.clear()

    def weight(self, kind: str, g: int):
        """Codes, block scales, tensor scale and bf16 fake-quant value of one
        expert weight (FROZEN_ALL quantization of the master weight)."""
        key = (kind, g)
        if key not in self._wq:
            w = getattr(self, "w_" + kind)[g].astype(np.float32)
            ts = float(getattr(self, kind + "_ts")[g])
            sb = getattr(self, kind + "_sb")[g]
            codes, sb_out, _ = quantize(w, FROZEN_ALL, s_g=ts, s_b=sb)
            _, bits, _, _ = fake_quant(w, FROZEN_ALL, s_g=ts, s_b=sb)
            self._wq[key] = (codes, sb_out, ts, bf16_bits_to_f32(bits).astype(np.float64))
        return self._wq[key]


def route(ids: np.ndarray, experts: int):
    """Per group, the (token, slot) pairs routed to it in increasing token
    order (slot None for the shared expert, which takes every token)."""
    T = ids.shape[0]
    out = []
    for e in range(experts):
        t, j = np.nonzero(ids == e)  # row-major scan: increasing token, then slot
        out.append((t, j))
    out.append((np.arange(T), None))
    return out


def expert_forward(L: Layer, g: int, xr: np.ndarray, quantized: bool = True, rounded: bool = True):
    """Forward of group g on rows xr [n, H]; returns the intermediates."""
    rnd = to_bf16 if rounded else (lambda v: v)
    H = xr.shape[1]
    F = L.w_gate.shape[1]
    st = {}
    if quantized:
        xc, xsb, _ = quantize(xr.astype(np.float32), FROZEN_GLOBAL, s_g=float(L.x_ts[g]))
        xf, xbits = dequantize(xc, xsb, float(L.x_ts[g]), H)
        st["x_codes"], st["x_sb"] = xc, xsb
        st["x_hat"] = bf16_bits_to_f32(xbits).astype(np.float64)
        hg = gemm_w4a4(xc, xsb, float(L.x_ts[g]), *L.weight("gate", g)[:3], H)
        hu = gemm_w4a4(xc, xsb, float(L.x_ts[g]), *L.weight("up", g)[:3], H)
    else:
        st["x_hat"] = xr
        hg = xr @ L.w_gate[g].astype(np.float64).T
        hu = xr @ L.w_up[g].astype(np.float64).T
    st["h_gate"], st["h_up"] = rnd(hg), rnd(hu)
    a = rnd(silu(st["h_gate"]) * st["h_up"])
    st["a"] = a
    if quantized:
        ac, asb, _ = quantize(a.astype(np.float32), FROZEN_GLOBAL, s_g=float(L.a_ts[g]))
        _, abits = dequantize(ac, asb, float(L.a_ts[g]), F)
        st["a_codes"], st["a_sb"] = ac, asb
        st["a_hat"] = bf16_bits_to_f32(abits).astype(np.float64)
        y = gemm_w4a4(ac, asb, float(L.a_ts[g]), *L.weight("down", g)[:3], F)
    else:
        st["a_hat"] = a
        y = a @ L.w_down[g].astype(np.float64).T
    st["y"] = rnd(y)
    return st


def expert_backward(L: Layer, g: int, st: dict, dyp: np.ndarray, quantized: bool = True, rounded: bool = True):
    """Straight-through backward of group g given dY of its rows (already
    multiplied by the combine weights and rounded): returns dA, [dG | dU],
    dX of the rows and the weight gradients."""
    rnd = to_bf16 if rounded else (lambda v: v)
    if quantized:
        wg, wu, wd = L.weight("gate", g)[3], L.weight("up", g)[3], L.weight("down", g)[3]
    else:
        wg, wu, wd = (w[g].astype(np.float64) for w in (L.w_gate, L.w_up, L.w_down))
    da = rnd(dyp @ wd)                                     # [n, F]
    hg, hu = st["h_gate"], st["h_up"]
    dg = rnd(da * hu * silu_grad(hg))
    du = rnd(da * silu(hg))
    dx = rnd(dg @ wg + du @ wu)                            # [n, H]
    return {
        "dA": da, "dG": dg, "dU": du, "dX": dx,
        "dW_down": rnd(dyp.T @ st["a_hat"]),               # [H, F]
        "dW_gate": rnd(dg.T @ st["x_hat"]),                # [F, H]
        "dW_up": rnd(du.T @ st["x_hat"]),
    }


def layer_step(L: Layer, dy: np.ndarray | None, quantized: bool = True, rounded: bool = True,
               groups=None):
    """Forward (and backward when dy is given) of the whole layer.

    groups: if given, only these groups are computed (the outputs then hold
    only their contributions); for sampled checks of large layers.
    Returns a dict with y, dx, d_combine, and per group the forward state,
    the backward results and the token/slot lists."""
    rnd = to_bf16 if rounded else (lambda v: v)
    T, H = L.x.shape
    E = L.experts
    segs = route(L.ids, E)
    y_acc = np.zeros((T, H))
    dx_acc = np.zeros((T, H))
    d_cw = np.zeros(L.cw.shape)
    per = {}
    todo = range(E + 1) if groups is None else groups
    routed_y = {}
    for g in todo:
        t, j = segs[g]
        if len(t) == 0:
            per[g] = {"tokens": t, "slots": j, "fwd": None, "bwd": None}
            continue
        st = expert_forward(L, g, L.x[t], quantized, rounded)
        w = L.cw[t, j] if j is not None else np.ones(len(t))
        routed_y[g] = st["y"]
        bwd = None
        if dy is not None:
            dyp = rnd(w[:, None] * dy[t])
            bwd = expert_backward(L, g, st, dyp, quantized, rounded)
            bwd["dY"] = dyp
            dx_acc[t] += bwd["dX"]
            if j is not None:
                d_cw[t, j] = np.einsum("nh,nh->n", dy[t], st["y"])
        y_acc[t] += w[:, None] * st["y"]
        per[g] = {"tokens": t, "slots": j, "fwd": st, "bwd": bwd}
    out = {"y": rnd(y_acc), "groups": per, "segments": segs}
    if dy is not None:
        out["dx"] = rnd(dx_acc)
        out["d_combine"] = d_cw
    return out


def combine_rows(y: np.ndarray, slot_row: np.ndarray, weights: np.ndarray, shared_base: int) -> np.ndarray:
    """The layer output from its permuted expert rows: token t's output is
    sum_j w[t, j] y[slot_row[t, j]] + y[shared_base + t] (a slot routed
    nowhere, slot_row -1, contributes nothing), summed in float64 and
    rounded to bf16 once -- the combine of y_t = sum_j w_tj E_{e_tj}(x_t) +
    E_shared(x_t) written over the row buffer of the expert outputs."""
    T, k = slot_row.shape
    out = np.zeros((T, y.shape[1]))
    for t in range(T):
        for j in range(k):
            r = int(slot_row[t, j])
            if r >= 0:
                out[t] += float(weights[t, j]) * y[r]
        out[t] += y[shared_base + t]
    return to_bf16(out)


def gather_sum_rows(dxp: np.ndarray, slot_row: np.ndarray, shared_base: int) -> np.ndarray:
    """dx of each token from the permuted rows' input gradients:
    sum_j dxp[slot_row[t, j]] + dxp[shared_base + t], float64, rounded to bf16."""
    return combine_rows(dxp, slot_row, np.ones(slot_row.shape), shared_base)
