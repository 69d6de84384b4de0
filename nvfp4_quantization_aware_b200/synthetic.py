"""Seeded synthetic workloads shaped like the linear layers and logits of a QAD
student step.  Holds no NVFP4 or KL arithmetic: it only draws tensors.

Both the CUDA path and the CPU oracle are fed from these generators (the
oracle receives host copies of exactly the same bits), so this module is the
one thing the two sides share.

Distributions ("N(mu, sigma)" is mean and standard deviation):

* activations:            bf16 N(0, 1)
* weights:                bf16 N(0, 0.02), a Bernoulli(p) subset multiplied by
                          an outlier factor (p = 0.5 %, x30 for the tiny linear;
                          p = 0.1 %, x50 for MoE expert / lm_head weights)
* channel-scaled acts:    N(0, 1) * c_k with c_k ~ LogNormal(0, 1) per K-channel
* logits (tiny):          teacher fp32 N(0, 4), student = teacher + N(0, 0.5)
* logits (vocabulary):    teacher bf16 N(0, 3) with one uniformly drawn entry per
                          row raised by +12, student = teacher + N(0, 1)
* routing:                per token, 6 distinct experts of 128 drawn uniformly;
                          combine weights softmax of N(0, 1) router logits over
                          the 6; the shared expert has weight 1.

Shapes follow the pages' workloads: MoE layers with 128 routed experts plus one
shared expert and top-6 routing, a hidden size of 2048 with expert FFN width
1024, a 131072-entry vocabulary head and 4096-wide dense linears.
"""
from __future__ import annotations

import torch

BF16 = torch.bfloat16
F32 = torch.float32


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def activations(rows: int, cols: int, seed: int, device="cpu", dtype=BF16) -> torch.Tensor:
    g = _gen(seed, device)
    return torch.randn(rows, cols, generator=g, device=device, dtype=F32).to(dtype)


def weights(rows: int, cols: int, seed: int, device="cpu", std: float = 0.02,
            outlier_p: float = 0.001, outlier_mult: float = 50.0, dtype=BF16) -> torch.Tensor:
    g = _gen(seed, device)
    w = torch.randn(rows, cols, generator=g, device=device, dtype=F32) * std
    mask = torch.rand(rows, cols, generator=g, device=device, dtype=F32) < outlier_p
    w = torch.where(mask, w * outlier_mult, w)
    return w.to(dtype)


def channel_scaled_activations(rows: int, cols: int, seed: int, device="cpu", dtype=BF16) -> torch.Tensor:
    g = _gen(seed, device)
    c = torch.exp(torch.randn(cols, generator=g, device=device, dtype=F32))
    x = torch.randn(rows, cols, generator=g, device=device, dtype=F32) * c
    return x.to(dtype)


def logits_pair(rows: int, vocab: int, seed: int, device="cpu", teacher_std: float = 3.0,
                noise_std: float = 1.0, boost: float | None = 12.0, dtype=BF16,
                chunk_rows: int = 1024):
    """Teacher/student logits.  Generated in row chunks so that the fp32
    intermediates of a 16384 x 131072 pair stay small; chunk c uses seed
    seed * 1_000_003 + c."""
    t = torch.empty(rows, vocab, device=device, dtype=dtype)
    s = torch.empty(rows, vocab, device=device, dtype=dtype)
    for c, r0 in enumerate(range(0, rows, chunk_rows)):
        r1 = min(rows, r0 + chunk_rows)
        g = _gen(int(seed) * 1_000_003 + c, device)
        tt = torch.randn(r1 - r0, vocab, generator=g, device=device, dtype=F32) * teacher_std
        if boost is not None:
            idx = torch.randint(0, vocab, (r1 - r0,), generator=g, device=device)
            tt[torch.arange(r1 - r0, device=device), idx] += boost
        tt = tt.to(dtype)
        ss = tt.to(F32) + torch.randn(r1 - r0, vocab, generator=g, device=device, dtype=F32) * noise_std
        t[r0:r1] = tt
        s[r0:r1] = ss.to(dtype)
    return t, s


def routing(tokens: int, experts: int, topk: int, seed: int, device="cpu"):
    """Uniform top-k routing: returns (expert ids int32 [tokens, topk], combine
    weights fp32 [tokens, topk])."""
    g = _gen(seed, device)
    keys = torch.rand(tokens, experts, generator=g, device=device, dtype=F32)
    ids = torch.topk(keys, topk, dim=1).indices.to(torch.int32)
    logits = torch.randn(tokens, topk, generator=g, device=device, dtype=F32)
    w = torch.softmax(logits, dim=1)
    return ids, w


# --------------------------------------------------------------------------
# the five workloads
# --------------------------------------------------------------------------

def tiny_qad_linear(seed: int = 0, device="cpu"):
    """X 64x1024 bf16, W 1024x1024 bf16 (0.5 % outliers x30), fp32 logits
    64x8192 (teacher N(0,4), student = teacher + N(0,0.5))."""
    x = activations(64, 1024, seed, device)
    w = weights(1024, 1024, seed + 1, device, outlier_p=0.005, outlier_mult=30.0)
    t, s = logits_pair(64, 8192, seed + 2, device, teacher_std=4.0, noise_std=0.5, boost=None, dtype=F32)
    return {"x": x, "w": w, "teacher": t, "student": s, "T": 1.0}


MOE_EXPERTS = 128
EXPERT_SHAPE = (2048, 1024)
LM_HEAD_SHAPE = (131072, 2048)


def weight_sweep(seed: int = 0, device="cpu", experts: int = MOE_EXPERTS, lm_head: bool = True,
                 expert_shape=EXPERT_SHAPE, lm_head_shape=LM_HEAD_SHAPE):
    """128 expert weights 2048x1024 and one lm_head 131072x2048, bf16
    N(0, 0.02) with 0.1 % outliers x50.  Tensor i uses seed + i."""
    ws = [weights(*expert_shape, seed + i, device) for i in range(experts)]
    if lm_head:
        ws.append(weights(*lm_head_shape, seed + experts, device))
    return ws


def w4a4_gemm(M: int, seed: int = 0, device="cpu", N: int = 4096, K: int = 4096):
    """Activations M x K with per-channel LogNormal scales, weights N x K from
    the expert/lm_head weight generator."""
    x = channel_scaled_activations(M, K, seed, device)
    w = weights(N, K, seed + 1, device)
    return {"x": x, "w": w}


def distill_logits(seed: int = 0, device="cpu", rows: int = 16384, vocab: int = 131072):
    t, s = logits_pair(rows, vocab, seed, device)
    return {"teacher": t, "student": s, "T": 1.0}


def moe_layer(seed: int = 0, device="cpu", tokens: int = 4096, hidden: int = 2048, ffn: int = 1024,
              experts: int = MOE_EXPERTS, topk: int = 6, drift: float = 0.1, w_std: float = 0.02):
    """One MoE layer step: x [tokens, hidden]; for every group g (routed
    experts 0..experts-1, then the shared expert) gate/up weights
    [ffn, hidden] and a down weight [hidden, ffn], stacked along dim 0;
    routing ids/weights; the gradient dy of the layer output.

    Frozen-scale inputs:
      * w0_gate / w0_up / w0_down: the weights at calibration time (the
        frozen weight scales are taken from them); the step's master weights
        are w = w0 + N(0, drift * w_std), i.e. a student that has trained for a
        while, so a few blocks leave their frozen range;
      * x_ts, a_ts [experts + 1] fp32: seeded stand-ins for calibrated
        activation tensor scales.  x_ts ~ U(1.49e-3, 1.86e-3) puts the largest
        representable magnitude at 4 to 5 standard deviations of x ~ N(0, 1);
        a_ts ~ U(0.9, 1.1) * 5.36e-3 * hidden * E[w^2], the same for the
        SwiGLU output (about (4 sigma_h)^2 with sigma_h^2 = hidden * E[w^2])."""
    x = activations(tokens, hidden, seed, device)
    ids, cw = routing(tokens, experts, topk, seed + 1, device)
    n = experts + 1
    out = {"x": x, "ids": ids, "combine": cw, "dy": activations(tokens, hidden, seed + 2, device)}
    for k, (rows, cols, off) in {"gate": (ffn, hidden, 10), "up": (ffn, hidden, 11),
                                 "down": (hidden, ffn, 12)}.items():
        w0 = torch.stack([weights(rows, cols, seed + off + 3 * e, device, std=w_std) for e in range(n)])
        g = _gen(seed + 7 + off, device)
        noise = torch.randn(w0.shape, generator=g, device=device, dtype=F32) * (drift * w_std)
        out["w0_" + k] = w0
        out["w_" + k] = (w0.to(F32) + noise).to(BF16)
    g = _gen(seed + 5, device)
    out["x_ts"] = (torch.rand(n, generator=g, device=device, dtype=F32) * (1.86e-3 - 1.49e-3) + 1.49e-3)
    ew2 = w_std ** 2 * (1.0 - 0.001 + 0.001 * 50.0 ** 2)
    out["a_ts"] = (torch.rand(n, generator=g, device=device, dtype=F32) * 0.2 + 0.9) * (5.36e-3 * hidden * ew2)
    return out
