"""Pins for the oracle's W4A4 GEMM and KL distillation loss (no GPU).

GEMM: closed forms (all-ones), exact integer products against numpy int64
matmul, and torch.matmul in float64 on operands decoded by ml_dtypes (a
decode route independent of the oracle's tables).
KL: KL >= 0, KL = 0 for identical logits, shift invariance, sum of the
gradient is zero, the two-class (Bernoulli) closed form, the uniform-teacher
closed form, central finite differences and torch.log_softmax in float64.
"""
import math

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_quantization_aware_b200 import synthetic as S


def _pack(codes4: np.ndarray) -> np.ndarray:
    c = codes4.astype(np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def _decode(codes: np.ndarray, sb: np.ndarray, sg: float) -> np.ndarray:
    lo, hi = codes & 0xF, codes >> 4
    q = np.stack([lo, hi], -1).reshape(codes.shape[0], -1).astype(np.uint8)
    v = q.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    s = np.repeat(sb.view(ml_dtypes.float8_e4m3fn).astype(np.float64), 16, axis=1)
    return v * s * np.float64(sg)


# ---------------------------------------------------------------- GEMM

def test_gemm_all_ones_closed_form():
    M, N, K = 3, 5, 64
    a = _pack(np.full((M, K), 2))  # E2M1 index 2 = 1.0
    b = _pack(np.full((N, K), 2))
    sa = np.full((M, K // 16), 0x38, np.uint8)  # 1.0
    sb = np.full((N, K // 16), 0x38, np.uint8)
    c = O.gemm_w4a4(a, sa, 0.5, b, sb, 0.25, K)
    assert np.all(c == K * 0.5 * 0.25)


def test_gemm_integer_operands_exact():
    rng = np.random.default_rng(0)
    M, N, K = 17, 9, 96
    # E2M1 codes whose values are integers: 0, 1, 2, 3, 4, 6 and negatives
    int_codes = np.array([0, 2, 4, 5, 6, 7, 10, 12, 13, 14, 15], np.uint8)
    qa = rng.choice(int_codes, (M, K))
    qb = rng.choice(int_codes, (N, K))
    # power-of-two block scales 1, 2, 4 (0x38, 0x40, 0x48)
    sa = rng.choice(np.array([0x38, 0x40, 0x48], np.uint8), (M, K // 16))
    sb = rng.choice(np.array([0x38, 0x40, 0x48], np.uint8), (N, K // 16))
    c = O.gemm_w4a4(_pack(qa), sa, 1.0, _pack(qb), sb, 1.0, K)
    ia = qa.view(ml_dtypes.float4_e2m1fn).astype(np.int64) * np.repeat(2 ** ((sa.astype(np.int64) - 0x38) // 8), 16, 1)
    ib = qb.view(ml_dtypes.float4_e2m1fn).astype(np.int64) * np.repeat(2 ** ((sb.astype(np.int64) - 0x38) // 8), 16, 1)
    assert np.array_equal(c, (ia @ ib.T).astype(np.float64))


def test_gemm_matches_torch_matmul_on_decoded_operands():
    x = S.activations(40, 128, 1).float().numpy()
    w = S.weights(24, 128, 2, outlier_p=0.01, outlier_mult=30).float().numpy()
    ca, sa, ga = O.quantize(x)
    cb, sb, gb = O.quantize(w)
    c = O.gemm_w4a4(ca, sa, ga, cb, sb, gb, 128)
    ref = torch.from_numpy(_decode(ca, sa, ga)) @ torch.from_numpy(_decode(cb, sb, gb)).T
    assert np.allclose(c, ref.numpy(), rtol=1e-12, atol=1e-12)
    # and it is (close to) the float product of the unquantized operands
    rel = np.linalg.norm(c - x.astype(np.float64) @ w.T.astype(np.float64)) / np.linalg.norm(x @ w.T)
    assert rel < 0.2


def test_gemm_rows_subset_matches_full():
    x = S.activations(30, 64, 3).float().numpy()
    w = S.weights(20, 64, 4).float().numpy()
    ca, sa, ga = O.quantize(x)
    cb, sb, gb = O.quantize(w)
    full = O.gemm_w4a4(ca, sa, ga, cb, sb, gb, 64)
    rows = np.array([29, 0, 7, 7])
    sub = O.gemm_w4a4_rows(ca, sa, ga, cb, sb, gb, 64, rows)
    assert np.array_equal(sub, full[rows])


# ---------------------------------------------------------------- KL

def _logits(rows, V, seed, scale=3.0):
    rng = np.random.default_rng(seed)
    t = rng.standard_normal((rows, V)) * scale
    s = t + rng.standard_normal((rows, V))
    return t, s


def test_kl_nonnegative_and_zero_for_identical():
    t, s = _logits(6, 50, 0)
    loss, row, grad = O.kl(t, s)
    assert np.all(row >= 0) and loss > 0
    loss0, row0, grad0 = O.kl(t, t)
    assert np.all(np.abs(row0) < 1e-12) and np.all(np.abs(grad0) < 1e-15)


def test_kl_shift_invariance():
    t, s = _logits(4, 33, 1)
    base, row, g = O.kl(t, s)
    sh_t = t + np.arange(4)[:, None] * 7.5
    sh_s = s - np.arange(4)[:, None] * 3.25
    l2, row2, g2 = O.kl(sh_t, sh_s)
    assert np.allclose(row, row2, rtol=1e-10, atol=1e-12)
    assert np.allclose(g, g2, rtol=1e-9, atol=1e-15)


def test_kl_gradient_rows_sum_to_zero():
    t, s = _logits(5, 64, 2)
    _, _, g = O.kl(t, s, T=2.0)
    assert np.all(np.abs(g.sum(axis=1)) < 1e-15)


def test_kl_bernoulli_closed_form():
    for a, b, T in [(0.3, -1.2, 1.0), (2.0, 2.5, 0.7), (-4.0, 1.0, 3.0)]:
        t = np.array([[0.0, a]])
        s = np.array([[0.0, b]])
        p = 1 / (1 + math.exp(-a / T))
        q = 1 / (1 + math.exp(-b / T))
        ref = p * math.log(p / q) + (1 - p) * math.log((1 - p) / (1 - q))
        loss, row, g = O.kl(t, s, T=T, grad_scale=1.0)
        assert abs(loss - ref) < 1e-14
        # d/db of KL = (q - p) / T for the second class
        assert abs(g[0, 1] - (q - p) / T) < 1e-14


def test_kl_uniform_teacher_closed_form():
    V = 17
    rng = np.random.default_rng(3)
    s = rng.standard_normal((1, V)) * 2
    t = np.zeros((1, V))
    lse = math.log(np.exp(s[0] - s[0].max()).sum()) + s[0].max()
    ref = -math.log(V) - np.mean(s[0] - lse)
    loss, _, _ = O.kl(t, s)
    assert abs(loss - ref) < 1e-13


def test_kl_finite_differences():
    rng = np.random.default_rng(4)
    t = rng.standard_normal((3, 7)) * 2
    s = rng.standard_normal((3, 7)) * 2
    T = 1.3
    _, _, g = O.kl(t, s, T=T)  # grad_scale = 1/rows: gradient of the mean
    h = 1e-6
    for i in range(3):
        for v in range(7):
            sp, sm = s.copy(), s.copy()
            sp[i, v] += h
            sm[i, v] -= h
            fd = (O.kl(t, sp, T=T, want_grad=False)[0] - O.kl(t, sm, T=T, want_grad=False)[0]) / (2 * h)
            assert abs(fd - g[i, v]) < 1e-8


def test_kl_matches_torch_log_softmax():
    t, s = _logits(8, 257, 5)
    T = 0.9
    lt = torch.log_softmax(torch.from_numpy(t) / T, dim=1)
    ls = torch.log_softmax(torch.from_numpy(s) / T, dim=1)
    ref_row = (lt.exp() * (lt - ls)).sum(1).numpy()
    ref_g = ((ls.exp() - lt.exp()) / T / 8).numpy()
    loss, row, g = O.kl(t, s, T=T)
    assert np.allclose(row, ref_row, rtol=1e-12, atol=1e-14)
    assert abs(loss - ref_row.mean()) < 1e-13
    assert np.allclose(g, ref_g, rtol=1e-10, atol=1e-16)
    # torch's own KL divergence (input = log p_s, target = log p_t)
    kd = torch.nn.functional.kl_div(ls, lt, reduction="batchmean", log_target=True)
    assert abs(float(kd) - loss) < 1e-12


def test_kl_grad_scale_and_boosted_teacher():
    d = S.logits_pair(4, 1000, 0, teacher_std=3.0, noise_std=1.0, boost=12.0, dtype=torch.float32)
    t, s = d[0].double().numpy(), d[1].double().numpy()
    _, row, g1 = O.kl(t, s, grad_scale=1.0)
    _, _, g2 = O.kl(t, s, grad_scale=0.125)
    assert np.allclose(g2, g1 * 0.125, rtol=1e-15, atol=0)
    assert np.all(row > 0)
