"""Pins of the weight-only NVFP4 product oracle (oracle.gemm_w4a16).

* brute force on a tiny case: every weight rebuilt from its code and block
  scale through the scalar decoders, one binary32 product, one bf16
  rounding, and the dot products summed term by term in Python;
* agreement with the W4A4 oracle (a separate C summation of exact products)
  whenever the dequantized weights are exact in bf16: with a power-of-two
  tensor scale, value(q) (2 significant bits) times an E4M3 value (4 bits)
  fits bf16's 8, and the activations are taken as the exact dequantization
  of their own NVFP4 codes;
* the bf16 rounding of the weights is really applied: with a tensor scale
  that is not a power of two the two products differ, by at most the bf16
  rounding error of the weights.
"""
import numpy as np
import pytest

import oracle as O


def _weights(rng, N, K):
    return (rng.normal(0, 0.02, (N, K)) * np.exp(rng.normal(0, 0.5, (N, K)))).astype(np.float32)


def test_brute_force_tiny():
    rng = np.random.default_rng(0)
    M, N, K = 2, 3, 32
    a_bits = O.bf16_round(rng.normal(0, 1, (M, K)))
    a = O.bf16_bits_to_f32(a_bits)
    w = _weights(rng, N, K)
    codes, sb, sg = O.quantize(w, O.DYNAMIC)
    got = O.gemm_w4a16(a, codes, sb, sg, K)
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                byte = int(codes[n, k // 2])
                q = (byte >> 4) if (k & 1) else (byte & 0xF)
                d = np.float32(O.e4m3_value(int(sb[n, k // 16]))) * np.float32(sg)
                prod = np.float32(np.float32(O.e2m1_value(q)) * d)
                w_hat = float(O.bf16_bits_to_f32(np.array([O.bf16_round_scalar(float(prod))], np.uint16))[0])
                acc += float(a[m, k]) * w_hat
            assert abs(got[m, n] - acc) <= 1e-12 * max(1.0, abs(acc))


@pytest.mark.parametrize("shape", [(5, 7, 64), (33, 20, 256)])
def test_equals_w4a4_when_weights_are_exact_in_bf16(shape):
    M, N, K = shape
    rng = np.random.default_rng(M + N)
    x = rng.normal(0, 1, (M, K)).astype(np.float32)
    w = _weights(rng, N, K)
    sg_a, sg_w = 2.0 ** -9, 2.0 ** -13
    ca, sa, _ = O.quantize(x, O.FROZEN_GLOBAL, s_g=sg_a)
    cw, sw, _ = O.quantize(w, O.FROZEN_GLOBAL, s_g=sg_w)
    a_hat, a_bits = O.dequantize(ca, sa, sg_a, K)
    assert np.array_equal(O.bf16_bits_to_f32(a_bits), a_hat)  # exact in bf16 too
    c16 = O.gemm_w4a16(a_hat, cw, sw, sg_w, K)
    c4 = O.gemm_w4a4(ca, sa, sg_a, cw, sw, sg_w, K)
    assert np.abs(c16 - c4).max() <= 1e-13 * np.abs(c4).max()


def test_weight_rounding_is_applied():
    rng = np.random.default_rng(3)
    M, N, K = 16, 24, 128
    x = rng.normal(0, 1, (M, K)).astype(np.float32)
    w = _weights(rng, N, K)
    ca, sa, ga = O.quantize(x, O.FROZEN_GLOBAL, s_g=2.0 ** -9)
    cw, sw, gw = O.quantize(w, O.DYNAMIC)          # s_g = amax / 2688, not a power of two
    a_hat, _ = O.dequantize(ca, sa, ga, K)
    c16 = O.gemm_w4a16(a_hat, cw, sw, gw, K)
    c4 = O.gemm_w4a4(ca, sa, ga, cw, sw, gw, K)
    w_exact, _ = O.dequantize(cw, sw, gw, K)        # binary32 products, before the bf16 rounding
    bound = (np.abs(a_hat).astype(np.float64) @ np.abs(w_exact).astype(np.float64).T) * 2.0 ** -8
    diff = np.abs(c16 - c4)
    assert diff.max() > 0.0
    assert np.all(diff <= bound * (1 + 1e-6) + 1e-30)
