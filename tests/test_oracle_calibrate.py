"""Pins of the MSE block-scale calibration oracle (oracle.calibrate_mse)
against the pinned fake-quantizer: the chosen scale is the arg-min found by
an independent search that fake-quantizes every candidate code through
oracle.fake_quant, it is never worse than the amax scale, exactly
representable blocks give zero error, all-zero blocks take code 0, and the
choice is invariant under a common power-of-two scaling."""
import numpy as np
import pytest

import oracle as O


def _err_via_fake_quant(xb: np.ndarray, s_g: float, code: int) -> float:
    sb = np.full((xb.shape[0], xb.shape[1] // 16), code, np.uint8)
    y, _, _, _ = O.fake_quant(xb, O.FROZEN_ALL, s_g=s_g, s_b=sb)
    return float(np.sum((xb.astype(np.float64) - y.astype(np.float64)) ** 2))


@pytest.mark.parametrize("seed", range(3))
def test_choice_is_the_argmin_over_all_codes(seed):
    rng = np.random.default_rng(seed)
    x = (rng.normal(0, 1, (3, 32)) * np.exp(rng.normal(0, 1, (3, 32)))).astype(np.float32)
    s_g = float(np.abs(x).max() / 2688.0)
    sb, err = O.calibrate_mse(x, s_g)
    for r in range(3):
        for b in range(2):
            xb = x[r:r + 1, 16 * b:16 * b + 16]
            errs = np.array([_err_via_fake_quant(xb, s_g, c) for c in range(127)])
            c = int(sb[r, b])
            assert errs[c] <= errs.min() * (1 + 1e-5) + 1e-30           # an arg-min (fp32 vs fp64 sums)
            assert not np.any(errs[:c] < errs[c] * (1 - 1e-5) - 1e-30)  # no clearly better smaller code
            assert abs(float(err[r, b]) - errs[c]) <= 1e-5 * errs[c] + 1e-30


def test_never_worse_than_the_amax_scale():
    rng = np.random.default_rng(7)
    x = rng.normal(0, 0.02, (64, 256)).astype(np.float32)
    x[rng.random(x.shape) < 0.01] *= 40
    codes, sb_amax, s_g = O.quantize(x, O.DYNAMIC)
    sb, err = O.calibrate_mse(x, s_g)
    y, _, _, _ = O.fake_quant(x, O.FROZEN_ALL, s_g=s_g, s_b=sb_amax)
    e_amax = ((x.astype(np.float64) - y) ** 2).reshape(64, 16, 16).sum(-1)
    assert np.all(err.astype(np.float64) <= e_amax * (1 + 1e-5) + 1e-30)
    assert np.mean(err) < np.mean(e_amax)  # and strictly better on average


def test_representable_block_has_zero_error_and_zero_block_takes_code_zero():
    s_g = 0.01
    d = float(np.float32(O.e4m3_value(0x30) * s_g))
    vals = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -6, -4, -3, -2, -1.5, -1, -0.5, 0], np.float32)
    x = np.stack([(vals * np.float32(d)).astype(np.float32), np.zeros(16, np.float32)])
    sb, err = O.calibrate_mse(x, s_g)
    assert err[0, 0] == 0.0
    assert sb[1, 0] == 0 and err[1, 0] == 0.0


def test_power_of_two_scaling_invariance():
    rng = np.random.default_rng(9)
    x = rng.normal(0, 1, (8, 64)).astype(np.float32)
    s_g = float(np.abs(x).max() / 2688.0)
    sb, err = O.calibrate_mse(x, s_g)
    sb2, err2 = O.calibrate_mse(x * 4, s_g * 4)
    assert np.array_equal(sb, sb2)
    assert np.allclose(err2, err * 16, rtol=0, atol=0)
