"""Pins for the oracle's quantize / dequantize / fake-quant (no GPU).

Checked against hand-worked blocks (tests/golden/quant_blocks.txt), library
conversions (ml_dtypes E2M1/E4M3 of the same binary32 quotients), closed-form
cases, the error bound of round-to-nearest and the mode semantics of the two
scale strategies.
"""
import os

import ml_dtypes
import numpy as np
import pytest

import oracle as O
from nvfp4_quantization_aware_b200 import synthetic as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
MODES = {"DYNAMIC": O.DYNAMIC, "FROZEN_GLOBAL": O.FROZEN_GLOBAL, "FROZEN_ALL": O.FROZEN_ALL}


def _unpack(codes: np.ndarray) -> np.ndarray:
    lo = codes & 0xF
    hi = codes >> 4
    return np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)


def _bf16_input(t):
    return t.float().numpy()


def test_golden_blocks():
    with open(os.path.join(GOLDEN, "quant_blocks.txt")) as f:
        lines = [l.strip() for l in f if l.strip() and not l.startswith("#")]
    assert len(lines) >= 5
    for line in lines:
        name, mode, sg, sb, xs, exp_sb, exp_codes = [p.strip() for p in line.split("|")]
        x = np.array([[float(v) for v in xs.split()]], dtype=np.float32)
        sb_in = None if sb == "-" else np.array([[int(sb, 16)]], dtype=np.uint8)
        codes, sb_out, sg_out = O.quantize(x, MODES[mode], s_g=float(sg), s_b=sb_in)
        assert int(sb_out[0, 0]) == int(exp_sb, 16), name
        assert list(_unpack(codes)[0]) == [int(c) for c in exp_codes.split()], name
        assert sg_out == np.float32(float(sg))


def test_dynamic_single_max_element():
    # x = [6, 0, ...]: s_g = 6/2688 (binary32), s_b saturates at 448, q = 6.
    x = np.zeros((1, 16), np.float32)
    x[0, 0] = 6.0
    codes, sb, sg = O.quantize(x)
    assert sg == np.float32(6.0) / np.float32(2688.0)
    assert sb[0, 0] == 0x7E
    assert list(_unpack(codes)[0]) == [7] + [0] * 15


def test_all_zero_tensor():
    x = np.zeros((5, 32), np.float32)
    codes, sb, sg = O.quantize(x)
    assert sg == 0.0 and not sb.any() and not codes.any()
    y, yb, _, _ = O.fake_quant(x)
    assert not y.any() and not yb.any()


def _library_reference_codes(x, sg, sb):
    """E2M1 codes from ml_dtypes on the same binary32 quotients x / d."""
    rows, cols = x.shape
    d = (sb.astype(np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float32) * np.float32(sg))
    d = np.repeat(d, 16, axis=1).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = (x / d).astype(np.float32)
    codes = q.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    codes[d == 0] = 0
    return codes


def _library_reference_scales(x, sg):
    rows, cols = x.shape
    ab = np.abs(x).reshape(rows, cols // 16, 16).max(axis=2).astype(np.float32)
    if sg == 0:
        return np.zeros_like(ab, dtype=np.uint8)
    t = (ab / (np.float32(6.0) * np.float32(sg))).astype(np.float32)
    t = np.minimum(t, np.float32(448.0))  # saturate
    return t.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)


@pytest.mark.parametrize("seed", [0, 1])
def test_quantize_matches_library_conversions(seed):
    x = _bf16_input(S.weights(96, 256, seed, outlier_p=0.01, outlier_mult=40))
    codes, sb, sg = O.quantize(x)
    assert sg == np.float32(np.abs(x).max()) / np.float32(2688.0)
    assert np.array_equal(sb, _library_reference_scales(x, sg))
    assert np.array_equal(_unpack(codes), _library_reference_codes(x, sg, sb))


def test_quantize_brute_force_nearest_on_tiny_blocks():
    # Exhaustive check on small blocks: each code is the nearest of all 16 E2M1
    # codes to x/d (ties to even index), and s_b is the nearest of all 127
    # finite E4M3 values to a_b / (6 s_g).
    rng = np.random.default_rng(7)
    e4 = O.e4m3_table()[:0x7F]
    e2 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)
    for trial in range(200):
        x = (rng.standard_normal((1, 16)) * rng.choice([0.01, 1, 50])).astype(np.float32)
        sg = np.float32(rng.uniform(0.001, 0.2))
        codes, sb, _ = O.quantize(x, O.FROZEN_GLOBAL, s_g=float(sg))
        t = np.float32(np.abs(x).max()) / (np.float32(6.0) * sg)
        tt = min(float(t), 448.0)
        dist = np.abs(e4 - tt)
        best = np.flatnonzero(dist == dist.min())
        assert int(sb[0, 0]) in best and (len(best) == 1 or int(sb[0, 0]) % 2 == 0)
        d = np.float32(e4[sb[0, 0]]) * sg
        for i, c in enumerate(_unpack(codes)[0]):
            q = float(np.float32(x[0, i]) / d)
            a = min(abs(q), 6.0)
            dd = np.abs(e2 - a)
            cand = np.flatnonzero(dd == dd.min())
            assert (c & 7) in cand and (len(cand) == 1 or (c & 7) % 2 == 0)
            assert (c >> 3) == (1 if np.signbit(q) else 0)


def test_block_holding_the_tensor_max_uses_full_range():
    x = _bf16_input(S.weights(64, 128, 3))
    codes, sb, sg = O.quantize(x)
    r, c = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    assert sb[r, c // 16] == 0x7E  # 448
    assert (_unpack(codes)[r, c] & 7) == 7  # |q| = 6


def test_frozen_modes_reproduce_dynamic():
    x = _bf16_input(S.activations(40, 96, 4))
    c0, sb0, sg0 = O.quantize(x, O.DYNAMIC)
    c1, sb1, sg1 = O.quantize(x, O.FROZEN_GLOBAL, s_g=sg0)
    c2, sb2, sg2 = O.quantize(x, O.FROZEN_ALL, s_g=sg0, s_b=sb0)
    assert np.array_equal(c0, c1) and np.array_equal(sb0, sb1) and sg1 == sg0
    assert np.array_equal(c0, c2) and np.array_equal(sb0, sb2) and sg2 == sg0


def test_frozen_all_uses_given_scales_not_data():
    x = _bf16_input(S.activations(8, 32, 5))
    sb = np.full((8, 2), 0x38, np.uint8)  # 1.0
    codes, sb_out, _ = O.quantize(x, O.FROZEN_ALL, s_g=1.0, s_b=sb)
    assert np.array_equal(sb_out, sb)
    ref = (np.clip(x, -6, 6).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF)
    assert np.array_equal(_unpack(codes), ref)


def test_fake_quant_equals_dequant_of_quant_bitwise():
    x = _bf16_input(S.weights(64, 160, 6, outlier_p=0.005, outlier_mult=30))
    codes, sb, sg = O.quantize(x)
    f32, b16 = O.dequantize(codes, sb, sg, x.shape[1])
    y32, yb16, sb2, sg2 = O.fake_quant(x)
    assert np.array_equal(f32.view(np.uint32), y32.view(np.uint32))
    assert np.array_equal(b16, yb16)
    assert np.array_equal(sb, sb2) and sg == sg2


def test_dequantize_matches_library_decode():
    x = _bf16_input(S.weights(32, 64, 8))
    codes, sb, sg = O.quantize(x)
    f32, b16 = O.dequantize(codes, sb, sg, 64)
    q = _unpack(codes).astype(np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float32)
    d = (sb.view(ml_dtypes.float8_e4m3fn).astype(np.float32) * np.float32(sg)).astype(np.float32)
    ref = (q * np.repeat(d, 16, axis=1)).astype(np.float32)
    assert np.array_equal(f32.view(np.uint32), ref.view(np.uint32))
    import torch
    ref16 = torch.from_numpy(ref).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(b16, ref16)


def test_negative_zero_is_kept():
    x = np.zeros((1, 16), np.float32)
    x[0, 0] = 6.0
    x[0, 1] = -0.001  # rounds to zero, keeps its sign
    codes, sb, sg = O.quantize(x)
    assert _unpack(codes)[0, 1] == 8
    y, yb, _, _ = O.fake_quant(x)
    assert yb[0, 1] == 0x8000


def test_fake_quant_idempotent_with_frozen_scales():
    x = _bf16_input(S.weights(48, 128, 9, outlier_p=0.005, outlier_mult=30))
    y, yb, sb, sg = O.fake_quant(x)
    y_as_bf16 = O.bf16_bits_to_f32(yb)
    y2, yb2, sb2, sg2 = O.fake_quant(y_as_bf16, O.FROZEN_ALL, s_g=sg, s_b=sb)
    assert np.array_equal(yb, yb2)


def test_dynamic_refake_keeps_tensor_scale():
    # Re-quantizing dynamically keeps s_g (the tensor max survives exactly:
    # it maps to |q| = 6 at s_b = 448 and d * 6 reproduces it up to the bf16
    # rounding); block scales of blocks whose max rounded below 6 may move.
    x = _bf16_input(S.weights(48, 128, 10))
    y, yb, sb, sg = O.fake_quant(x)
    y2, yb2, sb2, sg2 = O.fake_quant(O.bf16_bits_to_f32(yb))
    amax_y = np.abs(O.bf16_bits_to_f32(yb)).max()
    assert sg2 == np.float32(amax_y) / np.float32(2688.0)
    assert abs(sg2 - sg) <= 2 ** -7 * sg


def test_fake_quant_error_bound():
    # Round-to-nearest error: unsaturated elements are within half an E2M1
    # step of x/d (0.25 d below 2, 0.5 d in [2, 4), 1 d in [4, 6)), plus the
    # binary32 / bf16 output roundings.
    x = _bf16_input(S.weights(64, 256, 11, outlier_p=0.01, outlier_mult=40))
    y, yb, sb, sg = O.fake_quant(x)
    d = np.repeat((sb.view(ml_dtypes.float8_e4m3fn).astype(np.float64) * sg), 16, axis=1)
    q = np.abs(x.astype(np.float64)) / np.where(d == 0, 1, d)
    half_step = np.where(q < 2, 0.25, np.where(q < 4, 0.5, 1.0)) * d
    err = np.abs(O.bf16_bits_to_f32(yb).astype(np.float64) - x)
    unsat = q <= 6
    slack = np.abs(x) * 2.0 ** -8 + 1e-30
    assert np.all(err[unsat] <= half_step[unsat] + slack[unsat])
    # saturated elements sit exactly at +-6 d (rounded)
    sat = q > 6
    assert np.allclose(np.abs(O.bf16_bits_to_f32(yb)[sat]), 6 * d[sat], rtol=2 ** -7)


def test_quantize_respects_row_stride():
    x = _bf16_input(S.activations(7, 48, 12))
    big = np.zeros((7, 80), np.float32)
    big[:, :48] = x
    big[:, 48:] = 1e6  # garbage beyond the logical columns must be ignored
    codes, sb, sg = O.quantize(x)
    sg2 = np.zeros(1, np.float32)
    sb2 = np.zeros((7, 3), np.uint8)
    codes2 = np.zeros((7, 24), np.uint8)
    st = O.lib().oracle_quantize(O._ptr(big), 7, 48, 80, O.DYNAMIC, O._ptr(sg2), O._ptr(sb2), O._ptr(codes2))
    assert st == 0 and sg2[0] == sg and np.array_equal(sb2, sb) and np.array_equal(codes2, codes)


def test_quantize_rejects_bad_shapes():
    x = np.zeros((2, 20), np.float32)
    with pytest.raises(ValueError):
        O.quantize(x)
