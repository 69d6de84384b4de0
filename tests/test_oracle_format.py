"""Pins for the oracle's element and scale formats (no GPU).

The oracle's E2M1 / E4M3 / bf16 conversions are checked against things other
than themselves: hand-worked fixtures (tests/golden), the library conversions
of ml_dtypes and torch (run, not retyped), exhaustive sweeps and closed forms.
"""
import math
import os

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line


# ---------------------------------------------------------------- E2M1

def test_e2m1_value_set_with_sign():
    # E2M1 value set {0, 0.5, 1, 1.5, 2, 3, 4, 6} with a sign bit (bit 3).
    vals = [O.e2m1_value(c) for c in range(16)]
    assert vals[:8] == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert vals[8:] == [-v for v in vals[:8]]
    assert math.copysign(1.0, vals[8]) == -1.0  # code 8 is negative zero


def test_e2m1_value_set_matches_bit_layout():
    # 1 sign, 2 exponent (bias 1), 1 mantissa bit; exponent 0 is subnormal.
    for idx in range(8):
        e, m = idx >> 1, idx & 1
        ref = (m * 0.5) if e == 0 else (1 + m / 2) * 2.0 ** (e - 1)
        assert O.e2m1_value(idx) == ref


def test_e2m1_golden_rounding():
    for line in _rows("e2m1_rounding.txt"):
        v, code = line.split()
        assert O.e2m1_encode(float(v)) == int(code), line


def _ml_e2m1_code(v: np.ndarray) -> np.ndarray:
    # ml_dtypes float4_e2m1fn stores the 4-bit code in the low nibble of a byte
    return v.astype(np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF


def test_e2m1_matches_ml_dtypes_on_all_bf16_values():
    # every finite bf16 bit pattern, as the element/scale quotient
    bits = np.arange(1 << 16, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    f = f[np.isfinite(f)]
    ref = _ml_e2m1_code(f)
    got = np.array([O.e2m1_encode(float(v)) for v in f], dtype=np.uint8)
    assert np.array_equal(got, ref)


def test_e2m1_matches_ml_dtypes_dense_sweep():
    rng = np.random.default_rng(0)
    mids = np.float32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    mids = np.concatenate([mids, -mids])
    # random values, every midpoint and both of its binary32 neighbours
    v = np.concatenate([rng.uniform(-7, 7, 20000).astype(np.float32), mids,
                        np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(10) * np.sign(mids))])
    ref = _ml_e2m1_code(v)
    got = np.array([O.e2m1_encode(float(x)) for x in v], dtype=np.uint8)
    assert np.array_equal(got, ref)


def test_e2m1_nearest_by_brute_force_distance():
    # independent of the oracle's loop: the chosen value is at minimal distance
    rng = np.random.default_rng(1)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    for v in rng.uniform(-6, 6, 3000):
        c = O.e2m1_encode(float(np.float32(v)))
        dist = np.abs(abs(float(np.float32(v))) - grid)
        assert dist[c & 7] == dist.min()


# ---------------------------------------------------------------- E4M3

def test_e4m3_golden_values():
    for line in _rows("e4m3_values.txt"):
        code, val = line.split()
        assert O.e4m3_value(int(code, 16)) == float(val), line


def test_e4m3_table_matches_torch_and_ml_dtypes():
    codes = np.arange(256, dtype=np.uint8)
    ours = O.e4m3_table()
    ml = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    th = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for ref in (ml, th):
        same = (ours == ref) | (np.isnan(ours) & np.isnan(ref))
        assert same.all()
    assert np.isnan(ours[0x7F]) and np.isnan(ours[0xFF])
    assert np.nanmax(ours) == 448.0


def test_e4m3_encode_matches_libraries_in_range():
    rng = np.random.default_rng(2)
    table = O.e4m3_table()[:0x7F]
    mids = (table[1:] + table[:-1]) / 2
    t = np.concatenate([
        rng.uniform(0, 448, 20000),
        np.exp(rng.uniform(np.log(2.0 ** -12), np.log(448), 20000)),
        mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9), table,
    ]).astype(np.float32)
    t = t[(t >= 0) & (t <= 448)]
    ref_ml = t.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    ref_th = torch.from_numpy(t.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([O.e4m3_encode(float(x)) for x in t], dtype=np.uint8)
    assert np.array_equal(got, ref_ml)
    assert np.array_equal(got, ref_th)


def test_e4m3_saturates_above_448():
    for t in [448.0, 448.5, 463.9, 464.0, 500.0, 1e30, float("inf")]:
        assert O.e4m3_encode(t) == 0x7E


def test_e4m3_underflow_rounds_to_zero():
    # smallest subnormal is 2^-9; half of it is a tie -> even code 0
    assert O.e4m3_encode(2.0 ** -10) == 0
    assert O.e4m3_encode(2.0 ** -10 * 1.0001) == 1
    assert O.e4m3_encode(0.0) == 0


# ---------------------------------------------------------------- bf16 rounding

def test_bf16_round_matches_torch_on_float32_inputs():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(5000) * 10.0 ** rng.integers(-30, 30, 5000),
                        [0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38, 1e-40, -1e-40]]).astype(np.float32)
    ref = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = O.bf16_round(x.astype(np.float64))
    assert np.array_equal(got, ref)


def test_bf16_round_has_no_double_rounding():
    # 1 + 2^-8 + 2^-30 is just above the midpoint between 1 and 1 + 2^-7: the
    # nearest bf16 is 1 + 2^-7 (0x3F81).  Rounding through binary32 first
    # would land exactly on the midpoint and then tie to 1.0 (0x3F80).
    x = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert int(O.bf16_round(np.array([x]))[0]) == 0x3F81
    assert int(O.bf16_round(np.array([1.0 + 2.0 ** -8]))[0]) == 0x3F80  # exact tie -> even


def test_bf16_round_overflow_to_inf():
    big = (2 - 2.0 ** -7) * 2.0 ** 127
    assert int(O.bf16_round(np.array([big]))[0]) == 0x7F7F
    assert int(O.bf16_round(np.array([2.0 ** 128]))[0]) == 0x7F80
    assert int(O.bf16_round(np.array([-(2.0 ** 128)]))[0]) == 0xFF80


# ---------------------------------------------------------------- storage

def test_storage_cost_matches_memory_claim():
    # 4-bit codes + one 8-bit scale per 16 elements = 4.5 bits per element, so
    # NVFP4 stores ~1.8x less than FP8 (8 bits), the figure the Nemotron-3-Nano
    # NVFP4 article gives ("etwa 1,8-fach").
    x = np.zeros((3, 64), np.float32)
    codes, sb, _ = O.quantize(x)
    bytes_per_elem = (codes.nbytes + sb.nbytes) / x.size
    assert bytes_per_elem == 0.5625
    assert round(1.0 / bytes_per_elem, 2) == 1.78
    assert abs(1.0 / bytes_per_elem - 1.8) < 0.05


# ---------------------------------------------------------------- swizzled layout

def test_swizzled_offset_hand_examples():
    # 128-row x 4-block tiles of 512 bytes; inside a tile row r, block kb sit at
    # (r % 32) * 16 + (r // 32) * 4 + kb.  Worked by hand for cols = 256 (16
    # blocks -> 4 tiles along the row).
    assert O.swizzled_scale_offset(0, 0, 256) == 0
    assert O.swizzled_scale_offset(0, 3, 256) == 3
    assert O.swizzled_scale_offset(1, 0, 256) == 16
    assert O.swizzled_scale_offset(32, 0, 256) == 4
    assert O.swizzled_scale_offset(33, 2, 256) == 16 + 4 + 2
    assert O.swizzled_scale_offset(127, 3, 256) == 31 * 16 + 3 * 4 + 3
    assert O.swizzled_scale_offset(0, 4, 256) == 512
    assert O.swizzled_scale_offset(128, 0, 256) == 4 * 512
    assert O.swizzled_scale_offset(129, 5, 256) == (4 + 1) * 512 + 16 + 1


def test_swizzled_layout_is_a_bijection_and_chunks_are_contiguous():
    rows, cols = 300, 16 * 10
    nblk = cols // 16
    offs = np.array([[O.swizzled_scale_offset(r, kb, cols) for kb in range(nblk)] for r in range(rows)])
    assert len(np.unique(offs)) == offs.size
    assert offs.max() < O.swizzled_scale_bytes(rows, cols)
    # the 4 scales of a row inside one 64-element chunk are 4 consecutive bytes
    # (one 32-bit word per row and chunk)
    for r in range(rows):
        for kb in range(0, nblk - nblk % 4, 4):
            assert list(offs[r, kb:kb + 4]) == list(range(offs[r, kb], offs[r, kb] + 4))
    sb = np.arange(rows * nblk, dtype=np.uint32).reshape(rows, nblk).astype(np.uint8)
    sw = O.swizzle_scales(sb, cols)
    assert np.array_equal(sw[offs.ravel()], sb.ravel())
