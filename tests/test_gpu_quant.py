"""GPU parity of quantize / fake-quant / dequantize against the CPU oracle.

Codes, block scales (both layouts), tensor scales and fake-quant outputs must
be bit-exact; inputs come from the seeded generators, the oracle gets exact
host copies of the same bits.
"""
import numpy as np
import pytest
import torch

import oracle as O
import nvfp4_quantization_aware_b200 as Q
from nvfp4_quantization_aware_b200 import synthetic as S

pytestmark = pytest.mark.gpu

DEV = "cuda"
MODES = [Q.DYNAMIC, Q.FROZEN_GLOBAL, Q.FROZEN_ALL]


def _host_f32(x: torch.Tensor) -> np.ndarray:
    return x.float().cpu().numpy()


def _bits16(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _bits32(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int32).cpu().numpy().view(np.uint32)


def _frozen_inputs(xh):
    """Scales for the frozen modes: a dynamic oracle pass (as calibration would
    produce), so frozen calls see realistic s_g / s_b."""
    codes, sb, sg = O.quantize(xh, O.DYNAMIC)
    return sg, sb


def _run_and_compare(x: torch.Tensor, mode: int, layout: int = Q.SCALES_ROWMAJOR):
    xh = _host_f32(x)
    rows, cols = x.shape
    sg_in, sb_in = _frozen_inputs(xh)
    if mode == Q.DYNAMIC:
        ref_codes, ref_sb, ref_sg = O.quantize(xh, O.DYNAMIC)
        ts = None
        bs = None
    elif mode == Q.FROZEN_GLOBAL:
        ref_codes, ref_sb, ref_sg = O.quantize(xh, O.FROZEN_GLOBAL, s_g=sg_in * 1.25)
        ts = torch.tensor([np.float32(sg_in * 1.25)], device=DEV)
        bs = None
    else:
        # perturb the frozen block scales so they differ from what the data implies
        sb_f = np.clip(sb_in.astype(np.int32) + (np.arange(sb_in.size).reshape(sb_in.shape) % 3) - 1, 0, 0x7E).astype(np.uint8)
        ref_codes, ref_sb, ref_sg = O.quantize(xh, O.FROZEN_ALL, s_g=sg_in, s_b=sb_f)
        ts = torch.tensor([np.float32(sg_in)], device=DEV)
        bs = torch.from_numpy(sb_f).to(DEV)
    codes, sbs, tsg = Q.nvfp4_quantize(x, mode=mode, tensor_scale=ts, block_scales=bs,
                                       layout=layout if mode != Q.FROZEN_ALL else Q.SCALES_ROWMAJOR)
    torch.cuda.synchronize()
    assert np.array_equal(codes.cpu().numpy(), ref_codes), "codes differ"
    assert _bits32(tsg)[0] == np.float32(ref_sg).view(np.uint32), "tensor scale differs"
    if layout == Q.SCALES_MMA and mode != Q.FROZEN_ALL:
        assert np.array_equal(sbs.cpu().numpy(), O.swizzle_scales(ref_sb, cols)), "MMA scales differ"
    else:
        assert np.array_equal(sbs.cpu().numpy(), ref_sb), "block scales differ"
    return ref_codes, ref_sb, ref_sg


SHAPES = [(1, 16), (3, 48), (17, 272), (64, 1024), (130, 1040), (5, 4096), (257, 64)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_quantize_parity(shape, mode, dtype):
    x = S.weights(*shape, seed=shape[0] * 7 + shape[1], device=DEV, outlier_p=0.01, outlier_mult=40, dtype=dtype)
    _run_and_compare(x, mode)


@pytest.mark.parametrize("shape", [(1, 16), (130, 1040), (300, 80), (128, 256)])
@pytest.mark.parametrize("mode", [Q.DYNAMIC, Q.FROZEN_GLOBAL])
def test_quantize_mma_layout_parity(shape, mode):
    x = S.activations(*shape, seed=11 + shape[0], device=DEV)
    _run_and_compare(x, mode, layout=Q.SCALES_MMA)


def test_quantize_row_stride():
    big = S.activations(33, 160, seed=3, device=DEV)
    x = big[:, :96]
    assert x.stride(0) == 160
    ref_codes, ref_sb, ref_sg = O.quantize(_host_f32(x), O.DYNAMIC)
    codes, sb, sg = Q.nvfp4_quantize(x)
    assert np.array_equal(codes.cpu().numpy(), ref_codes) and np.array_equal(sb.cpu().numpy(), ref_sb)


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_fake_quant_parity(mode, dtype):
    x = S.weights(96, 1040, seed=5, device=DEV, outlier_p=0.005, outlier_mult=30, dtype=dtype)
    xh = _host_f32(x)
    sg_in, sb_in = _frozen_inputs(xh)
    if mode == Q.DYNAMIC:
        ref32, ref16, ref_sb, ref_sg = O.fake_quant(xh)
        y, sb, sg = Q.nvfp4_fake_quant(x, mode, return_scales=True)
    elif mode == Q.FROZEN_GLOBAL:
        ref32, ref16, ref_sb, ref_sg = O.fake_quant(xh, O.FROZEN_GLOBAL, s_g=sg_in)
        y, sb, sg = Q.nvfp4_fake_quant(x, mode, tensor_scale=torch.tensor([sg_in], device=DEV), return_scales=True)
    else:
        ref32, ref16, ref_sb, ref_sg = O.fake_quant(xh, O.FROZEN_ALL, s_g=sg_in, s_b=sb_in)
        sb_t = torch.from_numpy(sb_in).to(DEV)
        y, sb, sg = Q.nvfp4_fake_quant(x, mode, tensor_scale=torch.tensor([sg_in], device=DEV), block_scales=sb_t,
                                       return_scales=True)
    torch.cuda.synchronize()
    if dtype == torch.bfloat16:
        assert np.array_equal(_bits16(y), ref16)
    else:
        assert np.array_equal(_bits32(y), ref32.view(np.uint32))
    assert np.array_equal(sb.cpu().numpy(), ref_sb)
    assert _bits32(sg)[0] == np.float32(ref_sg).view(np.uint32)


def test_fake_quant_in_place_alias():
    x = S.activations(64, 1024, seed=6, device=DEV)
    ref32, ref16, _, _ = O.fake_quant(_host_f32(x))
    Q.nvfp4_fake_quant(x, Q.DYNAMIC, out=x)
    torch.cuda.synchronize()
    assert np.array_equal(_bits16(x), ref16)


def test_fake_quant_equals_gpu_dequant_of_quant():
    x = S.weights(200, 512, seed=7, device=DEV)
    y = Q.nvfp4_fake_quant(x)
    codes, sb, sg = Q.nvfp4_quantize(x)
    z = Q.nvfp4_dequantize(codes, sb, sg, 512)
    zm = Q.nvfp4_dequantize(*Q.nvfp4_quantize(x, layout=Q.SCALES_MMA)[:2], sg, 512, layout=Q.SCALES_MMA)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), z.view(torch.int16))
    assert torch.equal(y.view(torch.int16), zm.view(torch.int16))


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_dequantize_parity(out_dtype):
    x = S.weights(77, 320, seed=8, device=DEV, outlier_p=0.01, outlier_mult=50)
    codes, sb, sg = Q.nvfp4_quantize(x)
    out = Q.nvfp4_dequantize(codes, sb, sg, 320, out_dtype=out_dtype)
    ref32, ref16 = O.dequantize(codes.cpu().numpy(), sb.cpu().numpy(), float(sg.cpu()[0]), 320)
    if out_dtype == torch.bfloat16:
        assert np.array_equal(_bits16(out), ref16)
    else:
        assert np.array_equal(_bits32(out), ref32.view(np.uint32))


def test_every_bf16_value_through_e2m1():
    # FROZEN_ALL with s_g = 1 and s_b = 1.0 makes d = 1, so each code is the
    # E2M1 rounding of the bf16 value itself: every finite bf16 pattern once.
    bits = np.arange(1 << 16, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    f = f[np.isfinite(f)]
    pad = (-f.size) % 16
    f = np.concatenate([f, np.zeros(pad, np.float32)]).reshape(-1, 16)
    x = torch.from_numpy(f).to(torch.bfloat16).to(DEV)
    sb = np.full((f.shape[0], 1), 0x38, np.uint8)
    ref_codes, _, _ = O.quantize(f, O.FROZEN_ALL, s_g=1.0, s_b=sb)
    codes, _, _ = Q.nvfp4_quantize(x, Q.FROZEN_ALL, tensor_scale=torch.ones(1, device=DEV),
                                   block_scales=torch.from_numpy(sb).to(DEV))
    assert np.array_equal(codes.cpu().numpy(), ref_codes)
    # same values as f32 input (the f32 path divides with IEEE division)
    codes32, _, _ = Q.nvfp4_quantize(x.float(), Q.FROZEN_ALL, tensor_scale=torch.ones(1, device=DEV),
                                     block_scales=torch.from_numpy(sb).to(DEV))
    assert np.array_equal(codes32.cpu().numpy(), ref_codes)


def test_block_scale_rounding_sweep():
    # Blocks [m, small...] for a sweep of maxima m: the block scale is
    # E4M3(m / (6 s_g)), crossing every E4M3 rounding midpoint and saturation.
    rng = np.random.default_rng(0)
    table = O.e4m3_table()[:0x7F]
    mids = (table[1:] + table[:-1]) / 2
    sg = np.float32(1.0 / 6.0)
    t = np.concatenate([mids, table, rng.uniform(0, 460, 4000), [448, 460, 470, 1e4]])
    m = (t * 6.0 * float(sg)).astype(np.float32)
    m = np.concatenate([m, np.nextafter(m, np.float32(0)), np.nextafter(m, np.float32(1e30))])
    m = torch.from_numpy(m).to(torch.bfloat16).float().numpy()  # bf16-representable
    blocks = np.zeros((m.size, 16), np.float32)
    blocks[:, 0] = m
    blocks[:, 5] = -m * 0.3
    blocks[:, 9] = m * 0.77
    blocks = torch.from_numpy(blocks).to(torch.bfloat16).float().numpy()  # what the kernel sees
    x = torch.from_numpy(blocks).to(torch.bfloat16).to(DEV)
    ref_codes, ref_sb, _ = O.quantize(blocks, O.FROZEN_GLOBAL, s_g=float(sg))
    codes, sb, _ = Q.nvfp4_quantize(x, Q.FROZEN_GLOBAL, tensor_scale=torch.tensor([sg], device=DEV))
    assert np.array_equal(sb.cpu().numpy(), ref_sb)
    assert np.array_equal(codes.cpu().numpy(), ref_codes)


def test_special_tensors():
    # all zeros, negative zeros, tiny (subnormal s_g), huge magnitudes
    cases = [
        np.zeros((4, 32), np.float32),
        -np.zeros((4, 32), np.float32),
        (np.random.default_rng(1).standard_normal((8, 64)) * 1e-38).astype(np.float32),
        (np.random.default_rng(2).standard_normal((8, 64)) * 1e37).astype(np.float32),
    ]
    for c in cases:
        c = torch.from_numpy(c).to(torch.bfloat16).float().numpy()
        x = torch.from_numpy(c).to(torch.bfloat16).to(DEV)
        ref_codes, ref_sb, ref_sg = O.quantize(c, O.DYNAMIC)
        codes, sb, sg = Q.nvfp4_quantize(x)
        assert np.array_equal(codes.cpu().numpy(), ref_codes)
        assert np.array_equal(sb.cpu().numpy(), ref_sb)
        assert _bits32(sg)[0] == np.float32(ref_sg).view(np.uint32)
        y32, y16, _, _ = O.fake_quant(c)
        assert np.array_equal(_bits16(Q.nvfp4_fake_quant(x)), y16)


def test_division_selftest_exhaustive():
    mismatches, first = Q.nvfp4_selftest_division()
    assert mismatches == 0, hex(first)


def test_empty_tensor():
    x = torch.empty(0, 64, dtype=torch.bfloat16, device=DEV)
    codes, sb, sg = Q.nvfp4_quantize(x)
    torch.cuda.synchronize()
    assert codes.numel() == 0 and float(sg.cpu()[0]) == 0.0


def test_bad_arguments_raise():
    x = torch.zeros(4, 40, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(Q.NVFP4Error):
        Q.nvfp4_quantize(x)
    with pytest.raises(ValueError):
        Q.nvfp4_quantize(torch.zeros(4, 32, dtype=torch.bfloat16))  # CPU tensor


def test_weight_sweep_expert_parity():
    # a slice of the MoE weight sweep at full expert size (2048 x 1024)
    for i in (0, 77):
        w = S.weights(2048, 1024, seed=i, device=DEV)
        for mode in MODES:
            _run_and_compare(w, mode)
    _run_and_compare(S.weights(2048, 1024, seed=5, device=DEV), Q.DYNAMIC, layout=Q.SCALES_MMA)


@pytest.mark.slow
def test_weight_sweep_full_size_parity():
    # The whole 128-expert + lm_head sweep, dynamic then frozen (scales from
    # the dynamic pass), every code and scale compared.
    O.set_threads(max(1, O.get_threads()))
    ws = S.weight_sweep(seed=0, device=DEV)
    for i, w in enumerate(ws):
        if i % 16 != 0 and i != len(ws) - 1:
            continue  # every 16th expert plus the 131072 x 2048 lm_head
        xh = _host_f32(w)
        ref_codes, ref_sb, ref_sg = O.quantize(xh, O.DYNAMIC)
        codes, sb, sg = Q.nvfp4_quantize(w)
        assert np.array_equal(codes.cpu().numpy(), ref_codes), i
        assert np.array_equal(sb.cpu().numpy(), ref_sb), i
        codes_f, _, _ = Q.nvfp4_quantize(w, Q.FROZEN_ALL, tensor_scale=sg, block_scales=sb)
        assert torch.equal(codes_f, codes), i


def test_grouped_quantize_matches_oracle_and_single_calls():
    # mixed shapes, an empty tensor, more tensors than one launch holds, and
    # large tensors among small ones
    shapes = [(64, 1024), (4001, 272), (2048, 4096), (0, 32), (3, 48), (130, 1040)] + [(40, 256)] * 150 + \
        [(6000, 2048)]
    xs = [S.weights(r, c, seed=100 + i, device=DEV, outlier_p=0.01, outlier_mult=40) for i, (r, c) in enumerate(shapes)]
    for mode in [Q.DYNAMIC, Q.FROZEN_GLOBAL, Q.FROZEN_ALL]:
        if mode == Q.DYNAMIC:
            codes, sbs, ts = Q.nvfp4_quantize_grouped(xs, mode)
        else:
            ref_sg = torch.empty(len(xs), device=DEV)
            ref_sb = []
            for i, x in enumerate(xs):
                c, sb, sg = Q.nvfp4_quantize(x)
                ref_sg[i] = sg[0] * (1.25 if mode == Q.FROZEN_GLOBAL else 1.0)
                ref_sb.append(sb)
            codes, sbs, ts = Q.nvfp4_quantize_grouped(xs, mode, tensor_scales=ref_sg,
                                                      block_scales=ref_sb if mode == Q.FROZEN_ALL else None)
        torch.cuda.synchronize()
        for i, x in enumerate(xs):
            if i % 7 != 0 and i not in (1, 2, 3, 4, 5, len(xs) - 1):
                continue
            xh = _host_f32(x)
            if mode == Q.DYNAMIC:
                rc, rsb, rsg = O.quantize(xh, O.DYNAMIC)
            elif mode == Q.FROZEN_GLOBAL:
                rc, rsb, rsg = O.quantize(xh, O.FROZEN_GLOBAL, s_g=float(ts[i].cpu()))
            else:
                rc, rsb, rsg = O.quantize(xh, O.FROZEN_ALL, s_g=float(ts[i].cpu()), s_b=sbs[i].cpu().numpy())
            assert np.array_equal(codes[i].cpu().numpy(), rc), (mode, i)
            assert np.array_equal(sbs[i].cpu().numpy(), rsb), (mode, i)
            assert _bits32(ts[i:i + 1])[0] == np.float32(rsg).view(np.uint32), (mode, i)


def test_grouped_mma_layout_and_fake_quant():
    xs = [S.activations(r, c, seed=200 + r, device=DEV) for r, c in [(130, 1040), (128, 256), (1, 16)]]
    codes, sbs, ts = Q.nvfp4_quantize_grouped(xs, Q.DYNAMIC, layout=Q.SCALES_MMA)
    ys = Q.nvfp4_fake_quant_grouped(xs, Q.DYNAMIC)
    torch.cuda.synchronize()
    for i, x in enumerate(xs):
        xh = _host_f32(x)
        rc, rsb, rsg = O.quantize(xh, O.DYNAMIC)
        assert np.array_equal(codes[i].cpu().numpy(), rc)
        assert np.array_equal(sbs[i].cpu().numpy(), O.swizzle_scales(rsb, x.shape[1]))
        _, y16, _, _ = O.fake_quant(xh)
        assert np.array_equal(_bits16(ys[i]), y16)


def test_launch_counter_counts_kernels():
    x = S.activations(64, 256, seed=1, device=DEV)
    n0 = Q.nvfp4_launch_count()
    Q.nvfp4_quantize(x)                      # small dynamic group: one cluster launch
    Q.nvfp4_quantize(x, Q.FROZEN_GLOBAL, tensor_scale=torch.ones(1, device=DEV))  # encode
    assert Q.nvfp4_launch_count() - n0 == 2
    xs = [S.activations(16, 64, seed=3 + i, device=DEV) for i in range(150)]
    n0 = Q.nvfp4_launch_count()
    Q.nvfp4_quantize_grouped(xs)  # 144 tensors (2304 chunks): amax + encode; 6 tensors (96 chunks): one launch
    assert Q.nvfp4_launch_count() - n0 == 3
    big = S.activations(64, 2064, seed=2, device=DEV)  # 320 chunks: amax + encode
    n0 = Q.nvfp4_launch_count()
    Q.nvfp4_quantize(big)
    assert Q.nvfp4_launch_count() - n0 == 2


@pytest.mark.parametrize("rows,cols", [(64, 2048), (64, 2064), (1, 16), (3, 8192), (2048, 2048)])
def test_dynamic_small_and_large_paths_match_oracle(rows, cols):
    # 64 x 2048 is the largest group the one-launch cluster path takes (256
    # chunks of 512 elements); 64 x 2064 (320 chunks) takes amax + encode
    x = S.weights(rows, cols, seed=rows + cols, device=DEV, outlier_p=0.01, outlier_mult=30)
    codes, sb, ts = Q.nvfp4_quantize(x, Q.DYNAMIC)
    ref_codes, ref_sb, ref_sg = O.quantize(_host_f32(x), O.DYNAMIC)
    assert np.array_equal(codes.cpu().numpy(), ref_codes)
    assert np.array_equal(sb.cpu().numpy(), ref_sb)
    assert np.float32(ts.cpu().numpy()[0]).view(np.uint32) == np.float32(ref_sg).view(np.uint32)


def test_unaligned_rows_use_narrow_accesses():
    # input rows 16-byte but not 32-byte aligned, code rows 4-byte but not
    # 8-byte aligned, fake-quant output rows 16-byte aligned only
    big = S.weights(37, 160, seed=21, device=DEV, outlier_p=0.01, outlier_mult=30)
    x = big[:, 8:104]
    assert (x.data_ptr() % 32) == 16
    codes_buf = torch.zeros(37, 52, dtype=torch.uint8, device=DEV)
    codes = codes_buf[:, 4:52]
    assert codes.stride(0) == 52 and codes.data_ptr() % 8 == 4
    ref_codes, ref_sb, ref_sg = O.quantize(_host_f32(x), O.DYNAMIC)
    c, sb, sg = Q.nvfp4_quantize(x, codes=codes)
    torch.cuda.synchronize()
    assert np.array_equal(c.cpu().numpy(), ref_codes) and np.array_equal(sb.cpu().numpy(), ref_sb)
    assert not codes_buf[:, :4].any()  # nothing written outside the view
    ybuf = torch.zeros(37, 112, dtype=torch.bfloat16, device=DEV)
    y = ybuf[:, 8:104]
    Q.nvfp4_fake_quant(x, out=y)
    _, y16, _, _ = O.fake_quant(_host_f32(x))
    assert np.array_equal(_bits16(y), y16)
    assert not ybuf[:, :8].any() and not ybuf[:, 104:].any()
    # f32 input with 16-byte aligned rows
    xf = S.activations(9, 200, seed=22, device=DEV, dtype=torch.float32)[:, 4:196]
    rc, rsb, rsg = O.quantize(_host_f32(xf), O.DYNAMIC)
    c2, sb2, _ = Q.nvfp4_quantize(xf)
    assert np.array_equal(c2.cpu().numpy(), rc) and np.array_equal(sb2.cpu().numpy(), rsb)
