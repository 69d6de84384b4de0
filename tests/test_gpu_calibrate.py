"""GPU parity of the MSE block-scale calibration (nvfp4_calibrate_mse): the
chosen E4M3 codes and the least error per block are bit-exact against the
oracle (the error decides the code, so both sides compute it in binary32 in
the same order)."""
import numpy as np
import pytest
import torch

import oracle as O
import nvfp4_quantization_aware_b200 as Q
from nvfp4_quantization_aware_b200 import synthetic as S

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _host(x):
    return x.float().cpu().numpy()


@pytest.mark.parametrize("rows,cols", [(1, 16), (3, 48), (17, 272), (64, 1024), (130, 1040)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_calibrate_matches_oracle(rows, cols, dtype):
    x = S.weights(rows, cols, seed=rows + cols, device=DEV, outlier_p=0.01, outlier_mult=40, dtype=dtype)
    _, _, ts = Q.nvfp4_quantize(x, Q.DYNAMIC)
    sb, err = Q.nvfp4_calibrate_mse(x, ts, want_err=True)
    torch.cuda.synchronize()
    rsb, rerr = O.calibrate_mse(_host(x), float(ts.cpu()[0]))
    assert np.array_equal(sb.cpu().numpy(), rsb)
    assert np.array_equal(err.cpu().numpy().view(np.uint32), rerr.view(np.uint32))


def test_calibrate_special_blocks_and_frozen_use():
    # zero blocks, a tiny tensor scale (large quotients), a huge one (all codes round to 0)
    x = S.activations(8, 256, seed=5, device=DEV)
    x[0, :16] = 0
    x[1, 16:32] = 1e-3
    for s_g in (1e-6, 0.05, 10.0):
        ts = torch.tensor([s_g], device=DEV)
        sb = Q.nvfp4_calibrate_mse(x, ts)
        rsb, _ = O.calibrate_mse(_host(x), s_g)
        assert np.array_equal(sb.cpu().numpy(), rsb), s_g
    # the calibrated scales feed FROZEN_ALL quantization
    _, _, ts = Q.nvfp4_quantize(x, Q.DYNAMIC)
    sb = Q.nvfp4_calibrate_mse(x, ts)
    codes, _, _ = Q.nvfp4_quantize(x, Q.FROZEN_ALL, tensor_scale=ts, block_scales=sb)
    rc, _, _ = O.quantize(_host(x), O.FROZEN_ALL, s_g=float(ts.cpu()[0]), s_b=sb.cpu().numpy())
    assert np.array_equal(codes.cpu().numpy(), rc)


def test_calibrate_grouped_expert_weights():
    ws = [S.weights(2048, 1024, seed=40 + i, device=DEV) for i in range(3)]
    _, _, ts = Q.nvfp4_quantize_grouped(ws, Q.DYNAMIC)
    sbs = Q.nvfp4_calibrate_mse_grouped(ws, ts)
    torch.cuda.synchronize()
    for i in (0, 2):
        rows = np.random.default_rng(i).choice(2048, 64, replace=False)
        rsb, _ = O.calibrate_mse(_host(ws[i])[rows], float(ts[i].cpu()))
        assert np.array_equal(sbs[i].cpu().numpy()[rows], rsb), i
