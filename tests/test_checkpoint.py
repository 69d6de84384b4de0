"""Save / load of NVFP4 tensors (codes, block scales, tensor scale) is
bit-exact: dequantize(load(save(q))) == dequantize(q), here with the
oracle's quantizer and dequantizer on the host (the GPU form is in
tests/test_gpu_failure.py)."""
import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_quantization_aware_b200 import synthetic as S
from nvfp4_quantization_aware_b200.checkpoint import load_nvfp4, save_nvfp4


def _q(x):
    codes, sb, sg = O.quantize(x.float().numpy(), O.DYNAMIC)
    return torch.from_numpy(codes), torch.from_numpy(sb), torch.tensor([sg], dtype=torch.float32)


def test_round_trip_is_bitwise(tmp_path):
    ws = {"expert0.w_gate": S.weights(96, 256, seed=1), "expert0.w_down": S.weights(256, 96, seed=2),
          "lm_head": S.weights(33, 1040, seed=3)}
    qs = {k: _q(v) for k, v in ws.items()}
    path = str(tmp_path / "q.nvfp4")
    save_nvfp4(path, {k: (*q, "rowmajor") for k, q in qs.items()}, meta={"step": 50, "mode": "frozen"})
    got, meta = load_nvfp4(path)
    assert meta == {"step": 50, "mode": "frozen"}
    assert set(got) == set(ws)
    for k, (c, sb, ts) in qs.items():
        c2, sb2, ts2, layout = got[k]
        assert layout == "rowmajor"
        assert torch.equal(c2, c) and torch.equal(sb2, sb)
        assert ts2.view(torch.int32).item() == ts.view(torch.int32).item()
        cols = ws[k].shape[1]
        _, b1 = O.dequantize(c.numpy(), sb.numpy(), float(ts[0]), cols)
        _, b2 = O.dequantize(c2.numpy(), sb2.numpy(), float(ts2[0]), cols)
        assert np.array_equal(b1, b2)
        # resuming frozen-scale QAD: FROZEN_ALL with the loaded scales reproduces the codes
        c3, _, _ = O.quantize(ws[k].float().numpy(), O.FROZEN_ALL, s_g=float(ts2[0]), s_b=sb2.numpy())
        assert np.array_equal(c3, c.numpy())


def test_mma_layout_and_errors(tmp_path):
    c, sb, ts = _q(S.weights(130, 64, seed=4))
    mma = torch.from_numpy(O.swizzle_scales(sb.numpy(), 64))
    path = str(tmp_path / "m.nvfp4")
    save_nvfp4(path, {"w": (c, mma, ts, "mma")})
    got, _ = load_nvfp4(path)
    assert torch.equal(got["w"][1], mma) and got["w"][3] == "mma"
    with pytest.raises(ValueError):
        save_nvfp4(path, {"w": (c, sb[:, :1], ts, "rowmajor")})
    with open(path, "r+b") as f:
        f.write(b"XXXX")
    with pytest.raises(ValueError):
        load_nvfp4(path)
