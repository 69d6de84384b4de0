"""Failure detection on the device without faulting it, and the checkpoint
round trip of device-quantized tensors.

* A bounded device wait that nothing ends expires after its limit, the
  kernel sets the device error word and returns: nvfp4_device_error reports
  NVFP4_ERR_TIMEOUT with code 1, and the context stays usable (a quantize
  right after matches the oracle).
* Host-side fault injection: the armed call fails with NVFP4_ERR_CUDA
  before launching (the binding raises), leaves no device error behind, and
  the same call succeeds afterwards with the oracle's result; in the MoE
  step the forward and the backward are one outermost call each.
* dequantize(load(save(q))) == dequantize(q) bit for bit for tensors
  quantized on the GPU.
"""
import numpy as np
import pytest
import torch

import oracle as O
import nvfp4_quantization_aware_b200 as Q
from nvfp4_quantization_aware_b200 import synthetic as S
from nvfp4_quantization_aware_b200.checkpoint import load_nvfp4, save_nvfp4
from moe_cases import remap_unused

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _oracle_codes(x):
    return O.quantize(x.float().cpu().numpy(), O.DYNAMIC)


def test_bounded_wait_expires_and_reports_timeout():
    assert Q.nvfp4_device_error() == (0, 0)
    Q.nvfp4_selftest_timeout(200_000)  # ~0.1 ms at 2 GHz
    assert Q.nvfp4_device_error() == (6, 1)  # NVFP4_ERR_TIMEOUT, word 1; the word is cleared
    assert Q.nvfp4_device_error() == (0, 0)
    x = S.activations(64, 512, seed=8, device=DEV)
    codes, sb, ts = Q.nvfp4_quantize(x, Q.DYNAMIC)
    rc, rsb, rsg = _oracle_codes(x)
    assert np.array_equal(codes.cpu().numpy(), rc) and np.array_equal(sb.cpu().numpy(), rsb)


def test_injected_failure_raises_and_the_next_call_works():
    x = S.activations(32, 256, seed=9, device=DEV)
    Q.nvfp4_fault_inject(1)
    try:
        with pytest.raises(Q.NVFP4Error) as e:
            Q.nvfp4_quantize(x, Q.DYNAMIC)
        assert e.value.status == 5
    finally:
        Q.nvfp4_fault_inject(0)
    torch.cuda.synchronize()
    assert Q.nvfp4_device_error() == (0, 0)
    codes, _, _ = Q.nvfp4_quantize(x, Q.DYNAMIC)
    assert np.array_equal(codes.cpu().numpy(), _oracle_codes(x)[0])


def test_injected_failure_in_the_moe_step():
    d = S.moe_layer(seed=4, tokens=130, hidden=256, ffn=256, experts=4, topk=2)
    G = 5
    w = {}
    for k in ("gate", "up", "down"):
        w0 = d["w0_" + k].to(DEV)
        _, sbs, ts = Q.nvfp4_quantize_grouped([w0[g] for g in range(G)], Q.DYNAMIC)
        sb = torch.cat(sbs).contiguous()
        rows, cols = w0.shape[1], w0.shape[2]
        w["w_" + k] = d["w_" + k].to(DEV).reshape(G * rows, cols).contiguous()
        w[k + "_ts"], w[k + "_sb"] = ts, sb
        w[k + "_sb_mma"] = Q.nvfp4_scales_to_mma(sb, G * rows, cols)
    w["x_ts"], w["a_ts"] = d["x_ts"].to(DEV), d["a_ts"].to(DEV)
    step = Q.MoeLayerStep(130, 256, 256, 4, 2, w)
    x, ids, cw, dy = (d[n].to(DEV) for n in ("x", "ids", "combine", "dy"))
    y_ref = step.forward(x, ids, cw).clone()
    grads_ref = [t.clone() for t in step.backward(dy)]
    torch.cuda.synchronize()
    Q.nvfp4_fault_inject(2)  # the forward is call 1 (its parts are not counted), the backward call 2
    try:
        y = step.forward(x, ids, cw)
        with pytest.raises(Q.NVFP4Error):
            step.backward(dy)
    finally:
        Q.nvfp4_fault_inject(0)
    assert torch.equal(y, y_ref)
    grads = step.backward(dy)
    torch.cuda.synchronize()
    assert Q.nvfp4_device_error() == (0, 0)
    for a, b in zip(grads, grads_ref):
        assert torch.equal(a, b)


@pytest.mark.parametrize("layout", ["rowmajor", "mma"])
def test_checkpoint_round_trip_of_device_tensors(tmp_path, layout):
    xs = {"w_gate": S.weights(384, 512, seed=1, device=DEV), "lm_head_part": S.weights(200, 1040, seed=2, device=DEV)}
    lay = Q.SCALES_ROWMAJOR if layout == "rowmajor" else Q.SCALES_MMA
    qs = {k: Q.nvfp4_quantize(v, Q.DYNAMIC, layout=lay) for k, v in xs.items()}
    path = str(tmp_path / "ckpt.nvfp4")
    save_nvfp4(path, {k: (*q, layout) for k, q in qs.items()}, meta={"step": 50})
    got, meta = load_nvfp4(path, device=DEV)
    assert meta["step"] == 50
    for k, (c, sb, ts) in qs.items():
        c2, sb2, ts2, lay2 = got[k]
        assert lay2 == layout
        cols = xs[k].shape[1]
        d1 = Q.nvfp4_dequantize(c, sb, ts, cols, layout=lay)
        d2 = Q.nvfp4_dequantize(c2, sb2, ts2, cols, layout=lay)
        assert torch.equal(d1.view(torch.int16), d2.view(torch.int16))
