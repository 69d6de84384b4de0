"""HostGroupedQuantizer (pinned host tensors in, pinned host results out, the
copies of one chunk overlapped with the kernels of another) against the
oracle and against the device-resident grouped quantize: codes, block scales
and tensor scales bit for bit, over several chunks and repeated runs."""
import numpy as np
import pytest
import torch

import oracle as O
import nvfp4_quantization_aware_b200 as Q
from nvfp4_quantization_aware_b200 import synthetic as S

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _tensors(dtype=torch.bfloat16):
    shapes = [(256, 1024), (64, 2048), (1000, 32), (512, 512), (3, 48), (2048, 256), (128, 4096)]
    xs = [S.weights(r, c, seed=40 + i, device="cpu").to(dtype) for i, (r, c) in enumerate(shapes)]
    return [x.pin_memory() for x in xs]


def _check_against_oracle(hq, xs, modes):
    for i, x in enumerate(xs):
        xh = x.float().numpy()
        ref_codes, ref_sb, ref_sg = O.quantize(xh, O.DYNAMIC)
        assert np.float32(hq.tensor_scales[i].item()) == np.float32(ref_sg), i
        assert np.array_equal(hq.block_scales[i].numpy(), ref_sb), i
        assert np.array_equal(hq.codes[i].numpy(), ref_codes), i


@pytest.mark.parametrize("passes", [(Q.DYNAMIC,), (Q.DYNAMIC, Q.FROZEN_ALL)])
def test_host_pipeline_matches_oracle_over_chunks_and_runs(passes):
    xs = _tensors()
    hq = Q.HostGroupedQuantizer(xs, DEV, passes=passes, chunk_bytes=1 << 20)
    assert len(hq.chunks) > 3
    for _ in range(3):
        hq.run()
        torch.cuda.synchronize()
        assert Q.nvfp4_device_error()[0] == 0
        _check_against_oracle(hq, xs, passes)


def test_host_pipeline_equals_device_grouped_quantize_f32():
    xs = _tensors(torch.float32)
    hq = Q.HostGroupedQuantizer(xs, DEV, chunk_bytes=2 << 20)
    hq.run()
    torch.cuda.synchronize()
    dx = [x.to(DEV) for x in xs]
    codes, sbs, ts = Q.nvfp4_quantize_grouped(dx, Q.DYNAMIC)
    torch.cuda.synchronize()
    for i in range(len(xs)):
        assert torch.equal(hq.codes[i], codes[i].cpu()), i
        assert torch.equal(hq.block_scales[i], sbs[i].cpu()), i
    assert torch.equal(hq.tensor_scales, ts.cpu())


def test_host_pipeline_frozen_global_uses_given_tensor_scales():
    xs = _tensors()
    given = [np.float32(O.quantize(x.float().numpy(), O.DYNAMIC)[2] * 1.5) for x in xs]
    hq = Q.HostGroupedQuantizer(xs, DEV, passes=(Q.FROZEN_GLOBAL,), tensor_scales=given, chunk_bytes=1 << 20)
    hq.run()
    torch.cuda.synchronize()
    for i, x in enumerate(xs):
        ref_codes, ref_sb, ref_sg = O.quantize(x.float().numpy(), O.FROZEN_GLOBAL, s_g=float(given[i]))
        assert np.float32(hq.tensor_scales[i].item()) == given[i]
        assert np.array_equal(hq.block_scales[i].numpy(), ref_sb), i
        assert np.array_equal(hq.codes[i].numpy(), ref_codes), i


def test_host_pipeline_runs_on_a_side_stream_in_order():
    xs = _tensors()
    hq = Q.HostGroupedQuantizer(xs, DEV, passes=(Q.DYNAMIC, Q.FROZEN_ALL), chunk_bytes=1 << 20)
    s = torch.cuda.Stream(DEV)
    with torch.cuda.stream(s):
        hq.run(s)
        # work queued on the caller's stream after run() sees the results
        after = hq.d_codes[0].clone()
    s.synchronize()
    assert torch.equal(after.cpu(), hq.codes[0])
