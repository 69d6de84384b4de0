"""The dense FP4 MMA throughput probe used for the GEMM's roofline: it runs,
leaves no device error, reports the documented flop count, and measures a
throughput between the GEMM's and the datasheet's (a probe that does no work
would read far above it)."""
import pytest
import torch

import nvfp4_quantization_aware_b200 as Q

pytestmark = pytest.mark.gpu


def test_probe_runs_and_counts_flop():
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    st = torch.cuda.current_stream()
    Q.nvfp4_probe_fp4_mma(100, sms, st)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    flop = Q.nvfp4_probe_fp4_mma(2000, sms, st)
    e1.record(st)
    torch.cuda.synchronize()
    assert flop == 2.0 * 128 * 256 * 64 * 4 * 2000 * sms
    assert Q.nvfp4_device_error() == (0, 0)
    tflops = flop / (e0.elapsed_time(e1) * 1e-3) / 1e12
    assert 1000.0 < tflops < 12000.0, tflops


def test_probe_rejects_bad_arguments():
    with pytest.raises(RuntimeError):
        Q.nvfp4_probe_fp4_mma(0, 1)
