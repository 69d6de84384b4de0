"""The sharded quantize / KL helpers with the CUDA operations on one GPU,
with the collectives emulated (two row shards, max and sum combined
directly): the sharded dynamic quantization is bit-exact against the
whole-tensor DYNAMIC call, and the sharded KL gives the whole-batch loss and
the same dLogits."""
import numpy as np
import pytest
import torch

import nvfp4_quantization_aware_b200 as Q
from nvfp4_quantization_aware_b200 import parallel as P
from nvfp4_quantization_aware_b200 import synthetic as S

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_sharded_dynamic_quantize_equals_whole_tensor():
    ops = P.cuda_ops()
    ws = [S.weights(2048, 1024, seed=60 + i, device=DEV) for i in range(3)] + [S.weights(33, 272, seed=9, device=DEV)]
    cut = [700, 1500, 1, 20]
    lo = [w[:c] for w, c in zip(ws, cut)]
    hi = [w[c:] for w, c in zip(ws, cut)]
    amax = torch.maximum(ops.tensor_amax(lo), ops.tensor_amax(hi))  # the all-reduce(max)
    ts = ops.scale_from_amax(amax)
    c_lo, sb_lo = ops.quantize_frozen_global(lo, ts)
    c_hi, sb_hi = ops.quantize_frozen_global(hi, ts)
    rc, rsb, rts = Q.nvfp4_quantize_grouped(ws, Q.DYNAMIC)
    torch.cuda.synchronize()
    assert torch.equal(ts.view(torch.int32), rts.view(torch.int32))
    for i in range(len(ws)):
        assert torch.equal(torch.cat([c_lo[i], c_hi[i]]), rc[i]), i
        assert torch.equal(torch.cat([sb_lo[i], sb_hi[i]]), rsb[i]), i


def test_sharded_kl_equals_whole_batch():
    t, s = S.logits_pair(64, 131072, seed=3, device=DEV)
    ops = P.cuda_ops()
    R = t.shape[0]
    row_a, g_a = ops.kl(t[:24], s[:24], 1.0, 1.0 / R)
    row_b, g_b = ops.kl(t[24:], s[24:], 1.0, 1.0 / R)
    loss = (row_a.double().sum() + row_b.double().sum()) / R  # the all-reduce(sum)
    full_loss, full_row, full_g = Q.qad_kl_fwd_bwd(t, s, want_row_kl=True)
    torch.cuda.synchronize()
    assert abs(float(loss) - float(full_loss)) <= 1e-6 * abs(float(full_loss))
    assert torch.equal(torch.cat([g_a, g_b]), full_g)
    assert torch.equal(torch.cat([row_a, row_b]), full_row)
