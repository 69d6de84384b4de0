"""The sharded quantize / KL helpers with the CUDA operations on one GPU and
the collectives emulated (row shards, the max and the sum combined
directly), compared with the oracle on the whole tensor:

* sharded dynamic quantization: codes, block scales and the tensor scale
  bit-exact against oracle.quantize(whole tensor, DYNAMIC) (the block scales
  depend only on a block and s_g, and s_g only on the global amax);
* sharded KL: the loss within 1e-4 relative, per-row KL within 1e-4 and the
  dLogits within 1e-3 relative Frobenius of oracle.kl on the whole batch
  (grad_scale = 1 / all rows on every shard).
"""
import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_quantization_aware_b200 import parallel as P
from nvfp4_quantization_aware_b200 import synthetic as S

pytestmark = pytest.mark.gpu
DEV = "cuda"
LOSS_RTOL = 1e-4
GRAD_RTOL = 1e-3


def _rel_fro(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


@pytest.mark.parametrize("shards", [2, 3])
def test_sharded_dynamic_quantize_matches_oracle(shards):
    ops = P.cuda_ops()
    ws = [S.weights(512, 1024, seed=60 + i, device=DEV) for i in range(3)] + [S.weights(33, 272, seed=9, device=DEV)]
    # uneven cuts, one shard of a single row and one empty-free ragged shard
    cuts = [np.linspace(0, w.shape[0], shards + 1).astype(int) for w in ws]
    cuts[1][1] = 1
    parts = [[w[c[r]:c[r + 1]] for w, c in zip(ws, cuts)] for r in range(shards)]
    amax = ops.tensor_amax(parts[0])
    for r in range(1, shards):
        amax = torch.maximum(amax, ops.tensor_amax(parts[r]))  # the all-reduce(max)
    ts = ops.scale_from_amax(amax)
    got = [ops.quantize_frozen_global(parts[r], ts) for r in range(shards)]
    torch.cuda.synchronize()
    for i, w in enumerate(ws):
        codes, sb, sg = O.quantize(w.float().cpu().numpy(), O.DYNAMIC)
        assert np.float32(sg).view(np.int32) == ts[i].cpu().numpy().view(np.int32), i
        c = torch.cat([got[r][0][i] for r in range(shards)]).cpu().numpy()
        b = torch.cat([got[r][1][i] for r in range(shards)]).cpu().numpy()
        assert np.array_equal(c, codes), i
        assert np.array_equal(b, sb), i


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_sharded_kl_matches_oracle(dtype):
    t, s = S.logits_pair(48, 40000, seed=3, device=DEV, dtype=dtype)
    ops = P.cuda_ops()
    R = t.shape[0]
    cuts = [0, 17, 18, 48]  # three shards, one of a single row
    rows, grads = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        row, g = ops.kl(t[a:b], s[a:b], 1.0, 1.0 / R)
        rows.append(row)
        grads.append(g)
    loss = sum(float(r.double().sum()) for r in rows) / R  # the all-reduce(sum)
    torch.cuda.synchronize()
    ref_loss, ref_row, ref_g = O.kl(t.double().cpu().numpy(), s.double().cpu().numpy(), T=1.0, grad_scale=1.0 / R)
    assert abs(loss - ref_loss) <= LOSS_RTOL * abs(ref_loss)
    got_row = torch.cat(rows).double().cpu().numpy()
    assert np.allclose(got_row, ref_row, rtol=LOSS_RTOL, atol=1e-6 * np.abs(ref_row).max())
    if dtype == torch.bfloat16:
        ref_g = O.bf16_bits_to_f32(O.bf16_round(ref_g)).astype(np.float64)
    else:
        ref_g = ref_g.astype(np.float32).astype(np.float64)
    got_g = torch.cat(grads).double().cpu().numpy()
    assert _rel_fro(got_g, ref_g) <= GRAD_RTOL
