"""GPU parity of the top-k KL loss + dLogits (qad_kl_topk_fwd_bwd) against the
oracle (oracle/topk.py).  The selected set is unique (ties by index), so the
gradient must be exactly zero outside it; loss and per-row KL within 1e-4
relative, dLogits within 1e-3 relative Frobenius against the oracle rounded
to the output dtype."""
import numpy as np
import pytest
import torch

import oracle as O
from oracle import topk as OT
import nvfp4_quantization_aware_b200 as Q
from nvfp4_quantization_aware_b200 import synthetic as S

pytestmark = pytest.mark.gpu
DEV = "cuda"
LOSS_RTOL = 1e-4
GRAD_RTOL = 1e-3


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _round(g, dtype):
    if dtype == torch.bfloat16:
        return O.bf16_bits_to_f32(O.bf16_round(g)).astype(np.float64)
    return g.astype(np.float32).astype(np.float64)


def _check(t, s, k, T=1.0, grad_scale=None):
    loss, row, g = Q.qad_kl_topk_fwd_bwd(t, s, k, temperature=T, grad_scale=grad_scale, want_row_kl=True)
    torch.cuda.synchronize()
    assert Q.nvfp4_device_error()[0] == 0
    th, sh = t.double().cpu().numpy(), s.double().cpu().numpy()
    gs = (1.0 / t.shape[0]) if grad_scale is None else grad_scale
    ref_loss, ref_row, ref_g = OT.kl_topk(th, sh, k, T=T, grad_scale=gs)
    got_row = row.cpu().numpy().astype(np.float64)
    assert np.allclose(got_row, ref_row, rtol=LOSS_RTOL, atol=1e-6 * max(1.0, np.abs(ref_row).max())), \
        (got_row, ref_row)
    assert abs(float(loss.cpu()[0]) - ref_loss) <= LOSS_RTOL * abs(ref_loss) + 1e-7
    got_g = g.double().cpu().numpy()
    for i in range(t.shape[0]):
        out = np.setdiff1d(np.arange(t.shape[1]), OT.topk_set(th[i], k))
        assert np.all(got_g[i, out] == 0.0), i
    if np.any(ref_g != 0):
        assert _rel(got_g, _round(ref_g, t.dtype)) <= GRAD_RTOL
    return loss, row, g


@pytest.mark.parametrize("V,k", [(16, 1), (16, 7), (16, 16), (16, 40), (1003, 100), (8193, 4096),
                                 (40000, 4096), (131072, 4096), (131072, 1)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_topk_vocab_sizes(V, k, dtype):
    t, s = S.logits_pair(5, V, seed=V + k, device=DEV, dtype=dtype)
    _check(t, s, k)


@pytest.mark.parametrize("V,k,span", [(40000, 3000, 3), (1003, 500, 3), (131072, 4096, 3), (131072, 4096, 60)])
def test_topk_ties_split_across_the_cluster(V, k, span):
    # integer-valued logits in [-span, span]: groups of equal teacher logits,
    # the k-th falls inside one, whose members span several CTAs of the row's
    # cluster (a few hundred ties per CTA with span 60, thousands with 3)
    g = torch.Generator().manual_seed(V + span)
    t = torch.randint(-span, span + 1, (4, V), generator=g).to(torch.bfloat16)
    s = (t.float() + torch.randn(4, V, generator=g)).to(torch.bfloat16)
    _check(t.to(DEV), s.to(DEV), k)


def test_topk_temperature_grad_scale_and_k_at_least_vocab_equals_full():
    t, s = S.logits_pair(6, 5000, seed=9, device=DEV, dtype=torch.bfloat16)
    _check(t, s, 700, T=2.0, grad_scale=0.3)
    l1, r1, g1 = Q.qad_kl_topk_fwd_bwd(t, s, 5000, want_row_kl=True)
    l2, r2, g2 = Q.qad_kl_fwd_bwd(t, s, want_row_kl=True)
    torch.cuda.synchronize()
    assert torch.allclose(r1, r2, rtol=1e-5, atol=1e-7)
    assert float((g1.float() - g2.float()).norm() / g2.float().norm()) <= 2e-3


def test_topk_distill_logits_rows():
    # the 131072-entry vocabulary, k = 4096 (the pages' setting), 64 rows
    d = S.distill_logits(seed=1, device=DEV, rows=64)
    _check(d["teacher"], d["student"], 4096)
