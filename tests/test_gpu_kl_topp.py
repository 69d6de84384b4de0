"""GPU parity of the top-p KL loss + dLogits (qad_kl_topp_fwd_bwd) against the
oracle (oracle/topp.py).  The set size |S| of every row must be a valid top-p
size: its cumulative teacher probability (float64, top-k order) reaches p and
one entry fewer does not, within TOL (the kernel sums hardware exponentials
in 64-bit fixed point); where no prefix sum lies within TOL of p it must equal
the oracle's exactly.  Given |S|, the loss, per-row KL and dLogits are those
of the top-k oracle with k = |S| (1e-4 / 1e-3 relative, zeros outside S)."""
import numpy as np
import pytest
import torch

import oracle as O
from oracle import topk as OT
from oracle import topp as OP
import nvfp4_quantization_aware_b200 as Q
from nvfp4_quantization_aware_b200 import synthetic as S

pytestmark = pytest.mark.gpu
DEV = "cuda"
LOSS_RTOL = 1e-4
GRAD_RTOL = 1e-3
TOL = 1e-6


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _round(g, dtype):
    if dtype == torch.bfloat16:
        return O.bf16_bits_to_f32(O.bf16_round(g)).astype(np.float64)
    return g.astype(np.float32).astype(np.float64)


def _check(t, s, p, T=1.0, grad_scale=None):
    loss, row, g, ks = Q.qad_kl_topp_fwd_bwd(t, s, p, temperature=T, grad_scale=grad_scale, want_row_kl=True,
                                             want_row_k=True)
    torch.cuda.synchronize()
    assert Q.nvfp4_device_error()[0] == 0
    th, sh = t.double().cpu().numpy(), s.double().cpu().numpy()
    rows, V = th.shape
    ks = ks.cpu().numpy()
    for i in range(rows):
        m = int(ks[i])
        if p >= 1.0:
            assert m == V
            continue
        assert 1 <= m <= V
        cum = OP.topp_cumulative(th[i], T)
        assert cum[m - 1] >= p - TOL, (i, m, cum[m - 1])
        assert m == 1 or cum[m - 2] < p + TOL, (i, m, cum[m - 2])
        m_ref = OP.topp_count(th[i], p, T)
        clear = abs(cum[m_ref - 1] - p) > TOL and (m_ref == 1 or abs(cum[m_ref - 2] - p) > TOL)
        if clear:
            assert m == m_ref, (i, m, m_ref)
    gs = (1.0 / rows) if grad_scale is None else grad_scale
    ref_loss, ref_row, ref_g = OP.kl_rows_k(th, sh, ks, T=T, grad_scale=gs)
    got_row = row.cpu().numpy().astype(np.float64)
    assert np.allclose(got_row, ref_row, rtol=LOSS_RTOL, atol=1e-6 * max(1.0, np.abs(ref_row).max()))
    assert abs(float(loss.cpu()[0]) - ref_loss) <= LOSS_RTOL * abs(ref_loss) + 1e-7
    got_g = g.double().cpu().numpy()
    for i in range(rows):
        out = np.setdiff1d(np.arange(V), OT.topk_set(th[i], int(ks[i])))
        assert np.all(got_g[i, out] == 0.0), i
    if np.any(ref_g != 0):
        assert _rel(got_g, _round(ref_g, t.dtype)) <= GRAD_RTOL
    return ks


@pytest.mark.parametrize("V", [16, 1003, 8193, 40000, 131072])
@pytest.mark.parametrize("p", [0.5, 0.9, 0.999])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_topp_vocab_sizes(V, p, dtype):
    t, s = S.logits_pair(4, V, seed=V + int(p * 1000), device=DEV, dtype=dtype)
    _check(t, s, p)


def test_topp_limits_temperature_and_grad_scale():
    t, s = S.logits_pair(5, 5000, seed=3, device=DEV, dtype=torch.bfloat16)
    ks = _check(t, s, 1e-9)
    assert np.all(ks == 1)
    ks = _check(t, s, 1.0)
    assert np.all(ks == 5000)
    _check(t, s, 0.8, T=2.0, grad_scale=0.3)
    _check(t, s, 0.8, T=0.5)
    # p >= 1 is the full-vocabulary loss: both kernels are within the loss bar
    # of the oracle, so within twice the bar of each other
    l1, r1, g1, _ = Q.qad_kl_topp_fwd_bwd(t, s, 1.5, want_row_kl=True)
    l2, r2, g2 = Q.qad_kl_fwd_bwd(t, s, want_row_kl=True)
    torch.cuda.synchronize()
    assert torch.allclose(r1, r2, rtol=2 * LOSS_RTOL, atol=2e-6)
    assert float((g1.float() - g2.float()).norm() / g2.float().norm()) <= 2e-3


@pytest.mark.parametrize("V,span,p", [(40000, 3, 0.6), (131072, 60, 0.95), (1003, 3, 0.3)])
def test_topp_ties_at_the_boundary(V, span, p):
    # integer-valued teacher logits: the boundary falls inside a group of
    # equal logits spread over the row's CTAs, ranked by index
    g = torch.Generator().manual_seed(V + span)
    t = torch.randint(-span, span + 1, (4, V), generator=g).to(torch.bfloat16)
    s = (t.float() + torch.randn(4, V, generator=g)).to(torch.bfloat16)
    _check(t.to(DEV), s.to(DEV), p)


def test_topp_uniform_rows_take_ceil_p_v():
    t = torch.zeros(3, 1000, dtype=torch.bfloat16, device=DEV)
    s, _ = S.logits_pair(3, 1000, seed=8, device=DEV, dtype=torch.bfloat16)
    ks = _check(t, s, 0.3005)
    assert np.all(ks == 301)


def test_topp_distill_logits_rows():
    d = S.distill_logits(seed=2, device=DEV, rows=32)
    _check(d["teacher"], d["student"], 0.95)
