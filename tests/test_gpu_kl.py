"""GPU parity of the fused KL distillation loss + dLogits against the oracle.

Bars: loss and per-row KL within 1e-4 relative; dLogits within 1e-3 relative
Frobenius norm per checked row set, against the oracle's float64 gradient
rounded to the output dtype (bf16 rounding alone would cost ~1.5e-3 against
unrounded values).
"""
import numpy as np
import pytest
import torch

import oracle as O
import nvfp4_quantization_aware_b200 as Q
from nvfp4_quantization_aware_b200 import synthetic as S

pytestmark = pytest.mark.gpu
DEV = "cuda"
LOSS_RTOL = 1e-4
GRAD_RTOL = 1e-3


def _rel_fro(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _ref_grad_in_dtype(g: np.ndarray, dtype) -> np.ndarray:
    if dtype == torch.bfloat16:
        return O.bf16_bits_to_f32(O.bf16_round(g)).astype(np.float64)
    return g.astype(np.float32).astype(np.float64)


def _check(t: torch.Tensor, s: torch.Tensor, T: float = 1.0, grad_scale=None, rows_to_check=None):
    loss, row_kl, grad = Q.qad_kl_fwd_bwd(t, s, temperature=T, grad_scale=grad_scale, want_row_kl=True)
    torch.cuda.synchronize()
    R = t.shape[0]
    idx = np.arange(R) if rows_to_check is None else np.asarray(rows_to_check)
    th = t[idx].double().cpu().numpy()
    sh = s[idx].double().cpu().numpy()
    gs = (1.0 / R) if grad_scale is None else grad_scale
    ref_loss, ref_row, ref_g = O.kl(th, sh, T=T, grad_scale=gs)
    got_row = row_kl.cpu().numpy()[idx].astype(np.float64)
    assert np.allclose(got_row, ref_row, rtol=LOSS_RTOL, atol=1e-6 * max(1.0, np.abs(ref_row).max())), \
        float(np.max(np.abs(got_row - ref_row) / np.abs(ref_row)))
    if rows_to_check is None:
        assert abs(float(loss.cpu()[0]) - ref_loss) <= LOSS_RTOL * abs(ref_loss) + 1e-7
    else:
        # the loss is the mean of the per-row values (a property at any size)
        assert abs(float(loss.cpu()[0]) - row_kl.double().mean().item()) <= 1e-6 * abs(row_kl.double().mean().item()) + 1e-9
    got_g = grad[idx].double().cpu().numpy()
    assert _rel_fro(got_g, _ref_grad_in_dtype(ref_g, t.dtype)) <= GRAD_RTOL
    return loss, row_kl, grad


def test_tiny_qad_logits_fp32():
    d = S.tiny_qad_linear(seed=0, device=DEV)
    _check(d["teacher"], d["student"])


@pytest.mark.parametrize("V", [16, 1000, 1003, 8193, 40000, 65560, 131072])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_vocab_sizes(V, dtype):
    # covers cluster sizes 1..8, ragged tails shorter than one 16-byte vector
    t, s = S.logits_pair(5, V, seed=V, device=DEV, dtype=dtype)
    _check(t, s)


def test_temperature_and_grad_scale():
    t, s = S.logits_pair(9, 5000, seed=1, device=DEV, dtype=torch.bfloat16)
    _check(t, s, T=2.5, grad_scale=0.37)
    _check(t, s, T=0.6)


def test_row_stride_and_forward_only():
    t0, s0 = S.logits_pair(7, 3000, seed=2, device=DEV, dtype=torch.float32)
    t = torch.zeros(7, 3008, device=DEV)
    s = torch.zeros(7, 3008, device=DEV)
    t[:, :3000] = t0
    s[:, :3000] = s0
    t, s = t[:, :3000], s[:, :3000]
    assert t.stride(0) == 3008
    loss, row, g = Q.qad_kl_fwd_bwd(t, s, want_grad=False, want_row_kl=True)
    assert g is None
    ref_loss, ref_row, _ = O.kl(t0.double().cpu().numpy(), s0.double().cpu().numpy(), want_grad=False)
    assert abs(float(loss.cpu()[0]) - ref_loss) <= LOSS_RTOL * ref_loss
    _check(t, s)


def test_identical_logits_give_zero():
    t, _ = S.logits_pair(6, 7000, seed=3, device=DEV, dtype=torch.bfloat16)
    loss, row, g = Q.qad_kl_fwd_bwd(t, t.clone(), want_row_kl=True)
    assert abs(float(loss.cpu()[0])) < 1e-5
    assert float(g.float().abs().max().cpu()) < 1e-7


def test_gradient_rows_sum_to_zero():
    t, s = S.logits_pair(4, 12345, seed=4, device=DEV, dtype=torch.float32)
    _, _, g = Q.qad_kl_fwd_bwd(t, s)
    sums = g.double().sum(1).abs().max().item()
    assert sums < 1e-6 * g.double().abs().sum(1).max().item() + 1e-12


def test_autograd_wrapper():
    t, s = S.logits_pair(8, 4096, seed=5, device=DEV, dtype=torch.float32)
    s = s.clone().requires_grad_(True)
    loss = Q.kl_distill_loss(s, t)
    (loss * 3.0).backward()
    ref_loss, _, ref_g = O.kl(t.double().cpu().numpy(), s.detach().double().cpu().numpy())
    assert abs(loss.item() - ref_loss) <= LOSS_RTOL * ref_loss
    assert _rel_fro(s.grad.double().cpu().numpy(), 3.0 * ref_g) <= GRAD_RTOL


def test_distill_logits_vocab_rows():
    # the 131072-entry vocabulary at full width, 64 rows, every row checked
    d = S.distill_logits(seed=0, device=DEV, rows=64)
    _check(d["teacher"], d["student"])


@pytest.mark.slow
def test_distill_logits_full_size_sampled():
    # 16384 x 131072 bf16 (2^31 logits per tensor); the oracle checks 48
    # seeded rows, the loss is checked as the mean of all per-row values.
    d = S.distill_logits(seed=0, device=DEV)
    rows = np.random.default_rng(0).choice(16384, 48, replace=False)
    rows = np.concatenate([[0, 16383], rows])
    _check(d["teacher"], d["student"], rows_to_check=rows)


# The persistent form (aligned bf16 rows, vocabulary a multiple of 8, at least
# 64 rows, cluster of 2 or more): rows spread over the resident clusters, the
# shared-memory ring wrapping several times per cluster.
@pytest.mark.parametrize("rows,V", [(64, 131072), (100, 131072), (70, 40000), (300, 16392), (1000, 32768)])
def test_persistent_rows(rows, V):
    t, s = S.logits_pair(rows, V, seed=rows + V, device=DEV, dtype=torch.bfloat16)
    _check(t, s, T=2.5, grad_scale=0.37)


def test_persistent_negative_grad_scale_and_stride():
    rows, V = 80, 65536
    t0, s0 = S.logits_pair(rows, V, seed=11, device=DEV, dtype=torch.bfloat16)
    t = torch.zeros(rows, V + 64, dtype=torch.bfloat16, device=DEV)
    s = torch.zeros(rows, V + 64, dtype=torch.bfloat16, device=DEV)
    t[:, :V] = t0
    s[:, :V] = s0
    t, s = t[:, :V], s[:, :V]
    _check(t, s, grad_scale=-0.5)
    loss, row, g = Q.qad_kl_fwd_bwd(t, s, want_grad=False, want_row_kl=True)
    assert g is None
    ref_loss, ref_row, _ = O.kl(t0.double().cpu().numpy(), s0.double().cpu().numpy(), want_grad=False)
    assert abs(float(loss.cpu()[0]) - ref_loss) <= LOSS_RTOL * ref_loss
