"""Top-k KL distillation loss, plain and slow -- TEST INFRASTRUCTURE ONLY.

Only the test suite, the smoke check and bench.py's CPU-baseline legs may
import this module; the product library never does.

The Qwen3.6-35B-A3B W4A4 tutorial (section "3. QAD") trains with the KL loss
restricted to the teacher's top-k vocabulary entries (`--logit_kl_topk
4096`), which avoids materialising dense [seq, vocab] probabilities.  The
page does not say how the two distributions are normalised on the selected
set; the reading here (the plainest one): both softmaxes are renormalised
over the teacher's top-k set S of each row,
    p_t^S = softmax(z_t[S] / T),  p_s^S = softmax(z_s[S] / T),
    KL_i  = sum_{v in S} p_t^S (log p_t^S - log p_s^S),
    dz_s[v] = grad_scale * (p_s^S[v] - p_t^S[v]) / T for v in S, 0 elsewhere.
S holds the k largest teacher logits; among equal logits the smaller
vocabulary index comes first (the order of a stable descending sort), so S
is unique.  k >= V selects the whole row (the full-vocabulary loss).

The loss and gradient on S are the pinned float64 oracle `oracle.kl` applied
to the gathered entries.
"""
from __future__ import annotations

import numpy as np

from . import kl


def topk_set(teacher_row: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest entries, ties by smaller index, in that order."""
    order = np.argsort(-np.asarray(teacher_row, dtype=np.float64), kind="stable")
    return order[:min(k, order.shape[0])]


def kl_topk(teacher: np.ndarray, student: np.ndarray, k: int, T: float = 1.0, grad_scale: float | None = None,
            want_grad: bool = True):
    """Returns (loss, row_kl [rows], grad [rows, V] or None) in float64."""
    t = np.asarray(teacher, dtype=np.float64)
    s = np.asarray(student, dtype=np.float64)
    rows, V = t.shape
    if grad_scale is None:
        grad_scale = 1.0 / rows if rows else 1.0
    row_kl = np.zeros(rows)
    grad = np.zeros((rows, V)) if want_grad else None
    for i in range(rows):
        sel = topk_set(t[i], k)
        _, rk, g = kl(t[i:i + 1, sel], s[i:i + 1, sel], T=T, grad_scale=grad_scale, want_grad=want_grad, threads=1)
        row_kl[i] = rk[0]
        if want_grad:
            grad[i, sel] = g[0]
    loss = float(row_kl.sum() / rows) if rows else 0.0
    return loss, row_kl, grad
