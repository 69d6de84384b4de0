"""Top-p (nucleus) KL distillation loss, plain and slow -- TEST INFRASTRUCTURE ONLY.

Only the test suite, the smoke check and bench.py's CPU-baseline legs may
import this module; the product library never does.

The Qwen3.6-35B-A3B W4A4 tutorial (section "5. 评估", where it analyses the
runs that hit the output-length cap) recommends, for the next QAD run,
selecting the teacher's top-p entries instead of the top-k ones, so that the
loss covers the teacher's entropy; it gives no formula.  The reading here (the
plainest one, and the top-k form of `oracle.topk` otherwise unchanged):
  * the teacher's probabilities at temperature T, p_t = softmax(z_t / T);
  * the entries ordered by decreasing teacher logit, equal logits by smaller
    vocabulary index (the top-k order);
  * S = the shortest prefix of that order whose teacher probability sum
    reaches p, for 0 < p < 1; p >= 1 selects the whole row;
  * loss and gradient: those of the top-k loss with k = |S| (both softmaxes
    renormalised over S, gradient zero outside S).
"""
from __future__ import annotations

import numpy as np

from .topk import kl_topk, topk_set


def topp_count(teacher_row: np.ndarray, p: float, T: float = 1.0) -> int:
    """|S| for one row: the smallest m whose first m entries (top-k order)
    carry teacher probability >= p, in float64; the whole row for p >= 1."""
    z = np.asarray(teacher_row, dtype=np.float64)
    V = z.shape[0]
    if p >= 1.0:
        return V
    w = np.exp((z - z.max()) / T)
    prob = w / w.sum()
    cum = np.cumsum(prob[topk_set(z, V)])
    return min(int(np.searchsorted(cum, p, side="left")) + 1, V)


def topp_cumulative(teacher_row: np.ndarray, T: float = 1.0) -> np.ndarray:
    """Cumulative teacher probability along the top-k order (float64)."""
    z = np.asarray(teacher_row, dtype=np.float64)
    w = np.exp((z - z.max()) / T)
    prob = w / w.sum()
    return np.cumsum(prob[topk_set(z, z.shape[0])])


def kl_rows_k(teacher: np.ndarray, student: np.ndarray, ks, T: float = 1.0, grad_scale: float | None = None):
    """Top-k loss with a k per row: (loss, row_kl [rows], grad [rows, V])."""
    t = np.asarray(teacher, dtype=np.float64)
    s = np.asarray(student, dtype=np.float64)
    rows, V = t.shape
    if grad_scale is None:
        grad_scale = 1.0 / rows if rows else 1.0
    row_kl = np.zeros(rows)
    grad = np.zeros((rows, V))
    for i in range(rows):
        _, rk, g = kl_topk(t[i:i + 1], s[i:i + 1], int(ks[i]), T=T, grad_scale=grad_scale)
        row_kl[i] = rk[0]
        grad[i] = g[0]
    loss = float(row_kl.sum() / rows) if rows else 0.0
    return loss, row_kl, grad


def kl_topp(teacher: np.ndarray, student: np.ndarray, p: float, T: float = 1.0, grad_scale: float | None = None):
    """Returns (loss, row_kl [rows], grad [rows, V], ks [rows]) in float64."""
    t = np.asarray(teacher, dtype=np.float64)
    ks = np.array([topp_count(t[i], p, T) for i in range(t.shape[0])], dtype=np.int64)
    loss, row_kl, grad = kl_rows_k(t, student, ks, T=T, grad_scale=grad_scale)
    return loss, row_kl, grad, ks
