"""Pins of the top-k KL oracle (oracle/topk.py): the selection against a
brute-force search over all k-subsets, the k >= V case against the
full-vocabulary loss, k = 1, KL >= 0, independence from everything outside
the selected set, and the gradient against central finite differences."""
import itertools

import numpy as np
import pytest

import oracle as O
from oracle import topk as OT


def _valid_topk(row, S):
    inside = set(S.tolist())
    for i in inside:
        for j in range(len(row)):
            if j in inside:
                continue
            if not (row[i] > row[j] or (row[i] == row[j] and i < j)):
                return False
    return True


@pytest.mark.parametrize("seed", range(6))
def test_selection_is_the_unique_valid_subset(seed):
    rng = np.random.default_rng(seed)
    V, k = 8, 3
    row = rng.integers(-2, 3, V).astype(np.float64)  # many ties
    got = OT.topk_set(row, k)
    valid = [np.array(c) for c in itertools.combinations(range(V), k) if _valid_topk(row, np.array(c))]
    assert len(valid) == 1
    assert sorted(got.tolist()) == valid[0].tolist()


def test_k_at_least_vocab_is_the_full_loss():
    rng = np.random.default_rng(1)
    t = rng.normal(0, 3, (4, 50))
    s = t + rng.normal(0, 1, (4, 50))
    for k in (50, 80):
        loss, row, g = OT.kl_topk(t, s, k)
        ref_loss, ref_row, ref_g = O.kl(t, s)
        assert np.allclose(row, ref_row, rtol=1e-13, atol=1e-15)
        assert np.allclose(g, ref_g, rtol=1e-12, atol=1e-16)
        assert abs(loss - ref_loss) <= 1e-13 * abs(ref_loss)


def test_single_entry_gives_zero():
    rng = np.random.default_rng(2)
    t = rng.normal(0, 3, (3, 40))
    s = rng.normal(0, 3, (3, 40))
    loss, row, g = OT.kl_topk(t, s, 1)
    assert loss == 0.0 and np.all(row == 0.0) and np.all(g == 0.0)


def test_nonnegative_and_local_to_the_selected_set():
    rng = np.random.default_rng(3)
    t = rng.normal(0, 3, (5, 200))
    s = t + rng.normal(0, 1, (5, 200))
    k = 17
    loss, row, g = OT.kl_topk(t, s, k)
    assert np.all(row >= 0.0)
    sets = [OT.topk_set(t[i], k) for i in range(5)]
    s2 = s.copy()
    t2 = t.copy()
    for i, S in enumerate(sets):
        out = np.setdiff1d(np.arange(200), S)
        s2[i, out] += rng.normal(0, 5, out.shape)          # any student values outside S
        kth = t[i, S].min()
        t2[i, out] = np.minimum(t2[i, out], kth) - 1.0      # teacher values outside S, still below S
        assert np.all(g[i, out] == 0.0)
    loss2, row2, g2 = OT.kl_topk(t2, s2, k)
    assert np.allclose(row2, row, rtol=1e-13) and np.allclose(g2, g, rtol=1e-12, atol=1e-18)


def test_gradient_matches_finite_differences():
    rng = np.random.default_rng(4)
    t = rng.normal(0, 2, (2, 30))
    s = t + rng.normal(0, 1, (2, 30))
    k, T = 9, 1.7
    _, _, g = OT.kl_topk(t, s, k, T=T, grad_scale=0.5)
    h = 1e-6
    for i in range(2):
        for v in range(30):
            sp, sm = s.copy(), s.copy()
            sp[i, v] += h
            sm[i, v] -= h
            fp = OT.kl_topk(t, sp, k, T=T, want_grad=False)[1][i]
            fm = OT.kl_topk(t, sm, k, T=T, want_grad=False)[1][i]
            assert abs(0.5 * (fp - fm) / (2 * h) - g[i, v]) < 1e-8
