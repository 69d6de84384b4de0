"""Pins of the top-p KL oracle (oracle/topp.py): the set size against exact
integer arithmetic on logits whose probabilities are rational, against a
brute-force search over all subsets on tiny rows, the closed form for
uniform logits, the limits p -> 0 and p >= 1, and the loss against the
full-vocabulary and top-k losses it must reduce to."""
import itertools
import math

import numpy as np
import pytest

import oracle as O
from oracle import topk as OT
from oracle import topp as OP


@pytest.mark.parametrize("T", [1.0, 2.0, 0.5])
@pytest.mark.parametrize("seed", range(4))
def test_count_matches_integer_arithmetic_on_rational_probabilities(T, seed):
    # z = T ln w with integer weights w: p_t = w / sum(w) exactly, so the
    # shortest prefix reaching p = (c + 1/2) / W follows from integer sums
    rng = np.random.default_rng(seed)
    V = 40
    w = rng.integers(1, 12, V)
    z = T * np.log(w.astype(np.float64))
    W = int(w.sum())
    order = sorted(range(V), key=lambda i: (-w[i], i))
    cum = np.cumsum([int(w[i]) for i in order])
    for c in range(0, W, 7):
        p = (c + 0.5) / W
        expect = int(np.argmax(cum >= c + 1)) + 1
        assert OP.topp_count(z, p, T) == expect, (c, W)


def _valid_prefix(row, S):
    inside = set(S)
    return all(row[i] > row[j] or (row[i] == row[j] and i < j) for i in inside for j in range(len(row)) if j not in inside)


@pytest.mark.parametrize("seed", range(5))
def test_count_is_the_smallest_valid_top_set_reaching_p(seed):
    rng = np.random.default_rng(10 + seed)
    V = 7
    row = rng.integers(-3, 3, V).astype(np.float64) * 0.7  # ties
    e = [math.exp(v - row.max()) for v in row]
    tot = math.fsum(e)
    for p in (0.05, 0.3, 0.55, 0.8, 0.97):
        best = None
        for m in range(1, V + 1):
            for S in itertools.combinations(range(V), m):
                if _valid_prefix(row, S) and math.fsum(e[i] for i in S) / tot >= p:
                    best = m
                    break
            if best is not None:
                break
        assert OP.topp_count(row, p) == best, (row, p)


def test_uniform_logits_take_ceil_p_v_entries():
    row = np.zeros(1000)
    for p, m in ((0.3005, 301), (0.0004, 1), (0.9995, 1000), (0.5001, 501)):
        assert OP.topp_count(row, p) == m
    # "reaches" is >=: with four equal entries (sums exact in binary) p = 1/2 takes two
    four = np.zeros(4)
    assert OP.topp_count(four, 0.5) == 2
    assert OP.topp_count(four, 0.25) == 1
    assert OP.topp_count(four, 0.75) == 3


def test_limits():
    rng = np.random.default_rng(3)
    row = rng.normal(0, 3, 500)
    assert OP.topp_count(row, 1.0) == 500
    assert OP.topp_count(row, 2.0) == 500
    assert OP.topp_count(row, 1e-12) == 1
    # the single largest entry alone reaches p exactly when p <= its probability
    pmax = np.exp(row.max() - row.max()) / np.exp(row - row.max()).sum()
    assert OP.topp_count(row, pmax * 0.999) == 1
    assert OP.topp_count(row, pmax * 1.001) == 2


def test_loss_reduces_to_full_and_top_k():
    rng = np.random.default_rng(5)
    t = rng.normal(0, 3, (5, 64))
    s = t + rng.normal(0, 1, (5, 64))
    loss, rk, g, ks = OP.kl_topp(t, s, 1.0, T=1.5)
    ref_loss, ref_rk, ref_g = O.kl(t, s, T=1.5)
    assert np.all(ks == 64)
    assert np.allclose(rk, ref_rk, rtol=1e-12, atol=1e-14)
    assert np.allclose(g, ref_g, rtol=1e-12, atol=1e-16)
    loss, rk, g, ks = OP.kl_topp(t, s, 0.7)
    for i in range(5):
        _, rki, gi = OT.kl_topk(t[i:i + 1], s[i:i + 1], int(ks[i]), grad_scale=1.0 / 5)
        assert rk[i] == rki[0]
        assert np.array_equal(g[i], gi[0])
        cum = OP.topp_cumulative(t[i])
        assert cum[ks[i] - 1] >= 0.7 and (ks[i] == 1 or cum[ks[i] - 2] < 0.7)
