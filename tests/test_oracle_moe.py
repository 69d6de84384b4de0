"""Pins of the MoE layer oracle (oracle/moe.py) against things other than
itself: routing invariants, closed forms of SiLU, finite differences of the
smooth layer for the straight-through backward, token-permutation
equivariance, locality of each expert, and the size of the quantization
error against the unquantized layer."""
import numpy as np
import pytest
import torch

from oracle import moe as OM
from nvfp4_quantization_aware_b200 import synthetic as S
from moe_cases import oracle_layer


def _small(seed=0, tokens=24, hidden=64, ffn=64, experts=4, topk=2):
    return S.moe_layer(seed=seed, tokens=tokens, hidden=hidden, ffn=ffn, experts=experts, topk=topk)


def test_silu_closed_forms():
    assert OM.silu(np.array([0.0]))[0] == 0.0
    assert OM.silu_grad(np.array([0.0]))[0] == 0.5
    g = np.array([-40.0, -3.0, -0.5, 0.7, 2.0, 40.0])
    np.testing.assert_allclose(OM.silu(g), g * (1.0 / (1.0 + np.exp(-g))), rtol=1e-15)
    assert abs(OM.silu(np.array([40.0]))[0] - 40.0) < 1e-12       # silu(g) -> g for large g
    assert abs(OM.silu(np.array([-40.0]))[0]) < 1e-15             # -> 0 for very negative g
    h = 1e-6
    fd = (OM.silu(g + h) - OM.silu(g - h)) / (2 * h)
    np.testing.assert_allclose(OM.silu_grad(g), fd, rtol=1e-7, atol=1e-9)


def test_route_lists_every_assignment_once_in_token_order():
    d = _small(tokens=50, experts=6, topk=3)
    ids = d["ids"].numpy()
    segs = OM.route(ids, 6)
    seen = set()
    for e, (t, j) in enumerate(segs[:-1]):
        assert np.all(np.diff(t) > 0)                 # increasing tokens, one slot per token
        for tt, jj in zip(t, j):
            assert ids[tt, jj] == e
            seen.add((int(tt), int(jj)))
    assert seen == {(t, j) for t in range(50) for j in range(3)}
    t, j = segs[-1]
    assert j is None and np.array_equal(t, np.arange(50))


def _smooth_layer(seed=3, T=5, H=8, F=4, E=3, k=2):
    rng = np.random.default_rng(seed)
    G = E + 1
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)])
    z = np.zeros(G)
    return OM.Layer(x=rng.normal(size=(T, H)), ids=ids, cw=rng.uniform(0.1, 1.0, (T, k)),
                    w_gate=rng.normal(0, 0.5, (G, F, H)), w_up=rng.normal(0, 0.5, (G, F, H)),
                    w_down=rng.normal(0, 0.5, (G, H, F)), gate_ts=z, up_ts=z, down_ts=z,
                    gate_sb=None, up_sb=None, down_sb=None, x_ts=z, a_ts=z), rng.normal(size=(T, H))


def _loss(L, dy):
    return float(np.sum(OM.layer_step(L, None, quantized=False, rounded=False)["y"] * dy))


def test_straight_through_backward_is_the_gradient_of_the_smooth_layer():
    # With Q = identity and no rounding the backward must be the exact
    # gradient of sum(dy * y): central differences on every input entry.
    L, dy = _smooth_layer()
    out = OM.layer_step(L, dy, quantized=False, rounded=False)
    h = 1e-6

    def fd(arr, idx):
        old = arr[idx]
        arr[idx] = old + h
        fp = _loss(L, dy)
        arr[idx] = old - h
        fm = _loss(L, dy)
        arr[idx] = old
        return (fp - fm) / (2 * h)

    for idx in np.ndindex(L.x.shape):
        assert abs(fd(L.x, idx) - out["dx"][idx]) < 1e-7 * max(1.0, abs(out["dx"][idx]))
    for idx in np.ndindex(L.cw.shape):
        assert abs(fd(L.cw, idx) - out["d_combine"][idx]) < 1e-7 * max(1.0, abs(out["d_combine"][idx]))
    for name, key in (("w_gate", "dW_gate"), ("w_up", "dW_up"), ("w_down", "dW_down")):
        arr = getattr(L, name)
        for g in range(arr.shape[0]):
            bwd = out["groups"][g]["bwd"]
            for idx in np.ndindex(arr.shape[1:]):
                want = fd(arr, (g,) + idx)
                got = 0.0 if bwd is None else bwd[key][idx]
                assert abs(want - got) < 1e-7 * max(1.0, abs(want)), (name, g, idx)


def test_token_permutation_permutes_outputs_bit_for_bit():
    d = _small(seed=1)
    L = oracle_layer(d)
    out = OM.layer_step(L, OM.to_bf16(L.x * 0.5))
    perm = np.random.default_rng(0).permutation(L.x.shape[0])
    Lp = oracle_layer(d)
    Lp.x, Lp.ids, Lp.cw = L.x[perm], L.ids[perm], L.cw[perm]
    outp = OM.layer_step(Lp, OM.to_bf16(L.x[perm] * 0.5))
    assert np.array_equal(outp["y"], out["y"][perm])
    assert np.array_equal(outp["dx"], out["dx"][perm])
    assert np.array_equal(outp["d_combine"], out["d_combine"][perm])
    for g in range(L.experts + 1):
        for key in ("dW_gate", "dW_up", "dW_down"):
            assert np.array_equal(outp["groups"][g]["bwd"][key], out["groups"][g]["bwd"][key])


def test_an_expert_only_affects_its_tokens():
    d = _small(seed=2)
    L = oracle_layer(d)
    y0 = OM.layer_step(L, None)["y"]
    e = 1
    L.w_down = L.w_down.copy()
    L.w_down[e] *= 0.5          # against the frozen scales: other codes
    L.forget_quantized_weights()
    y1 = OM.layer_step(L, None)["y"]
    mine = np.any(L.ids == e, axis=1)
    assert np.array_equal(y0[~mine], y1[~mine])
    assert not np.array_equal(y0[mine], y1[mine])


def test_quantized_layer_stays_near_the_unquantized_layer():
    # Three NVFP4 quantizations on the path: the output moves by a fraction
    # of its size (NVFP4's relative round-trip error on Gaussian data is
    # about 0.1), not by O(1) as a wrong index or transpose would give.
    d = _small(seed=4, tokens=64, hidden=128, ffn=128)
    L = oracle_layer(d)
    yq = OM.layer_step(L, None)["y"]
    ys = OM.layer_step(L, None, quantized=False, rounded=False)["y"]
    rel = np.linalg.norm(yq - ys) / np.linalg.norm(ys)
    assert 0.02 < rel < 0.3, rel


def test_shared_expert_alone_when_routed_weights_vanish():
    d = _small(seed=5)
    L = oracle_layer(d)
    L.cw = np.zeros_like(L.cw)
    out = OM.layer_step(L, None)
    st = OM.expert_forward(L, L.experts, L.x)
    assert np.array_equal(out["y"], st["y"])


def test_combine_rows_reproduces_the_layer_output():
    """combine_rows over the per-expert output rows (laid out as a row
    buffer, shared expert last) gives the layer_step output bit for bit, and
    gather_sum_rows of the per-expert dX rows gives the layer's dx."""
    d = _small(tokens=30, experts=5, topk=3)
    L = oracle_layer(d)
    dy = d["dy"].double().numpy()
    ref = OM.layer_step(L, dy)
    T, H = L.x.shape
    E = L.experts
    rows_y, rows_dx, base = [], [], 0
    slot_row = -np.ones(L.ids.shape, dtype=np.int64)
    for g, (t, j) in enumerate(ref["segments"]):
        per = ref["groups"][g]
        if len(t) == 0:
            continue
        if g < E:
            slot_row[t, j] = base + np.arange(len(t))
        else:
            shared_base = base
        rows_y.append(per["fwd"]["y"])
        rows_dx.append(per["bwd"]["dX"])
        base += len(t)
    y = np.concatenate(rows_y)
    dxp = np.concatenate(rows_dx)
    assert np.array_equal(OM.combine_rows(y, slot_row, L.cw, shared_base), ref["y"])
    assert np.array_equal(OM.gather_sum_rows(dxp, slot_row, shared_base), ref["dx"])


def test_combine_rows_hand_case():
    y = np.array([[1.0, 2.0], [3.0, -1.0], [0.5, 0.5], [10.0, 20.0], [-4.0, 8.0]])
    slot_row = np.array([[0, 2], [-1, 1]])
    w = np.array([[0.25, 2.0], [7.0, 0.5]])
    out = OM.combine_rows(y, slot_row, w, shared_base=3)
    # token 0: 0.25*[1,2] + 2*[0.5,0.5] + [10,20]; token 1: 0.5*[3,-1] + [-4,8]
    assert np.array_equal(out, [[11.25, 21.5], [-2.5, 7.5]])
    assert np.array_equal(OM.gather_sum_rows(y, slot_row, 3), [[11.5, 22.5], [-1.0, 7.0]])
