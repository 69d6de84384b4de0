"""Expert parallelism of the MoE layer step on the device: two ranks (two
processes on one GPU, exchanging through gloo on the host; no kernel of one
rank waits for the other's) each own half of the routed experts and half of
the tokens.  ExpertParallelMoE dispatches the routed rows, runs the owned
experts' FFNs on the received rows with qad_moe_expert_forward / _backward,
returns and combines them, and runs the shared expert on each rank's own
tokens.  Against the oracle's single-process layer (oracle/moe.py): the
output y, dx, d(combine weights) and every routed expert's weight gradients
(on its owner) within the MoE step's bar; the shared expert's weight
gradient (bf16 partials summed over the ranks) within the bound of that
extra rounding; the routed experts' weight gradients bit for bit against
the single-GPU step, whose row order the exchange preserves.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

import oracle as O
from oracle import moe as OM
from moe_cases import f64, oracle_layer

pytestmark = pytest.mark.gpu
MOE_RTOL = 1e-3
E, T, H, F, K = 8, 256, 256, 256, 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case():
    from nvfp4_quantization_aware_b200 import synthetic as S
    return S.moe_layer(seed=3, tokens=T, hidden=H, ffn=F, experts=E, topk=K)


def _weights(Q, d, groups, dev):
    """qad_moe_weights tensors of the listed groups (frozen scales from the
    library's DYNAMIC quantization of the calibration weights)."""
    out = {}
    for k in ("gate", "up", "down"):
        w0 = d["w0_" + k][groups].to(dev)
        G, rows, cols = w0.shape
        _, sbs, ts = Q.nvfp4_quantize_grouped([w0[g] for g in range(G)], Q.DYNAMIC)
        sb = torch.cat(sbs).contiguous()
        out["w_" + k] = d["w_" + k][groups].to(dev).reshape(G * rows, cols).contiguous()
        out[k + "_ts"] = ts
        out[k + "_sb"] = sb
        out[k + "_sb_mma"] = Q.nvfp4_scales_to_mma(sb, G * rows, cols)
    out["x_ts"] = d["x_ts"][groups].to(dev).contiguous()
    out["a_ts"] = d["a_ts"][groups].to(dev).contiguous()
    return out


def _worker(rank, world, port, q):
    import torch.distributed as dist
    import nvfp4_quantization_aware_b200 as Q
    from nvfp4_quantization_aware_b200 import parallel as P

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        dev = torch.device("cuda", 0)
        d = _case()
        per = E // world
        local = _weights(Q, d, list(range(rank * per, (rank + 1) * per)), dev)
        shared = _weights(Q, d, [E], dev)
        t0, t1 = rank * T // world, (rank + 1) * T // world
        x = d["x"][t0:t1].to(dev)
        ids = d["ids"][t0:t1].to(dev)
        cw = d["combine"][t0:t1].to(dev)
        dy = d["dy"][t0:t1].to(dev)
        ep = P.ExpertParallelMoE(H, F, E, local, shared)
        y = ep.forward(x, ids, cw)
        dx, (dwg, dwu, dwd), (sg, su, sd), dcw = ep.backward(dy)
        # this rank's own (bf16) partial of the shared expert's weight gradient
        own = Q.MoeExpertStep(H, F, 1, shared)
        own.forward(x, torch.zeros(x.shape[0], dtype=torch.int32, device=dev))
        _, pg, pu, pd = own.backward(dy)
        torch.cuda.synchronize()
        err = Q.nvfp4_device_error()
        to = lambda t: t.float().cpu().numpy()
        q.put((rank, {"y": to(y), "dx": to(dx), "dcw": dcw.double().cpu().numpy(), "dwg": to(dwg), "dwu": to(dwu),
                      "dwd": to(dwd), "sg": to(sg), "su": to(su), "sd": to(sd), "pg": to(pg), "pu": to(pu),
                      "pd": to(pd), "err": err}))
    except Exception as e:  # report instead of hanging the parent
        q.put((rank, {"exception": repr(e)}))
        raise
    finally:
        dist.destroy_process_group()


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def test_expert_parallel_layer_step_matches_oracle():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 2
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=600) for _ in range(world))
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for r in range(world):
        assert "exception" not in res[r], res[r]
        assert res[r]["err"] == (0, 0)

    d = _case()
    L = oracle_layer(d)
    ref = OM.layer_step(L, f64(d["dy"]))
    y = np.concatenate([res[r]["y"] for r in range(world)]).astype(np.float64)
    dx = np.concatenate([res[r]["dx"] for r in range(world)]).astype(np.float64)
    dcw = np.concatenate([res[r]["dcw"] for r in range(world)])
    assert _rel(y, ref["y"]) <= MOE_RTOL
    assert _rel(dx, ref["dx"]) <= MOE_RTOL
    assert _rel(dcw, ref["d_combine"]) <= MOE_RTOL
    per = E // world
    for g in range(E):
        r, i = divmod(g, per)
        b = ref["groups"][g]["bwd"]
        got = {k: res[r][k][i * rows:(i + 1) * rows].astype(np.float64)
               for k, rows in (("dwg", F), ("dwu", F), ("dwd", H))}
        if b is None:
            assert not any(v.any() for v in got.values()), g
            continue
        assert _rel(got["dwg"], b["dW_gate"]) <= MOE_RTOL, g
        assert _rel(got["dwu"], b["dW_up"]) <= MOE_RTOL, g
        assert _rel(got["dwd"], b["dW_down"]) <= MOE_RTOL, g
    # The shared expert runs on each rank's own tokens; its weight gradient is
    # the sum over the ranks of bf16 partials P_r, rounded once more.  Against
    # the oracle (one rounding of the exact sum S) the error is at most
    # 2^-9 (sum_r |P_r| + 2 |S|) per element: the bar is that bound in the
    # Frobenius norm (plus the 1e-4 of FP32 accumulation).
    b = ref["groups"][E]["bwd"]
    for k, pk, name in (("sg", "pg", "dW_gate"), ("su", "pu", "dW_up"), ("sd", "pd", "dW_down")):
        for r in range(world):  # the all-reduced gradient is the same on every rank
            assert np.array_equal(res[r][k], res[0][k])
        S_ref = b[name]
        bound = 2.0 ** -9 * (sum(np.linalg.norm(res[r][pk].astype(np.float64)) for r in range(world))
                             / np.linalg.norm(S_ref) + 2.0) + 1e-4
        assert _rel(res[0][k].astype(np.float64), S_ref) <= bound, (name, bound)
        # and the ranks' partials themselves sum to it within one rounding
        psum = sum(res[r][pk].astype(np.float64) for r in range(world))
        assert _rel(res[0][k].astype(np.float64), psum) <= 2.0 ** -8

    # the routed experts' weight gradients equal the single-GPU step's bit for
    # bit: the exchange delivers each expert's rows in the single-process order
    import nvfp4_quantization_aware_b200 as Q
    dev = torch.device("cuda", 0)
    w = _weights(Q, d, list(range(E + 1)), dev)
    step = Q.MoeLayerStep(T, H, F, E, K, w)
    step.forward(d["x"].to(dev), d["ids"].to(dev), d["combine"].to(dev))
    _, dwg1, dwu1, dwd1, _ = step.backward(d["dy"].to(dev))
    torch.cuda.synchronize()
    for g in range(E):
        r, i = divmod(g, per)
        assert np.array_equal(dwg1[g * F:(g + 1) * F].float().cpu().numpy(), res[r]["dwg"][i * F:(i + 1) * F]), g
        assert np.array_equal(dwd1[g * H:(g + 1) * H].float().cpu().numpy(), res[r]["dwd"][i * H:(i + 1) * H]), g


def test_expert_step_single_rank_equals_layer_step_rows():
    """One rank owning every expert: the expert-parallel step is the layer
    step; y and dx equal the single-GPU MoeLayerStep's within one bf16
    rounding of the combine (summed in a different order)."""
    import nvfp4_quantization_aware_b200 as Q
    from nvfp4_quantization_aware_b200 import parallel as P

    dev = torch.device("cuda", 0)
    d = _case()
    ep = P.ExpertParallelMoE(H, F, E, _weights(Q, d, list(range(E)), dev), _weights(Q, d, [E], dev))
    x, ids, cw, dy = (d[n].to(dev) for n in ("x", "ids", "combine", "dy"))
    y = ep.forward(x, ids, cw)
    dx, _, _, dcw = ep.backward(dy)
    step = Q.MoeLayerStep(T, H, F, E, K, _weights(Q, d, list(range(E + 1)), dev))
    y1 = step.forward(x, ids, cw)
    dx1, _, _, _, dcw1 = step.backward(dy)
    torch.cuda.synchronize()
    assert _rel(y.double().cpu().numpy(), y1.double().cpu().numpy()) <= 2 ** -8
    assert _rel(dx.double().cpu().numpy(), dx1.double().cpu().numpy()) <= 2 ** -8
    assert _rel(dcw.double().cpu().numpy(), dcw1.double().cpu().numpy()) <= 1e-5
