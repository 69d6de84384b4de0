"""Expert-parallel dispatch / combine of the MoE layer
(nvfp4_quantization_aware_b200.parallel.ep_*) on two gloo ranks on the CPU.
Each expert is a plain linear map (the device work is not under test here);
every rank rebuilds both ranks' tokens from their seeds and checks its own
outputs, input gradients and combine-weight gradients, and the weight
gradients of the experts it owns, against the single-process layer."""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from nvfp4_quantization_aware_b200 import parallel as P

E, T, K, H, HO = 8, 10, 3, 16, 12


def _inputs(rank):
    g = torch.Generator().manual_seed(100 + rank)
    x = torch.randn(T, H, generator=g, dtype=torch.float64)
    ids = torch.stack([torch.randperm(E, generator=g)[:K] for _ in range(T)]).to(torch.int32)
    combine = torch.softmax(torch.randn(T, K, generator=g, dtype=torch.float64), -1)
    dy = torch.randn(T, HO, generator=g, dtype=torch.float64)
    return x, ids, combine, dy


def _weights():
    g = torch.Generator().manual_seed(7)
    return torch.randn(E, HO, H, generator=g, dtype=torch.float64)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        W = _weights()
        per = E // world
        x, ids, combine, dy = _inputs(rank)
        # forward
        recv_x, recv_e, plan = P.ep_dispatch(x, ids, E)
        y_recv = torch.stack([recv_x[i] @ W[rank * per + int(recv_e[i])].T for i in range(recv_x.shape[0])]) \
            if recv_x.shape[0] else recv_x.new_zeros(0, HO)
        y, y_slot = P.ep_combine(y_recv, plan, combine)
        y_ref = sum(combine[:, j:j + 1] * torch.stack([x[t] @ W[int(ids[t, j])].T for t in range(T)])
                    for j in range(K))
        ok = torch.allclose(y.double(), y_ref, rtol=1e-12, atol=1e-12)
        # received rows: grouped by source rank, (token, slot) order within a source
        ok &= sum(plan.recv_counts) == recv_x.shape[0] and int(recv_e.min()) >= 0 and int(recv_e.max()) < per
        # backward
        dy_recv, d_combine = P.ep_combine_backward(dy, plan, combine, y_slot)
        dx_recv = torch.stack([dy_recv[i] @ W[rank * per + int(recv_e[i])] for i in range(dy_recv.shape[0])]) \
            if dy_recv.shape[0] else dy_recv.new_zeros(0, H)
        dW_local = torch.zeros(per, HO, H, dtype=torch.float64)
        for i in range(dy_recv.shape[0]):
            dW_local[int(recv_e[i])] += torch.outer(dy_recv[i], recv_x[i])
        dx = P.ep_dispatch_backward(dx_recv, plan)
        dx_ref = sum(combine[:, j:j + 1] * torch.stack([dy[t] @ W[int(ids[t, j])] for t in range(T)])
                     for j in range(K))
        dcomb_ref = torch.stack([torch.stack([dy[t] @ (W[int(ids[t, j])] @ x[t]) for j in range(K)]) for t in range(T)])
        ok &= torch.allclose(dx.double(), dx_ref, rtol=1e-12, atol=1e-12)
        ok &= torch.allclose(d_combine.double(), dcomb_ref, rtol=1e-12, atol=1e-12)
        dW_ref = torch.zeros(E, HO, H, dtype=torch.float64)
        for r in range(world):
            xr, idr, cr, dyr = _inputs(r)
            for t in range(T):
                for j in range(K):
                    dW_ref[int(idr[t, j])] += cr[t, j] * torch.outer(dyr[t], xr[t])
        ok &= torch.allclose(dW_local, dW_ref[rank * per:(rank + 1) * per], rtol=1e-12, atol=1e-12)
        q.put((rank, bool(ok)))
    finally:
        dist.destroy_process_group()


def test_expert_parallel_layer_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res == {0: True, 1: True}


def test_single_rank_is_the_identity_exchange():
    W = _weights()
    x, ids, combine, dy = _inputs(0)
    recv_x, recv_e, plan = P.ep_dispatch(x, ids, E)
    assert recv_x.shape[0] == T * K
    y_recv = torch.stack([recv_x[i] @ W[int(recv_e[i])].T for i in range(T * K)])
    y, _ = P.ep_combine(y_recv, plan, combine)
    y_ref = sum(combine[:, j:j + 1] * torch.stack([x[t] @ W[int(ids[t, j])].T for t in range(T)]) for j in range(K))
    assert torch.allclose(y.double(), y_ref, rtol=1e-12, atol=1e-12)
    with pytest.raises(ValueError):
        P.ep_dispatch(x, ids + E, E)
