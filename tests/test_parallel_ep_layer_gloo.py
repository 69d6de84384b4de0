"""ExpertParallelMoE's orchestration on two gloo ranks on the CPU: dispatch,
the owned experts' step on the received rows, combine, the shared expert on
each rank's own tokens, and in the backward the two exchanges and the
all-reduce of the shared expert's weight gradient.  The device expert steps
(qad_moe_expert_forward / _backward, tested on the GPU) are replaced by
float64 linear experts with the same interface, so that the whole layer can
be checked against a single-process float64 reference to 1e-12."""
import datetime
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from nvfp4_quantization_aware_b200 import parallel as P

E, T, K, H = 8, 12, 3, 16


class LinearExperts:
    """forward(x, ids) -> y[r] = W[ids[r]] x[r]; backward(dy) -> (dx, dW, 0, 0)."""

    def __init__(self, W):
        self.W = W

    def forward(self, x, ids):
        self.x, self.ids = x, ids.to(torch.int64)
        if x.shape[0] == 0:
            return x.new_zeros(0, H)
        return torch.einsum("rij,rj->ri", self.W[self.ids], x)

    def backward(self, dy):
        dW = torch.zeros_like(self.W)
        if dy.shape[0] == 0:
            return dy.new_zeros(0, H), dW, torch.zeros_like(dW), torch.zeros_like(dW)
        dx = torch.einsum("rij,ri->rj", self.W[self.ids], dy)
        dW.index_add_(0, self.ids, torch.einsum("ri,rj->rij", dy, self.x))
        return dx, dW, torch.zeros_like(dW), torch.zeros_like(dW)


def _inputs(rank):
    g = torch.Generator().manual_seed(200 + rank)
    x = torch.randn(T, H, generator=g, dtype=torch.float64)
    ids = torch.stack([torch.randperm(E, generator=g)[:K] for _ in range(T)]).to(torch.int32)
    combine = torch.softmax(torch.randn(T, K, generator=g, dtype=torch.float64), -1)
    dy = torch.randn(T, H, generator=g, dtype=torch.float64)
    return x, ids, combine, dy


def _weights():
    g = torch.Generator().manual_seed(11)
    return torch.randn(E + 1, H, H, generator=g, dtype=torch.float64)  # expert E: the shared one


def _layer(W, x, ids, combine):
    """Single-process reference: y = sum_j c_j W_{e_j} x + W_shared x."""
    return sum(combine[:, j:j + 1] * torch.einsum("tij,tj->ti", W[ids[:, j].long()], x) for j in range(K)) + x @ W[E].T


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
        ep = object.__new__(P.ExpertParallelMoE)
        ep.group, ep.experts, ep.hidden, ep.ffn, ep._ctx = None, E, H, H, None
        ep.local = LinearExperts(W[rank * per:(rank + 1) * per])
        ep.shared = LinearExperts(W[E:E + 1])
        x, ids, combine, dy = _inputs(rank)
        y = ep.forward(x, ids, combine)
        ok = torch.allclose(y, _layer(W, x, ids, combine), rtol=1e-12, atol=1e-12)
        dx, (dW_local, _, _), (dW_shared, _, _), d_combine = ep.backward(dy)
        # reference gradients of the whole two-rank batch
        xs, idss, cs, dys = zip(*[_inputs(r) for r in range(world)])
        Xa, Ia, Ca, Da = torch.cat(xs), torch.cat(idss), torch.cat(cs), torch.cat(dys)
        Wr = W.clone().requires_grad_(True)
        Xr = Xa.clone().requires_grad_(True)
        Cr = Ca.clone().requires_grad_(True)
        (_layer(Wr, Xr, Ia, Cr) * Da).sum().backward()
        sl = slice(rank * T, (rank + 1) * T)
        ok &= torch.allclose(dx, Xr.grad[sl], rtol=1e-12, atol=1e-12)
        ok &= torch.allclose(d_combine, Cr.grad[sl], rtol=1e-12, atol=1e-12)
        ok &= torch.allclose(dW_local, Wr.grad[rank * per:(rank + 1) * per], rtol=1e-12, atol=1e-12)
        ok &= torch.allclose(dW_shared[0], Wr.grad[E], rtol=1e-12, atol=1e-12)  # all-reduced over both ranks
        q.put((rank, bool(ok)))
    finally:
        dist.destroy_process_group()


def test_expert_parallel_layer_orchestration_on_two_gloo_ranks():
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
