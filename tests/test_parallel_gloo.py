"""The row-sharded quantize and KL helpers (nvfp4_quantization_aware_b200.parallel)
on two gloo ranks on the CPU, with the device operations replaced by the
oracle: each rank's codes, block scales and tensor scales must equal the
whole-tensor DYNAMIC quantization restricted to its rows, and the sharded KL
loss and dLogits must equal the whole-batch loss and gradient."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
from nvfp4_quantization_aware_b200 import parallel as P
from nvfp4_quantization_aware_b200 import synthetic as S


def _oracle_ops():
    def tensor_amax(xs):
        return torch.tensor([O.tensor_amax(x.float().numpy()) if x.numel() else 0.0 for x in xs],
                            dtype=torch.float32)

    def scale_from_amax(amax):
        return torch.tensor([O.lib().oracle_global_scale_from_amax(float(a)) for a in amax], dtype=torch.float32)

    def quantize_frozen_global(xs, ts):
        out = [O.quantize(x.float().numpy(), O.FROZEN_GLOBAL, s_g=float(t)) for x, t in zip(xs, ts)]
        return [torch.from_numpy(c) for c, _, _ in out], [torch.from_numpy(sb) for _, sb, _ in out]

    def kl(t, s, T, grad_scale):
        _, row, g = O.kl(t.double().numpy(), s.double().numpy(), T=T, grad_scale=grad_scale)
        return torch.from_numpy(row), torch.from_numpy(g)

    return P.ShardOps(tensor_amax, scale_from_amax, quantize_frozen_global, kl)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=__import__("datetime").timedelta(seconds=60))
    try:
        ops = _oracle_ops()
        ws = [S.weights(96, 256, seed=30 + i, outlier_p=0.01, outlier_mult=40) for i in range(3)]
        # rows split unevenly: rank 0 gets the first 40 rows
        cut = 40
        shards = [w[:cut] if rank == 0 else w[cut:] for w in ws]
        codes, sbs, ts = P.sharded_dynamic_quantize(shards, ops)
        ok = True
        for i, w in enumerate(ws):
            rc, rsb, rsg = O.quantize(w.float().numpy(), O.DYNAMIC)
            sl = slice(0, cut) if rank == 0 else slice(cut, None)
            ok &= np.array_equal(codes[i].numpy(), rc[sl]) and np.array_equal(sbs[i].numpy(), rsb[sl])
            ok &= np.float32(ts[i]).view(np.uint32) == np.float32(rsg).view(np.uint32)
        t, s = S.logits_pair(12, 500, seed=7, dtype=torch.float32, boost=None)
        rows = slice(0, 5) if rank == 0 else slice(5, None)
        loss, row_kl, g = P.sharded_kl(t[rows], s[rows], total_rows=12, ops=ops)
        ref_loss, ref_row, ref_g = O.kl(t.double().numpy(), s.double().numpy())
        ok &= abs(float(loss[0]) - ref_loss) <= 1e-12 * abs(ref_loss)
        ok &= np.allclose(g.numpy(), ref_g[rows], rtol=1e-14, atol=1e-20)
        q.put((rank, bool(ok)))
    finally:
        dist.destroy_process_group()


def test_sharded_quantize_and_kl_on_two_gloo_ranks():
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
