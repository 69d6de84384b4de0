#!/usr/bin/env python3
"""Benchmark of the NVFP4 QAD hot path on B200.

Headline workload (one JSON line on rank 0): the weight quantization sweep --
128 MoE expert weights 2048 x 1024 plus one 131072 x 2048 lm_head, bf16,
536,870,912 elements -- quantized to packed E2M1 codes + E4M3 block scales +
FP32 tensor scales, first with dynamic scales (amax recomputed) and then with
frozen scales (the dynamic pass's scales passed back in).  One step is both
passes over all 129 tensors.  value = algorithmic bytes / device time, with
2.5625 B per element and pass (2 B bf16 in, 0.5 B codes + 0.0625 B scales out;
the frozen pass reads the 0.0625 B scales instead of writing them).

Also measured in the same run and reported under "gemm" and "kl":
  * W4A4 GEMM: activations M x 4096 (M = 8192 and 128) quantized on the fly,
    weights 4096 x 4096 pre-quantized, bf16 out -- TFLOP/s;
  * KL distillation loss + dLogits over 16384 x 131072 bf16 teacher/student
    logits -- tokens/s and GB/s (6 B per logit);
  * the top-k KL loss (key "kl_topk"): the same logits, k = 4096 per row;
  * the top-p KL loss (key "kl_topp"): the same logits, p = 0.95;
  * weight-only NVFP4 (key "w4a16"): the same GEMM shapes with bf16
    activations, the weights dequantized in the main loop, beside W4A4 and
    the BF16 GEMM of the dequantized weights;
  * the tiny QAD linear (key "tiny"): microseconds per call of its dynamic
    fake-quant, quantize, GEMM and KL steps;
  * the dense FP4 MMA peak measured by the library's own probe (key
    "fp4_peak_probe", run last), which the GEMM's roofline takes as its peak;
  * the MSE block-scale calibration of the 128 expert weights ("calibrate_mse");
  * the MoE layer step (config "moe_step"): 4096 tokens, 128 routed experts
    + 1 shared, top-6, forward (grouped W4A4) + straight-through backward
    (BF16) -- tokens/s and per-phase times.

Timing: device time with CUDA events on the launching stream; the K timed
steps are one CUDA-graph replay of K consecutive steps, bracketed by a
barrier and synchronize; the maximum over ranks is reported.  Inputs are
larger than L2 (1.07 GB), so no flush is needed between steps; the GEMM
(25 MB of operands) cycles through copies of its weights (and, at M = 8192,
of its activations) totalling more than twice the L2, so every launch reads
its operands from HBM.

"e2e" repeats the headline step through the public API from pinned host
memory (HostGroupedQuantizer: host-to-device copies, both passes, and the
codes and scales copied back, overlapped chunk by chunk).

--impl reference times the CPU oracle (oracle/, test infrastructure) on the
host cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 quant GB/s & W4A4 GEMM TFLOPS (% of peak); QAD KL loss tokens/s"
BYTES_PER_ELEM = 2.5625
WORKLOAD = ("weight quantization sweep: 128 MoE experts 2048x1024 + lm_head 131072x2048 bf16, "
            "NVFP4 dynamic then frozen (FROZEN_ALL) quantize to packed codes + E4M3 block scales")
# DRAM bytes of one launch of the dominant kernel, from an ncu capture of the
# same kernel on 48 expert weights (100.7M elements: read 207.67 MB + write
# 34.78 MB = 2.408 B per element), scaled by elements to the whole sweep
# (536,870,912 elements); reported only while quantize.cu is the source that
# was captured (its SHA-256 below).
TRAFFIC = {"kernel": "group_encode_kernel<bf16,codes> (FROZEN_ALL, whole sweep)",
           "bytes": round((207.665152e6 + 34.7776e6) / (48 * 2048 * 1024) * 536870912),
           "source_sha256": "2c8e221a89a4d138b318ceb5cf4828d24f53c4f104793c0682673dcd9d83d014"}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def file_sha(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi SM clock / throttle-reason sampling during the measured region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), parts[4:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        load = [r for r in rows if r[0] > 600] or rows
        names = ["active", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in load for i in range(1, 5) if r[2][i].lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in load), "sm_max_mhz": max(r[1] for r in rows),
                "samples": len(load), "reasons": reasons}


# --------------------------------------------------------------------------- distributed

def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# --------------------------------------------------------------------------- our arm

def make_sweep(rank, device):
    from nvfp4_quantization_aware_b200 import synthetic as S
    return S.weight_sweep(seed=1000 * rank, device=device)


def run_ours(args, world, rank, local):
    import nvfp4_quantization_aware_b200 as Q
    dev = torch.device("cuda", local)
    P = peaks()
    sampler = ClockSampler(local)
    xs = make_sweep(rank, dev)
    n_elem = sum(x.numel() for x in xs)
    n = len(xs)
    ts = torch.zeros(n, dtype=torch.float32, device=dev)
    sbs = [torch.empty(x.shape[0], x.shape[1] // 16, dtype=torch.uint8, device=dev) for x in xs]
    codes_dyn = [torch.empty(x.shape[0], x.shape[1] // 2, dtype=torch.uint8, device=dev) for x in xs]
    codes_fro = [torch.empty(x.shape[0], x.shape[1] // 2, dtype=torch.uint8, device=dev) for x in xs]
    ws = torch.empty(int(Q.lib().nvfp4_grouped_workspace_size(Q.DYNAMIC)), dtype=torch.uint8, device=dev)

    def step():
        Q.nvfp4_quantize_grouped(xs, Q.DYNAMIC, tensor_scales=ts, block_scales=sbs, codes=codes_dyn, workspace=ws)
        Q.nvfp4_quantize_grouped(xs, Q.FROZEN_ALL, tensor_scales=ts, block_scales=sbs, codes=codes_fro)

    stream = torch.cuda.Stream(dev)
    K, W = args.steps, args.warmup
    sampler.start()
    with torch.cuda.stream(stream):
        for _ in range(W):
            step()
        stream.synchronize()
        # capture K consecutive steps, with external timing events between passes
        evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)] for _ in range(K)]
        g = torch.cuda.CUDAGraph()
        n0 = Q.nvfp4_launch_count()
        with torch.cuda.graph(g, stream=stream):
            for k in range(K):
                evs[k][0].record(stream)
                Q.nvfp4_quantize_grouped(xs, Q.DYNAMIC, tensor_scales=ts, block_scales=sbs, codes=codes_dyn,
                                         workspace=ws)
                evs[k][1].record(stream)
                Q.nvfp4_quantize_grouped(xs, Q.FROZEN_ALL, tensor_scales=ts, block_scales=sbs, codes=codes_fro)
                evs[k][2].record(stream)
        launches = Q.nvfp4_launch_count() - n0
        g.replay()  # untimed replay: warms the graph itself
        stream.synchronize()
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize(dev)
        start.record(stream)
        g.replay()
        end.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
    total_ms = start.elapsed_time(end)
    dyn_ms = [evs[k][0].elapsed_time(evs[k][1]) for k in range(K)]
    fro_ms = [evs[k][1].elapsed_time(evs[k][2]) for k in range(K)]
    del g
    t_max = max_over_ranks(total_ms, world)
    ms_per_step = t_max / K
    units = sum_over_ranks(float(n_elem), world)
    value = units * 2 * BYTES_PER_ELEM / (ms_per_step * 1e-3) / 1e9

    # dominant kernel: the frozen pass is one launch of the encode kernel over
    # the whole sweep (129 tensors <= one group)
    fro_avg = statistics.mean(fro_ms)
    dyn_avg = statistics.mean(dyn_ms)
    achieved = n_elem * BYTES_PER_ELEM / (fro_avg * 1e-3) / 1e9
    qsrc = os.path.join(ROOT, "nvfp4_quantization_aware_b200", "csrc", "quantize.cu")
    traffic = TRAFFIC["bytes"] if TRAFFIC["source_sha256"] == file_sha(qsrc) else None
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": P["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / P["hbm_gbs"], 4), "traffic": traffic,
                "kernel": TRAFFIC["kernel"], "peak_source": P["source"] + " (MEASURED_PEAKS hbm_gbs)",
                "algorithmic_bytes_per_launch": n_elem * BYTES_PER_ELEM, "avg_launch_ms": round(fro_avg, 5)}
    phases = {"dynamic_ms": round(dyn_avg, 4), "frozen_ms": round(fro_avg, 4),
              "dynamic_gbs": round(n_elem * BYTES_PER_ELEM / (dyn_avg * 1e-3) / 1e9, 1),
              "frozen_gbs": round(achieved, 1)}

    # ---- end to end through the public API, host buffers, copies inside
    e2e = run_e2e(Q, xs, dev, stream, min(K, 5), world)

    secondary = {}
    if not args.no_secondary:
        secondary["tiny"] = bench_tiny(Q, dev, stream)
        secondary["gemm"] = bench_gemm(Q, dev, stream, P, max(3, min(K, 20)))
        secondary["w4a16"] = bench_w4a16(Q, dev, stream, P, max(3, min(K, 20)))
        secondary["kl"] = bench_kl(Q, dev, stream, P, max(3, min(K, 10)))
        secondary["kl_topk"] = bench_kl_topk(Q, dev, stream, P, max(3, min(K, 10)))
        secondary["kl_topp"] = bench_kl_topp(Q, dev, stream, P, max(3, min(K, 5)))
        secondary["calibrate_mse"] = bench_calibrate(Q, dev, stream, xs, 3)
        secondary["moe_step"] = bench_moe(Q, dev, stream, P, max(3, min(K, 10)))
        # the FP4 probe runs last: its sustained launch (~70 ms at full tensor
        # power) would lower the clocks of whatever is timed right after it
        secondary["fp4_peak_probe"] = bench_fp4_peak(Q, dev, stream)
        apply_fp4_peak(secondary["gemm"], secondary["fp4_peak_probe"])
        peak = (secondary["fp4_peak_probe"] or {}).get("burst_tflops")
        gf = secondary["moe_step"]["phases"]["w4a4_gemms_forward"]
        if peak:
            gf["peak"] = peak
            gf["frac"] = round(gf["tflops"] / peak, 4)
            gf["peak_source"] = "own tcgen05 FP4 MMA probe, burst (fp4_peak_probe)"
    clocks = sampler.stop()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(xs)

    line = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": K, "warmup": W,
            "ms_per_step": round(ms_per_step, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOAD, "elements_per_gpu": n_elem, "tensors": n,
                       "bytes_per_element_per_pass": BYTES_PER_ELEM,
                       "l2": "inputs larger than L2 (1.07 GB of bf16 per GPU), no flush",
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "timing": "CUDA events around one graph replay of K steps"},
            "phases": phases, "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": int(launches), "clocks": clocks}
    line.update(secondary)
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_e2e(Q, xs, dev, stream, K, world):
    """Same metric through the public API with pinned host buffers: per step
    the inputs are copied host -> device, both passes run, and the frozen
    codes + block scales + tensor scales are copied back.  The library's
    HostGroupedQuantizer overlaps the copies of one chunk of tensors with the
    kernels of the next (three streams)."""
    hx = [x.cpu().pin_memory() for x in xs]
    hq = Q.HostGroupedQuantizer(hx, dev, passes=(Q.DYNAMIC, Q.FROZEN_ALL))
    with torch.cuda.stream(stream):
        hq.run(stream)
        stream.synchronize()
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize(dev)
        start.record(stream)
        for _ in range(K):
            hq.run(stream)
        end.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
    ms = max_over_ranks(start.elapsed_time(end), world) / K
    n_elem = sum(x.numel() for x in xs)
    units = sum_over_ranks(float(n_elem), world)
    return {"value": round(units * 2 * BYTES_PER_ELEM / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": hq.h2d_bytes, "d2h_bytes_per_step": hq.d2h_bytes, "ms_per_step": round(ms, 3),
            "steps": K, "chunks": len(hq.chunks)}


def flush_l2(buf):
    buf.zero_()


def bench_tiny(Q, dev, stream, reps=50):
    """The tiny QAD linear (latency-bound): microseconds per call of each step,
    each timed as one CUDA-graph replay of `reps` back-to-back calls (no L2
    flush: the whole working set is a few MB)."""
    from nvfp4_quantization_aware_b200 import synthetic as S
    d = S.tiny_qad_linear(seed=0, device=dev)
    x, w, t, s_ = d["x"], d["w"], d["teacher"], d["student"]
    M, K = x.shape
    N = w.shape[0]
    L = Q.lib()
    ws = torch.empty(int(L.nvfp4_quantize_workspace_size(M, K, Q.DYNAMIC)), dtype=torch.uint8, device=dev)
    xf, wf = torch.empty_like(x), torch.empty_like(w)
    xc = torch.empty(M, K // 2, dtype=torch.uint8, device=dev)
    xsf = torch.empty(Q.mma_scales_bytes(M, K), dtype=torch.uint8, device=dev)
    xts = torch.empty(1, dtype=torch.float32, device=dev)
    wc, wsf, wts = Q.nvfp4_quantize(w, Q.DYNAMIC, layout=Q.SCALES_MMA)
    c = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    grad = torch.empty_like(s_)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    kws = torch.empty(int(L.qad_kl_workspace_size(t.shape[0], t.shape[1], Q.F32)), dtype=torch.uint8, device=dev)
    calls = {
        "fake_quant_x_dynamic": lambda: Q.nvfp4_fake_quant(x, Q.DYNAMIC, tensor_scale=xts, out=xf, workspace=ws),
        "fake_quant_w_dynamic": lambda: Q.nvfp4_fake_quant(w, Q.DYNAMIC, tensor_scale=xts, out=wf, workspace=ws),
        "quantize_x_dynamic_mma": lambda: Q.nvfp4_quantize(x, Q.DYNAMIC, tensor_scale=xts, block_scales=xsf,
                                                           layout=Q.SCALES_MMA, codes=xc, workspace=ws),
        "gemm_w4a4_64x1024x1024": lambda: Q.nvfp4_gemm_w4a4(xc, xsf, xts, wc, wsf, wts, out=c),
        "kl_fwd_bwd_64x8192_f32": lambda: L.qad_kl_fwd_bwd(t.data_ptr(), s_.data_ptr(), Q.F32, t.shape[0], t.shape[1],
                                                           t.shape[1], 1.0, loss.data_ptr(), None, grad.data_ptr(),
                                                           t.shape[1], 1.0 / t.shape[0], kws.data_ptr(), kws.numel(),
                                                           stream.cuda_stream),
    }
    out = {}
    with torch.cuda.stream(stream):
        for name, call in calls.items():
            call()
            stream.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for _ in range(reps):
                    call()
            g.replay()
            stream.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            g.replay()
            e1.record(stream)
            stream.synchronize()
            out[name + "_us"] = round(e0.elapsed_time(e1) * 1e3 / reps, 2)
            del g
    out["config"] = ("tiny QAD linear: X 64x1024 bf16, W 1024x1024 bf16 (0.5% outliers x30), KL over 64x8192 fp32; "
                     "microseconds per call, back-to-back calls in one CUDA graph")
    return out


def bench_fp4_peak(Q, dev, stream):
    """Dense FP4 MMA throughput measured by the library's own probe (one CTA per
    SM issuing block-scaled FP4 tcgen05 MMAs back to back on resident tiles):
    a burst figure (median of 5 launches of ~1 ms) and a sustained one (one
    launch of ~50 ms, under the power cap)."""
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    res = {}
    with torch.cuda.stream(stream):
        for name, iters, reps in (("burst", 4000, 5), ("sustained", 200000, 1)):
            Q.nvfp4_probe_fp4_mma(iters, sms, stream)  # warm-up
            times, flop = [], 0.0
            for _ in range(reps):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                flop = Q.nvfp4_probe_fp4_mma(iters, sms, stream)
                e1.record(stream)
                stream.synchronize()
                times.append(e0.elapsed_time(e1))
            ms = statistics.median(times)
            res[f"{name}_tflops"] = round(flop / (ms * 1e-3) / 1e12, 1)
            res[f"{name}_ms"] = round(ms, 4)
    st, word = Q.nvfp4_device_error()
    res["device_error"] = [int(st), int(word)]
    res["datasheet_tflops"] = 9000.0
    res["method"] = ("tcgen05.mma.kind::mxf4nvf4.block_scale 128x256x64, UE4M3 scales, operands resident in "
                     "shared memory, one CTA per SM, CUDA events")
    return res


def apply_fp4_peak(gemm, probe):
    """Re-express the tensor-bound GEMM rooflines against the probe's burst peak."""
    peak = probe.get("burst_tflops") if probe else None
    if not peak:
        return
    for key, res in gemm.items():
        r = res.get("roofline") if isinstance(res, dict) else None
        if r and r.get("bound") == "tensor":
            r["peak"] = peak
            r["frac"] = round(r["achieved"] / peak, 4)
            r["peak_source"] = "own tcgen05 FP4 MMA probe, burst (fp4_peak_probe)"


def bench_gemm(Q, dev, stream, P, K, probe=None):
    """W4A4 GEMM on the config-3 shapes, X quantized on the fly.  Inputs are
    larger than L2 instead of flushing it: the timed steps cycle through
    copies of the weights (and, at M = 8192, of the activations) whose total
    exceeds twice the L2, so every step reads its operands from HBM.  K steps
    are one CUDA graph with events between the X quantize and the GEMM."""
    from nvfp4_quantization_aware_b200 import synthetic as S
    out = {}
    # peak: the library's own FP4 MMA probe (burst: the GEMM is timed in ~100 us
    # launches); without it, 4 x the measured dense BF16 peak (nominal FP4:BF16 9 : 2.25)
    if probe and probe.get("burst_tflops"):
        fp4_peak, fp4_src = probe["burst_tflops"], "own tcgen05 FP4 MMA probe, burst (fp4_peak_probe)"
    else:
        fp4_peak, fp4_src = 4.0 * P["bf16_tflops"], "4 x MEASURED_PEAKS bf16_tflops (nominal FP4:BF16 ratio)"
    l2 = 126 << 20
    with torch.cuda.stream(stream):
        w = S.weights(4096, 4096, seed=1, device=dev)
        wc, wsf, wts = Q.nvfp4_quantize(w, Q.DYNAMIC, layout=Q.SCALES_MMA)
        w_bytes = wc.numel() + wsf.numel()
        nw = max(2, -(-2 * l2 // w_bytes))  # weight copies: > 2 x L2 in all
        ws = [(wc.clone(), wsf.clone(), wts.clone()) for _ in range(nw)]
        del w
        for M in (8192, 128):
            x0 = S.channel_scaled_activations(M, 4096, seed=0, device=dev)
            x_bytes = x0.numel() * 2
            nx = max(1, min(nw, -(-2 * l2 // x_bytes))) if M >= 1024 else 1
            xs = [x0.clone() for _ in range(nx)]
            del x0
            xc = torch.empty(M, 2048, dtype=torch.uint8, device=dev)
            xsf = torch.empty(Q.mma_scales_bytes(M, 4096), dtype=torch.uint8, device=dev)
            xts = torch.empty(1, dtype=torch.float32, device=dev)
            c = torch.empty(M, 4096, dtype=torch.bfloat16, device=dev)
            qws = torch.empty(int(Q.lib().nvfp4_quantize_workspace_size(M, 4096, Q.DYNAMIC)), dtype=torch.uint8,
                              device=dev)

            def step(k):
                Q.nvfp4_quantize(xs[k % nx], Q.DYNAMIC, tensor_scale=xts, block_scales=xsf, layout=Q.SCALES_MMA,
                                 codes=xc, workspace=qws)

            for k in range(3):
                step(k)
                Q.nvfp4_gemm_w4a4(xc, xsf, xts, *ws[k % nw], out=c)
            stream.synchronize()
            steps = max(K, nw)
            evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)] for _ in range(steps)]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for k in range(steps):
                    evs[k][0].record(stream)
                    step(k)
                    evs[k][1].record(stream)
                    Q.nvfp4_gemm_w4a4(xc, xsf, xts, *ws[k % nw], out=c)
                    evs[k][2].record(stream)
            g.replay()
            stream.synchronize()
            q_ms = statistics.mean(evs[k][0].elapsed_time(evs[k][1]) for k in range(steps))
            g_ms = statistics.mean(evs[k][1].elapsed_time(evs[k][2]) for k in range(steps))
            del g
            # the same quantize + GEMM pairs with no timing events between them
            # (an event between two launches also keeps the second from starting
            # early): one event pair around all steps
            e0 = torch.cuda.Event(enable_timing=True, external=True)
            e1 = torch.cuda.Event(enable_timing=True, external=True)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                e0.record(stream)
                for k in range(steps):
                    step(k)
                    Q.nvfp4_gemm_w4a4(xc, xsf, xts, *ws[k % nw], out=c)
                e1.record(stream)
            g.replay()
            stream.synchronize()
            pair_ms = e0.elapsed_time(e1) / steps
            del g, xs
            flops = 2.0 * M * 4096 * 4096
            tflops = flops / (g_ms * 1e-3) / 1e12
            gemm_bytes = 4096 * 4096 * 0.5625 + M * 4096 * 0.5625 + M * 4096 * 2
            out[f"M{M}"] = {"tflops": round(tflops, 1), "gemm_ms": round(g_ms, 5), "x_quant_ms": round(q_ms, 5),
                            "end_to_end_tflops": round(flops / ((q_ms + g_ms) * 1e-3) / 1e12, 1),
                            "x_quant_plus_gemm_ms": round(pair_ms, 5),
                            "gemm_gbs": round(gemm_bytes / (g_ms * 1e-3) / 1e9, 1),
                            "weight_copies": nw, "activation_copies": nx, "steps": steps,
                            "roofline": {"bound": "tensor" if M >= 1024 else "hbm",
                                         "achieved": round(tflops, 1) if M >= 1024 else round(gemm_bytes / (g_ms * 1e-3) / 1e9, 1),
                                         "peak": round(fp4_peak, 1) if M >= 1024 else P["hbm_gbs"],
                                         "unit": "TFLOP/s" if M >= 1024 else "GB/s",
                                         "frac": round(tflops / fp4_peak, 4) if M >= 1024 else
                                         round(gemm_bytes / (g_ms * 1e-3) / 1e9 / P["hbm_gbs"], 4),
                                         "peak_source": fp4_src if M >= 1024 else "MEASURED_PEAKS hbm_gbs",
                                         "frac_of_datasheet_9pf": round(tflops / 9000.0, 4),
                                         "frac_of_4x_bf16": round(tflops / (4.0 * P["bf16_tflops"]), 4)}}
        del ws
    torch.cuda.empty_cache()
    out["config"] = ("x M x 4096 bf16 N(0,1)*LogNormal(0,1) per channel, dynamic NVFP4 on the fly; w 4096x4096 "
                     "pre-quantized; inputs larger than L2: steps cycle through weight (and M = 8192 activation) "
                     "copies totalling > 2 x L2, no flush")
    return out


def bench_w4a16(Q, dev, stream, P, K):
    """Weight-only NVFP4 (W4A16) against W4A4 and BF16 on the same 4096 x 4096
    weights: W4A16 dequantizes the weights in its main loop and runs the BF16
    tensor cores; the BF16 product of the already dequantized weights is timed
    beside it (this package's grouped BF16 GEMM and, as a library reference,
    torch.matmul / cuBLAS)."""
    from nvfp4_quantization_aware_b200 import synthetic as S
    out = {}
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    with torch.cuda.stream(stream):
        w = S.weights(4096, 4096, seed=1, device=dev)
        rc, rsf, rts = Q.nvfp4_quantize(w, Q.DYNAMIC)
        wc, wsf, wts = Q.nvfp4_quantize(w, Q.DYNAMIC, layout=Q.SCALES_MMA)
        w_hat = Q.nvfp4_fake_quant(w, Q.DYNAMIC)
        for M in (8192, 128):
            x = S.channel_scaled_activations(M, 4096, seed=0, device=dev)
            xc, xsf, xts = Q.nvfp4_quantize(x, Q.DYNAMIC, layout=Q.SCALES_MMA)
            c = torch.empty(M, 4096, dtype=torch.bfloat16, device=dev)
            off = torch.tensor([0, M], dtype=torch.int32, device=dev)
            ln = torch.tensor([M], dtype=torch.int32, device=dev)
            calls = {"w4a16": lambda: Q.nvfp4_gemm_w4a16(x, rc, rsf, rts, out=c),
                     "w4a4": lambda: Q.nvfp4_gemm_w4a4(xc, xsf, xts, wc, wsf, wts, out=c),
                     "bf16": lambda: Q.nvfp4_gemm_bf16_grouped(0, x, w_hat, off, ln, M, 4096, 4096, out=c),
                     "cublas_bf16": lambda: torch.matmul(x, w_hat.t(), out=c)}
            res = {}
            for name, call in calls.items():
                for _ in range(3):
                    call()
                evs = []
                for _ in range(K):
                    flush_l2(flush)
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    call()
                    e1.record(stream)
                    evs.append((e0, e1))
                stream.synchronize()
                ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
                res[name] = {"ms": round(ms, 5), "tflops": round(2.0 * M * 4096 * 4096 / (ms * 1e-3) / 1e12, 1)}
            res["w4a16_over_bf16_throughput"] = round(res["bf16"]["ms"] / res["w4a16"]["ms"], 3)
            res["w4a4_over_bf16_throughput"] = round(res["bf16"]["ms"] / res["w4a4"]["ms"], 3)
            out[f"M{M}"] = res
    out["config"] = ("x M x 4096 bf16, w 4096 x 4096 NVFP4 (dynamic scales); w4a4 takes x pre-quantized; "
                     "L2 flushed before each launch")
    return out


def bench_kl(Q, dev, stream, P, K):
    from nvfp4_quantization_aware_b200 import synthetic as S
    with torch.cuda.stream(stream):
        d = S.distill_logits(seed=0, device=dev)
        t, s = d["teacher"], d["student"]
        rows, V = t.shape
        grad = torch.empty_like(s)
        loss = torch.empty(1, dtype=torch.float32, device=dev)
        ws = torch.empty(int(Q.lib().qad_kl_workspace_size(rows, V, Q.BF16)), dtype=torch.uint8, device=dev)
        L = Q.lib()
        sptr = stream.cuda_stream

        def call():
            st = L.qad_kl_fwd_bwd(t.data_ptr(), s.data_ptr(), Q.BF16, rows, V, V, 1.0, loss.data_ptr(), None,
                                  grad.data_ptr(), V, 1.0 / rows, ws.data_ptr(), ws.numel(), sptr)
            assert st == 0, st

        for _ in range(3):
            call()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(K):
            call()
        e1.record(stream)
        stream.synchronize()
    ms = e0.elapsed_time(e1) / K
    gbs = 6.0 * rows * V / (ms * 1e-3) / 1e9
    del t, s, grad, d
    torch.cuda.empty_cache()
    return {"tokens_per_s": round(rows / (ms * 1e-3), 1), "ms": round(ms, 4), "gbs": round(gbs, 1),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": P["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / P["hbm_gbs"], 4), "kernel": "kl_row_kernel<bf16>",
                         "algorithmic_bytes_per_launch": 6 * rows * V},
            "config": "teacher/student bf16 16384 x 131072, teacher N(0,3) + one +12 entry per row, student = teacher + N(0,1), T=1"}


MOE_CONFIG = ("MoE layer step: 4096 tokens x hidden 2048 bf16 N(0,1), top-6 of 128 experts (uniform) + 1 shared, "
              "expert FFN 2048->1024->2048 SwiGLU, NVFP4 W4A4 with frozen scales, grouped W4A4 GEMMs forward, "
              "straight-through BF16 backward (dx, dW_gate/up/down, d combine)")


def make_moe_step(Q, dev, tokens=4096, hidden=2048, ffn=1024, experts=128, topk=6, seed=0):
    """Synthetic config-5 layer on the device with its frozen scales (from a
    DYNAMIC quantization of the calibration weights) and the step object."""
    from nvfp4_quantization_aware_b200 import synthetic as S
    d = S.moe_layer(seed=seed, device=dev, tokens=tokens, hidden=hidden, ffn=ffn, experts=experts, topk=topk)
    w = {}
    for k in ("gate", "up", "down"):
        w0 = d.pop("w0_" + k)
        G, rows, cols = w0.shape
        _, sbs, ts = Q.nvfp4_quantize_grouped([w0[g] for g in range(G)], Q.DYNAMIC)
        sb = torch.cat(sbs).contiguous()
        del w0, sbs
        w["w_" + k] = d.pop("w_" + k).reshape(G * rows, cols).contiguous()
        w[k + "_ts"], w[k + "_sb"] = ts, sb
        w[k + "_sb_mma"] = Q.nvfp4_scales_to_mma(sb, G * rows, cols)
    w["x_ts"], w["a_ts"] = d["x_ts"], d["a_ts"]
    step = Q.MoeLayerStep(tokens, hidden, ffn, experts, topk, w)
    return d, w, step


def bench_moe(Q, dev, stream, P, K):
    """The config-5 layer step (forward + backward), K steps in one graph
    replay; per-phase times from events inside the graph."""
    tokens, hidden, ffn, experts, topk = 4096, 2048, 1024, 128, 6
    with torch.cuda.stream(stream):
        d, w, step = make_moe_step(Q, dev, tokens, hidden, ffn, experts, topk)
        x, ids, cw, dy = d["x"], d["ids"], d["combine"], d["dy"]
        y = torch.empty_like(x)
        G = experts + 1
        dx = torch.empty_like(x)
        dwg = torch.empty(G * ffn, hidden, dtype=torch.bfloat16, device=dev)
        dwu = torch.empty_like(dwg)
        dwd = torch.empty(G * hidden, ffn, dtype=torch.bfloat16, device=dev)
        dcw = torch.empty(tokens, topk, dtype=torch.float32, device=dev)

        def one():
            step.forward(x, ids, cw, y=y)
            step.backward(dy, dx=dx, dw_gate=dwg, dw_up=dwu, dw_down=dwd, d_combine=dcw)

        for _ in range(3):
            one()
        stream.synchronize()
        evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)] for _ in range(K)]
        g = torch.cuda.CUDAGraph()
        n0 = Q.nvfp4_launch_count()
        with torch.cuda.graph(g, stream=stream):
            for k in range(K):
                evs[k][0].record(stream)
                step.forward(x, ids, cw, y=y)
                evs[k][1].record(stream)
                step.backward(dy, dx=dx, dw_gate=dwg, dw_up=dwu, dw_down=dwd, d_combine=dcw)
                evs[k][2].record(stream)
        launches = Q.nvfp4_launch_count() - n0
        g.replay()
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        stream.synchronize()
        st, word = Q.nvfp4_device_error()
        del g
        phases = moe_phases(Q, stream, step, w, tokens, hidden, ffn, experts, K)
    ms = e0.elapsed_time(e1) / K
    fwd = statistics.mean(evs[k][0].elapsed_time(evs[k][1]) for k in range(K))
    bwd = statistics.mean(evs[k][1].elapsed_time(evs[k][2]) for k in range(K))
    rows = tokens * topk + tokens
    f_flops = 6.0 * rows * hidden * ffn         # gate, up, down (W4A4)
    b_flops = 12.0 * rows * hidden * ffn        # dA, dX (2F), dW x3 (BF16)
    wp = phases["weight_pass"]
    gf = phases["w4a4_gemms"]
    bf = {"ms": round(bwd, 4), "tflops": round(b_flops / (bwd * 1e-3) / 1e12, 1)}
    bf["frac"] = round(bf["tflops"] / P["bf16_tflops_sustained"], 4)
    bf["peak"] = P["bf16_tflops_sustained"]
    bf["peak_source"] = "MEASURED_PEAKS bf16_tflops_sustained (the backward runs inside a seconds-long step)"
    bf["what"] = "whole backward: 5 BF16 grouped GEMMs (dA, dX, dW x3) and the elementwise steps, 1.16e12 flop"
    fp4_peak = (P.get("fp4_probe") or {}).get("burst_tflops") or 4.0 * P["bf16_tflops"]
    gf["peak"] = fp4_peak
    gf["frac"] = round(gf["tflops"] / fp4_peak, 4)
    gf["peak_source"] = ("own tcgen05 FP4 MMA probe, burst" if (P.get("fp4_probe") or {}).get("burst_tflops")
                         else "4 x MEASURED_PEAKS bf16_tflops")
    out = {"tokens_per_s": round(tokens / (ms * 1e-3), 1), "ms_per_step": round(ms, 4),
           "forward_ms": round(fwd, 4), "backward_ms": round(bwd, 4),
           "forward_fp4_tflops": round(f_flops / (fwd * 1e-3) / 1e12, 1),
           "backward_bf16_tflops": round(b_flops / (bwd * 1e-3) / 1e12, 1),
           # dominant kernel of the step: the per-step weight pass (group_encode_kernel<bf16, Both>,
           # 3 launches over the 387 expert weights: master weight in, codes + bf16 W^ out)
           "roofline": {"bound": "hbm", "achieved": wp["gbs"], "peak": P["hbm_gbs"], "unit": "GB/s",
                        "frac": round(wp["gbs"] / P["hbm_gbs"], 4),
                        "kernel": "group_encode_kernel<bf16,Both> (FROZEN_ALL weight pass, 3 launches)",
                        "algorithmic_bytes_per_step": wp["bytes"], "avg_step_ms": wp["ms"],
                        "share_of_step": round(wp["ms"] / ms, 4), "peak_source": "measured (MEASURED_PEAKS hbm_gbs)"},
           "phases": {"weight_pass": wp, "w4a4_gemms_forward": gf, "bf16_backward": bf},
           "gpu_launches_per_step": int(launches // K), "device_error": [int(st), int(word)],
           "config": MOE_CONFIG + "; inputs larger than L2 (weights 3.2 GB), no flush"}
    del d, w, step, x, y, dx, dwg, dwu, dwd, dcw
    torch.cuda.empty_cache()
    return out


def _graph_ms(stream, fn, K):
    """Mean device time of fn() over K calls captured in one CUDA graph."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(K):
            fn()
    g.replay()
    stream.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g.replay()
    e1.record(stream)
    stream.synchronize()
    del g
    return e0.elapsed_time(e1) / K


def moe_phases(Q, stream, step, w, tokens, hidden, ffn, experts, K):
    """Two phases of the layer step timed on their own, with the step's own
    buffers (after a forward): the weight pass (FROZEN_ALL quantize of the 3 G
    master weights to codes + bf16 W^, exactly the step's first call) and the
    three grouped W4A4 GEMMs of the forward."""
    G, H, F = experts + 1, hidden, ffn
    wg, wu, wd = w["w_gate"], w["w_up"], w["w_down"]
    cg, cu, cd = step.buffer("wg_codes"), step.buffer("wu_codes"), step.buffer("wd_codes")
    hgu, hd = step.buffer("wgu_hat"), step.buffer("wd_hat")
    xs = ([wg[g * F:(g + 1) * F] for g in range(G)] + [wu[g * F:(g + 1) * F] for g in range(G)] +
          [wd[g * H:(g + 1) * H] for g in range(G)])
    ts = ([w["gate_ts"][g:g + 1] for g in range(G)] + [w["up_ts"][g:g + 1] for g in range(G)] +
          [w["down_ts"][g:g + 1] for g in range(G)])
    sbs = ([w["gate_sb"][g * F:(g + 1) * F] for g in range(G)] + [w["up_sb"][g * F:(g + 1) * F] for g in range(G)] +
           [w["down_sb"][g * H:(g + 1) * H] for g in range(G)])
    codes = ([cg[g * F:(g + 1) * F] for g in range(G)] + [cu[g * F:(g + 1) * F] for g in range(G)] +
             [cd[g * H:(g + 1) * H] for g in range(G)])
    ys = ([hgu[2 * g * F:2 * g * F + F] for g in range(G)] + [hgu[2 * g * F + F:2 * (g + 1) * F] for g in range(G)] +
          [hd[g * H:(g + 1) * H] for g in range(G)])
    wp_ms = _graph_ms(stream, lambda: Q.nvfp4_quantize_fake_quant_grouped(xs, Q.FROZEN_ALL, ts, sbs, codes=codes,
                                                                           ys=ys), K)
    n = sum(x.numel() for x in xs)
    wp_bytes = n * (2.0 + 0.0625 + 0.5 + 2.0)  # bf16 in, block scales in, codes + bf16 W^ out
    seg_off, seg_len = step.buffer("seg_off"), step.buffer("seg_len")
    xc, xsf, ac, asf = step.buffer("x_codes"), step.buffer("x_scales"), step.buffer("a_codes"), step.buffer("a_scales")
    hg, hu, yr = step.buffer("h_gate"), step.buffer("h_up"), step.buffer("y_rows")

    def gemms():
        Q.nvfp4_gemm_w4a4_grouped(xc, xsf, w["x_ts"], seg_off, seg_len, cg, w["gate_sb_mma"], w["gate_ts"], F, out=hg)
        Q.nvfp4_gemm_w4a4_grouped(xc, xsf, w["x_ts"], seg_off, seg_len, cu, w["up_sb_mma"], w["up_ts"], F, out=hu)
        Q.nvfp4_gemm_w4a4_grouped(ac, asf, w["a_ts"], seg_off, seg_len, cd, w["down_sb_mma"], w["down_ts"], H, out=yr)

    g_ms = _graph_ms(stream, gemms, K)
    rows = tokens * 6 + tokens
    g_flops = 6.0 * rows * H * F
    return {"weight_pass": {"ms": round(wp_ms, 4), "bytes": int(wp_bytes), "gbs": round(wp_bytes / (wp_ms * 1e-3) / 1e9, 1),
                            "what": "FROZEN_ALL quantize of the 3 x 129 master weights to codes + bf16 W^ (811.6M elements, 4.5625 B each)"},
            "w4a4_gemms": {"ms": round(g_ms, 4), "tflops": round(g_flops / (g_ms * 1e-3) / 1e12, 1),
                           "what": "grouped W4A4 gate, up and down over the 28672 routed + shared rows (useful flop, padding excluded)"}}


def bench_kl_topk(Q, dev, stream, P, K, k=4096):
    """Top-k KL over the distillation logits (k = 4096 of 131072): each logit
    is still read once and every dLogit written (zero outside the set), so the
    algorithmic bytes are those of the full loss."""
    from nvfp4_quantization_aware_b200 import synthetic as S
    with torch.cuda.stream(stream):
        d = S.distill_logits(seed=0, device=dev)
        t, s = d["teacher"], d["student"]
        rows, V = t.shape
        grad = torch.empty_like(s)
        loss = torch.empty(1, dtype=torch.float32, device=dev)
        ws = torch.empty(int(Q.lib().qad_kl_workspace_size(rows, V, Q.BF16)), dtype=torch.uint8, device=dev)
        L = Q.lib()
        sptr = stream.cuda_stream

        def call():
            st = L.qad_kl_topk_fwd_bwd(t.data_ptr(), s.data_ptr(), Q.BF16, rows, V, V, k, 1.0, loss.data_ptr(), None,
                                       grad.data_ptr(), V, 1.0 / rows, ws.data_ptr(), ws.numel(), sptr)
            assert st == 0, st

        for _ in range(3):
            call()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(K):
            call()
        e1.record(stream)
        stream.synchronize()
    ms = e0.elapsed_time(e1) / K
    gbs = 6.0 * rows * V / (ms * 1e-3) / 1e9
    del t, s, grad, d
    torch.cuda.empty_cache()
    return {"tokens_per_s": round(rows / (ms * 1e-3), 1), "ms": round(ms, 4), "gbs": round(gbs, 1), "k": k,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": P["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / P["hbm_gbs"], 4), "kernel": "kl_topk_row_kernel<bf16>",
                         "algorithmic_bytes_per_launch": 6 * rows * V},
            "config": "distillation logits 16384 x 131072 bf16 (as kl), KL over the teacher's top-4096 per row"}


def bench_kl_topp(Q, dev, stream, P, K, p=0.95):
    """Top-p KL (the pages' suggested replacement for top-k) on the same
    distillation logits: tokens per second; also the mean set size."""
    from nvfp4_quantization_aware_b200 import synthetic as S
    with torch.cuda.stream(stream):
        d = S.distill_logits(seed=0, device=dev)
        t, s = d["teacher"], d["student"]
        rows, V = t.shape
        grad = torch.empty_like(s)
        ws = torch.empty(int(Q.lib().qad_kl_topp_workspace_size(rows, V, Q.BF16)), dtype=torch.uint8, device=dev)
        for _ in range(2):
            _, _, _, ks = Q.qad_kl_topp_fwd_bwd(t, s, p, dlogits=grad, workspace=ws, want_row_k=True)
        stream.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(K):
            Q.qad_kl_topp_fwd_bwd(t, s, p, dlogits=grad, workspace=ws)
        e1.record(stream)
        stream.synchronize()
        mean_k = float(ks.double().mean())
    ms = e0.elapsed_time(e1) / K
    del t, s, grad, d
    torch.cuda.empty_cache()
    gbs = 6.0 * rows * V / (ms * 1e-3) / 1e9
    return {"tokens_per_s": round(rows / (ms * 1e-3), 1), "ms": round(ms, 4), "gbs": round(gbs, 1), "p": p,
            "mean_set_size": round(mean_k, 1),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": P["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / P["hbm_gbs"], 4),
                         "kernel": "kl_topp_count_kernel<bf16> + kl_topk_row_kernel<bf16> (whole loss)",
                         "algorithmic_bytes_per_launch": 6 * rows * V},
            "config": "distillation logits 16384 x 131072 bf16 (as kl), KL over the teacher's top-p set per row "
                      "(set size kernel + top-k kernel with a k per row)"}


def bench_calibrate(Q, dev, stream, xs, K):
    """MSE block-scale calibration of the 128 expert weights (the frozen
    scales' starting point): elements per second and GB/s of input read."""
    exp = xs[:128]
    with torch.cuda.stream(stream):
        _, _, ts = Q.nvfp4_quantize_grouped(exp, Q.DYNAMIC)
        sbs = [torch.empty(x.shape[0], x.shape[1] // 16, dtype=torch.uint8, device=dev) for x in exp]
        Q.nvfp4_calibrate_mse_grouped(exp, ts, block_scales=sbs)
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(K):
            Q.nvfp4_calibrate_mse_grouped(exp, ts, block_scales=sbs)
        e1.record(stream)
        stream.synchronize()
    ms = e0.elapsed_time(e1) / K
    n = sum(x.numel() for x in exp)
    return {"ms": round(ms, 4), "gelem_per_s": round(n / (ms * 1e-3) / 1e9, 2),
            "config": "128 expert weights 2048x1024 bf16, s_g from amax, exhaustive search over E4M3 block scales"}


def cpu_baseline(xs):
    """The oracle (as it stands) on the host cores: dynamic then frozen
    quantize of the 128 expert weights (268M elements; the lm_head is left out
    to bound the time)."""
    import oracle as O
    cores = len(os.sched_getaffinity(0))
    O.set_threads(cores)
    hx = [x.float().cpu().numpy() for x in xs[:128]]
    t0 = time.perf_counter()
    for x in hx:
        c, sb, sg = O.quantize(x, O.DYNAMIC)
        O.quantize(x, O.FROZEN_ALL, s_g=sg, s_b=sb)
    dt = time.perf_counter() - t0
    n_elem = sum(x.size for x in hx)
    return {"value": round(n_elem * 2 * BYTES_PER_ELEM / dt / 1e9, 4), "unit": "GB/s", "cores": O.get_threads(),
            "kind": "oracle", "sample": f"128 expert weights 2048x1024 ({n_elem} elements), dynamic + frozen, {dt:.1f} s"}


# --------------------------------------------------------------------------- reference arm

def run_reference(args, world, rank):
    if rank != 0:
        return
    import oracle as O
    from nvfp4_quantization_aware_b200 import synthetic as S
    cores = len(os.sched_getaffinity(0))
    O.set_threads(cores)
    per_step = 8  # expert weights per step: a bounded sample of the sweep
    xs = [S.weights(2048, 1024, seed=i).float().numpy() for i in range(per_step)]

    def step():
        for x in xs:
            c, sb, sg = O.quantize(x, O.DYNAMIC)
            O.quantize(x, O.FROZEN_ALL, s_g=sg, s_b=sb)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    n_elem = sum(x.size for x in xs)
    value = n_elem * 2 * BYTES_PER_ELEM / dt / 1e9
    sample = f"{per_step} expert weights 2048x1024 per step ({n_elem} elements), dynamic + frozen"
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample": sample},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": O.get_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_profile_case(case: str):
    """Small single-kernel cases for ncu captures (inputs larger than L2, a
    few GB on the device at most): each kernel runs 2 warm-up + 3 launches."""
    import nvfp4_quantization_aware_b200 as Q
    from nvfp4_quantization_aware_b200 import synthetic as S
    dev = torch.device("cuda", 0)
    if case == "quant":
        xs = S.weight_sweep(seed=0, device=dev, experts=48, lm_head=False)  # 48 x 4 MiB = 201 MB
        ts = torch.zeros(len(xs), device=dev)
        sbs = [torch.empty(x.shape[0], x.shape[1] // 16, dtype=torch.uint8, device=dev) for x in xs]
        cd = [torch.empty(x.shape[0], x.shape[1] // 2, dtype=torch.uint8, device=dev) for x in xs]
        for _ in range(5):
            Q.nvfp4_quantize_grouped(xs, Q.DYNAMIC, tensor_scales=ts, block_scales=sbs, codes=cd)
            Q.nvfp4_quantize_grouped(xs, Q.FROZEN_ALL, tensor_scales=ts, block_scales=sbs, codes=cd)
    elif case == "gemm":
        w = S.weights(4096, 4096, seed=1, device=dev)
        x = S.channel_scaled_activations(8192, 4096, seed=0, device=dev)
        a = Q.nvfp4_quantize(x, Q.DYNAMIC, layout=Q.SCALES_MMA)
        b = Q.nvfp4_quantize(w, Q.DYNAMIC, layout=Q.SCALES_MMA)
        for _ in range(5):
            Q.nvfp4_gemm_w4a4(*a, *b)
    elif case == "gemm_small":
        w = S.weights(4096, 4096, seed=1, device=dev)
        x = S.channel_scaled_activations(128, 4096, seed=0, device=dev)
        a = Q.nvfp4_quantize(x, Q.DYNAMIC, layout=Q.SCALES_MMA)
        b = Q.nvfp4_quantize(w, Q.DYNAMIC, layout=Q.SCALES_MMA)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        for _ in range(5):
            flush_l2(flush)
            Q.nvfp4_gemm_w4a4(*a, *b)
    elif case == "moe":
        d, w, step = make_moe_step(Q, dev)
        for _ in range(3):
            step.forward(d["x"], d["ids"], d["combine"])
            step.backward(d["dy"])
    elif case == "kl":
        d = S.distill_logits(seed=0, device=dev, rows=2048)  # 2 x 512 MiB
        for _ in range(5):
            Q.qad_kl_fwd_bwd(d["teacher"], d["student"])
    elif case == "kl_topk":
        d = S.distill_logits(seed=0, device=dev, rows=2048)
        for _ in range(5):
            Q.qad_kl_topk_fwd_bwd(d["teacher"], d["student"], 4096)
    elif case == "kl_topp":
        d = S.distill_logits(seed=0, device=dev, rows=2048)
        for _ in range(5):
            Q.qad_kl_topp_fwd_bwd(d["teacher"], d["student"], 0.95)
    elif case == "w4a16":
        w = S.weights(4096, 4096, seed=1, device=dev)
        x = S.channel_scaled_activations(8192, 4096, seed=0, device=dev)
        codes, sb, ts = Q.nvfp4_quantize(w, Q.DYNAMIC)
        for _ in range(5):
            Q.nvfp4_gemm_w4a16(x, codes, sb, ts)
    elif case == "calibrate":
        xs = S.weight_sweep(seed=0, device=dev, experts=48, lm_head=False)
        ts = torch.zeros(len(xs), device=dev)
        Q.nvfp4_quantize_grouped(xs, Q.DYNAMIC, tensor_scales=ts)
        for _ in range(5):
            Q.nvfp4_calibrate_mse_grouped(xs, ts)
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": case, "ok": True}))


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-secondary", action="store_true", help="skip the GEMM and KL measurements")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", choices=["quant", "gemm", "gemm_small", "kl", "kl_topk", "kl_topp", "w4a16", "calibrate",
                             "moe"],
                    default=None,
                    help="run one small single-kernel case (for ncu captures) and exit")
    args = ap.parse_args()
    if args.profile:
        run_profile_case(args.profile)
        return
    if args.warmup < 3:
        args.warmup = 3
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: start the ranks under torch.distributed.run (NCCL)
        # and return its status; the bound on the whole job is well above the
        # process group's own timeout
        port = os.environ.get("MASTER_PORT", "29517")
        cmd = ["timeout", "-k", "60", "1800", sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
               f"--nproc-per-node={args.gpus}", "--master-addr=127.0.0.1", f"--master-port={port}",
               os.path.abspath(__file__), *sys.argv[1:]]
        sys.exit(subprocess.call(cmd))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != args.gpus and args.gpus > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    world, rank, local = dist_init()
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
