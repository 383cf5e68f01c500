#!/usr/bin/env python
"""Benchmark of the QLoRA linear layer (NF4 frozen weight + LoRA adapters) on B200.

One step = the layer's forward and backward on one batch of synthetic tokens,
i.e. h = x W~^T + (alpha/r)(x A^T)B^T, then dX, dA, dB (with the adapter
gradients all-reduced across ranks when N > 1). Workload: the LLaMA-13B-like
attention projection (W0 5120x5120 NF4 with double quantisation, 2048 tokens,
r = 16, alpha = 32). value = algorithmic fwd+bwd FLOP/s over all ranks.

Every rank also reports the end-to-end speed through the public API with host
buffers. At N = 1 the same run adds: the decode-shaped forward (W0 13824x5120,
M in {1,4,16}) as GB/s of 4-bit weight codes, the full-weight quantisation of
the Llama-2-70B-like MLP weight (28672x8192) as GB/s moved, that MLP's
fwd+bwd, the 160-projection stack, the adapter merge, the multi-adapter
forward, the step with 128-element blocks, the step with LoRA dropout, and
the CPU oracle's speed on a bounded sample.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                       [--skip-extras] [--leg decode|quantize|stack|mlp70b|merge|multi|block128|dropout]
       (N > 1: launch under torch.distributed.run, one rank per GPU)
"""
import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "QLoRA linear fwd+bwd TFLOP/s (large M) & NF4 weight GB/s (decode) vs roofline"
# DRAM bytes (read + write) per launch of the fused GEMM on this workload, mean of the forward and
# dgrad launches, from one ncu capture of the kernels as they are now (summary and command under
# profiles/). None whenever the kernel has changed since that capture.
GEMM_TRAFFIC_BYTES = 42.3e6
MAIN = "llama13b_attn_5120"
DECODE = "decode_mlp_up_13824x5120"
QUANT = "llama2_70b_mlp_28672x8192"
STACK = "llama13b_stack_40x4"
L2_FLUSH_BYTES = 512 << 20


def layer_flops(M, N, K, r):
    """Algorithmic FLOPs of one forward and one backward of the layer."""
    fwd = 2 * M * N * K + 2 * M * r * (K + N)
    bwd = 2 * M * N * K + 4 * M * N * r + 4 * M * K * r
    return fwd, bwd


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# --------------------------------------------------------------------------
# clocks during the timed region (NVML reads only)
# --------------------------------------------------------------------------
class ClockSampler:
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index, period_s=0.002):
        self.samples, self.reasons = [], 0
        self.period = period_s
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            handle = None
            try:
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                if not uuid.startswith("GPU-"):
                    uuid = "GPU-" + uuid
                handle = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            except Exception:
                handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.h = handle
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: report that instead of clocks
            self.err = str(e)
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                try:
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:
                    r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.reasons |= int(r)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"error": getattr(self, "err", "nvml unavailable")}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples), "reasons": names}


# --------------------------------------------------------------------------
# CPU oracle on a bounded sample (the reported baseline and the reference arm)
# --------------------------------------------------------------------------
def oracle_weight(w, inp):
    """The workload's frozen weight quantised once by the oracle (not timed: it is
    not part of a training step)."""
    import oracle
    return oracle.quantize(inp["W0"].numpy().reshape(-1), dq=w.double_quant)


def oracle_sample_step(w, inp, tokens, qw):
    """Oracle forward+backward on the first `tokens` tokens of the workload.
    Returns (flops, seconds)."""
    import oracle
    bits = workloads.bf16_bits
    x, A, B = bits(inp["x"][:tokens]), bits(inp["A"]), bits(inp["B"])
    dY = bits(inp["dY"][:tokens])
    t0 = time.perf_counter()
    oracle.qlora_fwd_rows(qw, w.N, w.K, x, A, B, w.r, w.alpha)
    oracle.qlora_bwd(qw, w.N, w.K, x, A, B, w.r, w.alpha, dY)
    dt = time.perf_counter() - t0
    f, b = layer_flops(tokens, w.N, w.K, w.r)
    return f + b, dt


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count()


def run_reference(args, rank, world):
    """The oracle as it stands, timed on the host cores (rank 0 only)."""
    if rank != 0:
        return
    w = workloads.WORKLOADS[MAIN]
    tokens = 4
    inp = workloads.make_inputs(w, M=tokens)
    qw = oracle_weight(w, inp)
    for _ in range(args.warmup):
        oracle_sample_step(w, inp, tokens, qw)
    tot_f, tot_t = 0, 0.0
    for _ in range(args.steps):
        f, t = oracle_sample_step(w, inp, tokens, qw)
        tot_f += f
        tot_t += t
    value = tot_f / tot_t / 1e12
    sample = (f"{tokens} of the {w.M} tokens per step: full forward and backward of those "
              f"tokens (h, dX rows, and their dA/dB contributions), W0 dequantised each step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{MAIN}: W0 5120x5120 NF4 double-quant, x {w.M}x5120 bf16, "
                               f"r=16, alpha=32, forward+backward", "parallelism": "cpu-oracle"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--skip-extras", action="store_true",
                    help="only the main fwd+bwd line (no decode/quantize/oracle/e2e legs)")
    ap.add_argument("--leg", default="all", choices=["all", "decode", "quantize", "stack", "mlp70b",
                                                     "merge", "multi", "block128", "dropout"],
                    help="run one secondary leg alone and print its JSON (for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import bit_nf4_quantized_05_b200 as q
    from bit_nf4_quantized_05_b200 import dp

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if args.leg != "all":
        if rank == 0:
            leg = {"decode": decode_leg, "quantize": quantize_leg, "stack": stack_leg,
                   "mlp70b": mlp70b_leg, "merge": merge_leg, "multi": multi_leg,
                   "block128": block128_leg, "dropout": dropout_leg}[args.leg]
            print(json.dumps({"leg": args.leg, **leg(q, dev, load_peaks())}), flush=True)
        return
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    peaks = load_peaks()

    w = workloads.WORKLOADS[MAIN]
    M, N, K, r, alpha = w.M, w.N, w.K, w.r, w.alpha
    inp = workloads.make_inputs(w)
    qw = q.nf4_quantize(inp["W0"].to(dev), double_quant=w.double_quant)
    x, A, B, dY = (inp[k].to(dev) for k in ("x", "A", "B", "dY"))
    h = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    u = torch.empty(M, r, dtype=torch.float32, device=dev)
    dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    flat, dA, dB = dp.grad_buffer(r, K, N, device=dev)
    ws_f = torch.empty(q.fwd_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(q.bwd_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step(xx=x, dYY=dY):
        q.qlora_linear_fwd(qw, xx, A, B, alpha, h=h, u=u, workspace=ws_f)
        q.qlora_linear_bwd(qw, xx, A, B, alpha, dYY, u=u, workspace=ws_b, outs=(dX, dA, dB))
        dp.allreduce_adapter_grads(flat, world)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = q.device_status(dev)
    if st != q.NF4_OK:
        raise RuntimeError(f"device status after warm-up: {q.status_string(st)}")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    # Timed region: K steps with only the two step events each (per-launch
    # events would sit between the kernels and stop each launch from
    # overlapping the tail of the one before).
    with ClockSampler(local_rank) as clk:
        for i in range(args.steps):
            flush.zero_()                      # L2 flush between timed steps (untimed)
            starts[i].record()
            step()
            ends[i].record()
        torch.cuda.synchronize()
    barrier()
    # Kernel durations: the same K steps again with the library's per-launch
    # CUDA events (recorded on the stream each kernel is launched on).
    q.profiling(True)
    for i in range(args.steps):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    barrier()
    q.profiling(False)
    prof = q.profile_read()
    per_step = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms = statistics.mean(per_step)
    if world > 1:
        t = torch.tensor([ms], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = float(t.item())
    f_fwd, f_bwd = layer_flops(M, N, K, r)
    value = world * (f_fwd + f_bwd) / (ms * 1e-3) / 1e12

    # roofline of the dominant kernel: the fused dequant-GEMM (forward + dgrad launches)
    g_launch = sum(prof.get(k, (0, 0.0))[0] for k in ("qlora_gemm_fwd", "qlora_gemm_dgrad"))
    g_ms = sum(prof.get(k, (0, 0.0))[1] for k in ("qlora_gemm_fwd", "qlora_gemm_dgrad"))
    g_flops = args.steps * ((2 * M * N * K + 2 * M * N * r) + (2 * M * N * K + 2 * M * K * r))
    g_tflops = g_flops / (g_ms * 1e-3) / 1e12 if g_ms > 0 else None
    roofline = {"bound": "tensor", "achieved": g_tflops, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": (g_tflops / peaks["bf16_tflops"]) if g_tflops else None,
                "traffic": GEMM_TRAFFIC_BYTES, "traffic_unit": "bytes per launch (ncu dram read + write)",
                "kernel": "qlora_gemm (forward + dgrad launches)",
                "peak_source": peaks["source"] + " bf16 burst",
                "avg_launch_us": 1e3 * g_ms / max(g_launch, 1)}
    kernels = {k: {"launches": n, "avg_us": 1e3 * t / max(n, 1), "share": t / max(
        sum(v[1] for v in prof.values()), 1e-12)} for k, (n, t) in prof.items()}
    gpu_launches = sum(n for n, _ in prof.values())

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"{MAIN}: W0 {N}x{K} NF4 (blocks of 64, double quant), "
                               f"x {M}x{K} bf16 per rank, r={r}, alpha={alpha:g}, fwd+bwd",
                   "global_batch_tokens": M * world, "parallelism": f"dp{world}",
                   "l2": "512 MiB buffer written before every timed step (outside the events)"},
        "roofline": roofline,
        "gpu_launches": gpu_launches,
        "clocks": clk.summary(),
        "kernels": kernels,
    }

    if not args.skip_extras:
        # every rank takes the same collective steps in the end-to-end leg
        e2e = e2e_leg(q, dp, qw, inp, w, args, dev, world)
        if rank == 0:
            line["e2e"] = e2e
    if rank == 0 and world == 1 and not args.skip_extras:
        # single-GPU legs: at N > 1 the other ranks would wait in the closing
        # barrier for minutes, beyond the process group's timeout
        line["decode"] = decode_leg(q, dev, peaks)
        line["quantize"] = quantize_leg(q, dev, peaks)
        line["mlp70b"] = mlp70b_leg(q, dev, peaks)
        line["stack"] = stack_leg(q, dev, peaks)
        line["merge"] = merge_leg(q, dev, peaks)
        line["multi_adapter"] = multi_leg(q, dev, peaks)
        line["block128"] = block128_leg(q, dev, peaks)
        line["dropout"] = dropout_leg(q, dev, peaks)
        line["cpu_baseline"] = cpu_baseline_leg(w, inp)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def e2e_leg(q, dp, qw, inp, w, args, dev, world):
    """Same metric through the public API with host buffers: every step copies
    x and dY in from pinned host memory and h, dX, dA, dB back out."""
    M, N, K, r, alpha = w.M, w.N, w.K, w.r, w.alpha
    hx = inp["x"].pin_memory()
    hdY = inp["dY"].pin_memory()
    oh = torch.empty(M, N, dtype=torch.bfloat16).pin_memory()
    odX = torch.empty(M, K, dtype=torch.bfloat16).pin_memory()
    ograd = torch.empty(r * K + N * r, dtype=torch.bfloat16).pin_memory()
    A, B = inp["A"].to(dev), inp["B"].to(dev)
    x = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    dY = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    flat, dA, dB = dp.grad_buffer(r, K, N, device=dev)

    def step():
        x.copy_(hx, non_blocking=True)
        dY.copy_(hdY, non_blocking=True)
        h, u = q.qlora_linear_fwd(qw, x, A, B, alpha)
        dX, _, _ = q.qlora_linear_bwd(qw, x, A, B, alpha, dY, u=u, outs=(torch.empty_like(x), dA, dB))
        dp.allreduce_adapter_grads(flat, world)
        oh.copy_(h, non_blocking=True)
        odX.copy_(dX, non_blocking=True)
        ograd.copy_(flat, non_blocking=True)

    steps = max(5, min(args.steps, 20))
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        step()
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    if world > 1:
        t = torch.tensor([ms], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = float(t.item())
    f, b = layer_flops(M, N, K, r)
    return {"value": world * (f + b) / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "ms_per_step": ms, "h2d_bytes_per_step": hx.nbytes + hdY.nbytes,
            "d2h_bytes_per_step": oh.nbytes + odX.nbytes + ograd.nbytes}


def decode_leg(q, dev, peaks, block=64, tokens=(1, 4, 16)):
    """Decode-shaped forward, GB/s counted on the 4-bit code bytes; 8 weight
    copies are rotated so that no call finds its weight in L2. The headline
    per-call time is device time from a CUDA-graph replay of back-to-back
    calls (both kernels of a call, the u partials and the weight stream)."""
    w = workloads.WORKLOADS[DECODE]
    W0 = workloads.make_weight(w).to(dev)
    copies = [q.nf4_quantize(W0, double_quant=True, block_size=block) for _ in range(8)]
    del W0
    code_bytes = w.N * w.K // 2
    out = {"workload": f"{DECODE}: W0 {w.N}x{w.K} NF4 (blocks of {block}) double quant "
                       f"(0.1% x20 outliers), r={w.r}; forward only", "code_bytes": code_bytes,
           "peak_gbs": peaks["hbm_gbs"]}
    for M in tokens:
        inp = workloads.make_inputs(w, M=M, with_dy=False)
        x, A, B = (inp[k].to(dev) for k in ("x", "A", "B"))
        h = torch.empty(M, w.N, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(q.fwd_workspace_bytes(M, w.N, w.K, w.r), dtype=torch.uint8, device=dev)
        for i in range(8):
            q.qlora_linear_fwd(copies[i], x, A, B, w.alpha, save_u=False, h=h, workspace=ws)
        torch.cuda.synchronize()
        iters = 64
        # (1) device time per call: 64 back-to-back calls captured in one CUDA
        # graph and replayed, so the host's per-call work (binding, argument
        # checks, launches) is not on the clock
        gs = torch.cuda.Stream()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=gs):
            for i in range(iters):
                q.qlora_linear_fwd(copies[i % 8], x, A, B, w.alpha, save_u=False, h=h, workspace=ws)
        graph.replay()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(4):
            graph.replay()
        e.record()
        torch.cuda.synchronize()
        graph_us = 1e3 * s.elapsed_time(e) / (4 * iters)
        del graph
        # (2) the same calls issued one by one from Python (host path on the clock)
        s.record()
        for i in range(iters):
            q.qlora_linear_fwd(copies[i % 8], x, A, B, w.alpha, save_u=False, h=h, workspace=ws)
        e.record()
        torch.cuda.synchronize()
        call_us = 1e3 * s.elapsed_time(e) / iters
        # (3) per-kernel CUDA events (they include the host's launch gaps)
        q.profiling(True)
        for i in range(iters):
            q.qlora_linear_fwd(copies[i % 8], x, A, B, w.alpha, save_u=False, h=h, workspace=ws)
        torch.cuda.synchronize()
        q.profiling(False)
        prof = q.profile_read()
        kern = {k: 1e3 * t / max(n, 1) for k, (n, t) in prof.items()}
        out[f"M{M}"] = {"graph_call_us": graph_us,
                        "gbs_graph_call": code_bytes / (graph_us * 1e-6) / 1e9,
                        "frac_graph_call": code_bytes / (graph_us * 1e-6) / 1e9 / peaks["hbm_gbs"],
                        "host_call_us": call_us, "kernel_event_us": kern}
    del copies
    torch.cuda.empty_cache()
    return out


def quantize_leg(q, dev, peaks, block=64):
    """Full-weight nf4_quantize of the 28672x8192 fp32 weight (double quant)."""
    w = workloads.WORKLOADS[QUANT]
    W0 = workloads.make_weight(w).to(dev)
    qw = q.nf4_quantize(W0, double_quant=True, block_size=block)
    torch.cuda.synchronize()
    nb = w.N * w.K // block
    moved = w.N * w.K * 4 + w.N * w.K // 2 + nb * 4 + nb + ((nb + 255) // 256) * 4
    iters = 10
    q.profiling(True)
    for _ in range(iters):
        q.nf4_quantize(W0, double_quant=True, out=qw)
    torch.cuda.synchronize()
    q.profiling(False)
    n, t = q.profile_read()["nf4_quantize"]
    us = 1e3 * t / n
    gbs = moved / (us * 1e-6) / 1e9
    # the same weight stored as bf16 (half the bytes in)
    W16 = W0.to(torch.bfloat16)
    del W0
    moved16 = moved - w.N * w.K * 2
    q.nf4_quantize(W16, double_quant=True, out=qw)
    torch.cuda.synchronize()
    q.profiling(True)
    for _ in range(iters):
        q.nf4_quantize(W16, double_quant=True, out=qw)
    torch.cuda.synchronize()
    q.profiling(False)
    n16, t16 = q.profile_read()["nf4_quantize"]
    us16 = 1e3 * t16 / n16
    gbs16 = moved16 / (us16 * 1e-6) / 1e9
    del W16, qw
    torch.cuda.empty_cache()
    return {"workload": f"{QUANT}: W0 {w.N}x{w.K} fp32 -> NF4 (blocks of {block}) + double quant",
            "bytes_moved": moved, "kernel_us": us, "gbs": gbs, "frac": gbs / peaks["hbm_gbs"],
            "peak_gbs": peaks["hbm_gbs"],
            "bf16_input": {"bytes_moved": moved16, "kernel_us": us16, "gbs": gbs16,
                           "frac": gbs16 / peaks["hbm_gbs"]}}


def multi_leg(q, dev, peaks):
    """Decode-shaped forward with per-token adapters over one NF4 base: the 13824x5120 weight
    (double quant), 16 tokens spread over 8 adapters of rank 8 (alpha 16), as one batch of a
    multi-adapter server. Device time per call from a CUDA-graph replay of 64 calls over 8
    rotated weight copies; GB/s on the 4-bit code bytes, as the decode leg."""
    w = workloads.WORKLOADS[DECODE]
    n_ad, r, M = 8, 8, 16
    W0 = workloads.make_weight(w).to(dev)
    copies = [q.nf4_quantize(W0, double_quant=True) for _ in range(8)]
    del W0
    wl = w.with_(r=n_ad * r)
    inp = workloads.make_inputs(wl, M=M, with_dy=False)
    x, A_all, B_all = (inp[k].to(dev) for k in ("x", "A", "B"))
    idx = (torch.arange(M, dtype=torch.int32) % n_ad).to(dev)
    alphas = [16.0] * n_ad
    h = torch.empty(M, w.N, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(q.fwd_workspace_bytes(M, w.N, w.K, n_ad * r), dtype=torch.uint8, device=dev)
    for i in range(8):
        q.qlora_multi_lora_fwd(copies[i], x, A_all, B_all, r, alphas, idx, h=h, workspace=ws)
    torch.cuda.synchronize()
    gs = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=gs):
        for i in range(64):
            q.qlora_multi_lora_fwd(copies[i % 8], x, A_all, B_all, r, alphas, idx, h=h, workspace=ws)
    graph.replay()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(4):
        graph.replay()
    e.record()
    torch.cuda.synchronize()
    us = 1e3 * s.elapsed_time(e) / (4 * 64)
    del graph, copies
    torch.cuda.empty_cache()
    code_bytes = w.N * w.K // 2
    gbs = code_bytes / (us * 1e-6) / 1e9
    return {"workload": f"{DECODE}: W0 {w.N}x{w.K} NF4 double quant; {M} tokens over {n_ad} "
                        f"adapters of r={r} (alpha 16), forward", "graph_call_us": us,
            "gbs_graph_call": gbs, "frac_graph_call": gbs / peaks["hbm_gbs"], "code_bytes": code_bytes}


def merge_leg(q, dev, peaks):
    """Adapter merge W~ + (alpha/r) B A of the 5120x5120 attention projection (r = 16), to a
    bf16 and to an fp32 weight. GB/s counts the bytes a merge must move: codes, 8-bit scale
    codes and group constants in, the merged weight out (the adapters are 0.3 MB). Four
    weight copies and outputs are rotated so that no launch finds its operands in L2."""
    w = workloads.WORKLOADS[MAIN]
    inp = workloads.make_inputs(w, M=0, with_dy=False)
    W0 = inp["W0"].to(dev)
    copies = [q.nf4_quantize(W0, double_quant=True) for _ in range(4)]
    del W0
    A, B = inp["A"].to(dev), inp["B"].to(dev)
    nb = w.N * w.K // 64
    out = {"workload": f"{MAIN}: W0 {w.N}x{w.K} NF4 double quant, r={w.r}, alpha={w.alpha:g}",
           "peak_gbs": peaks["hbm_gbs"]}
    for name, bf16 in (("bf16", True), ("fp32", False)):
        outs = [torch.empty(w.N, w.K, dtype=torch.bfloat16 if bf16 else torch.float32, device=dev)
                for _ in range(4)]
        moved = w.N * w.K // 2 + nb + ((nb + 255) // 256) * 4 + w.N * w.K * (2 if bf16 else 4)
        for i in range(4):
            q.qlora_merge(copies[i], A, B, w.alpha, bf16=bf16, out=outs[i])
        torch.cuda.synchronize()
        q.profiling(True)
        for i in range(20):
            q.qlora_merge(copies[i % 4], A, B, w.alpha, bf16=bf16, out=outs[i % 4])
        torch.cuda.synchronize()
        q.profiling(False)
        n, t = q.profile_read()["qlora_merge"]
        us = 1e3 * t / n
        gbs = moved / (us * 1e-6) / 1e9
        out[name] = {"bytes_moved": moved, "kernel_us": us, "gbs": gbs, "frac": gbs / peaks["hbm_gbs"]}
        del outs
    del copies
    torch.cuda.empty_cache()
    return out


def dropout_leg(q, dev, peaks, steps=50, p=0.05):
    """The main workload's forward + backward with LoRA dropout p = 0.05 on the adapter input
    (a seeded keep mask, drawn once): the rank-r kernels mask the landed x tiles, the dgrad
    GEMM writes dY W~ in fp32 and the adapter-add kernel masks, adds and rounds dX once.
    The adapter-add kernel is HBM-bound: it reads the fp32 base (4 B), writes dX (2 B) and
    reads the mask (1/8 B) per element of dX."""
    w = workloads.WORKLOADS[MAIN]
    M, N, K, r, alpha = w.M, w.N, w.K, w.r, w.alpha
    inp = workloads.make_inputs(w)
    qw = q.nf4_quantize(inp["W0"].to(dev), double_quant=w.double_quant)
    x, A, B, dY = (inp[k].to(dev) for k in ("x", "A", "B", "dY"))
    g = torch.Generator(device="cpu").manual_seed(w.seed + 17)
    keep = q.pack_keep((torch.rand(M, K, generator=g) >= p).to(dev))
    h = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    dA = torch.empty(r, K, dtype=torch.bfloat16, device=dev)
    dB = torch.empty(N, r, dtype=torch.bfloat16, device=dev)
    ws_f = torch.empty(q.fwd_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(int(q.lib.qlora_bwd_dropout_workspace_bytes(M, N, K, r)), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step():
        _, u = q.qlora_linear_fwd_dropout(qw, x, A, B, alpha, p, keep, h=h, workspace=ws_f)
        q.qlora_linear_bwd_dropout(qw, x, A, B, alpha, p, keep, dY, u=u, workspace=ws_b, outs=(dX, dA, dB))

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for s, e in ev:
        flush.zero_()
        s.record()
        step()
        e.record()
    torch.cuda.synchronize()
    ms = statistics.mean(s.elapsed_time(e) for s, e in ev)
    q.profiling(True)
    for _ in range(steps):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    q.profiling(False)
    prof = q.profile_read()
    f_fwd, f_bwd = layer_flops(M, N, K, r)
    add_n, add_t = prof.get("lora_dX_add", (0, 0.0))
    add_us = 1e3 * add_t / max(add_n, 1)
    add_bytes = M * K * 4 + M * K * 2 + M * K // 8
    del qw, x, A, B, dY, keep, h, dX, dA, dB, ws_f, ws_b, flush, inp
    torch.cuda.empty_cache()
    return {"workload": f"{MAIN}: W0 {N}x{K} NF4 double quant, x {M}x{K}, r={r}, LoRA dropout p={p}, "
                        f"fwd+bwd", "ms_per_step": ms, "tflops": (f_fwd + f_bwd) / (ms * 1e-3) / 1e12,
            "kernels_us": {k: 1e3 * t / max(n, 1) for k, (n, t) in prof.items()},
            "lora_dX_add": {"bytes": add_bytes, "kernel_us": add_us,
                            "gbs": add_bytes / (add_us * 1e-6) / 1e9 if add_us > 0 else None,
                            "frac": add_bytes / (add_us * 1e-6) / 1e9 / peaks["hbm_gbs"] if add_us > 0 else None}}


def block128_leg(q, dev, peaks, steps=50):
    """The main workload's fused forward + backward, the decode forward and the
    quantiser with 128-element blocks (the pages' other block size): the same
    kernels with two 64-element steps per scale."""
    from bit_nf4_quantized_05_b200 import dp
    w = workloads.WORKLOADS[MAIN]
    M, N, K, r, alpha = w.M, w.N, w.K, w.r, w.alpha
    inp = workloads.make_inputs(w)
    qw = q.nf4_quantize(inp["W0"].to(dev), double_quant=w.double_quant, block_size=128)
    x, A, B, dY = (inp[k].to(dev) for k in ("x", "A", "B", "dY"))
    h = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    u = torch.empty(M, r, dtype=torch.float32, device=dev)
    dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    flat, dA, dB = dp.grad_buffer(r, K, N, device=dev)
    ws_f = torch.empty(q.fwd_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(q.bwd_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step():
        q.qlora_linear_fwd(qw, x, A, B, alpha, h=h, u=u, workspace=ws_f)
        q.qlora_linear_bwd(qw, x, A, B, alpha, dY, u=u, workspace=ws_b, outs=(dX, dA, dB))

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for s, e in ev:
        flush.zero_()
        s.record()
        step()
        e.record()
    torch.cuda.synchronize()
    ms = statistics.mean(s.elapsed_time(e) for s, e in ev)
    f_fwd, f_bwd = layer_flops(M, N, K, r)
    del qw, x, A, B, dY, h, u, dX, ws_f, ws_b, flush, inp
    torch.cuda.empty_cache()
    return {"step": {"workload": f"{MAIN}: W0 {N}x{K} NF4 (blocks of 128, double quant), x {M}x{K}, "
                                 f"r={r}, fwd+bwd", "ms_per_step": ms,
                     "tflops": (f_fwd + f_bwd) / (ms * 1e-3) / 1e12},
            "decode": decode_leg(q, dev, peaks, block=128, tokens=(1, 16)),
            "quantize": quantize_leg(q, dev, peaks, block=128)}


def _time_steps(step, warmup, steps):
    """Mean device time (ms) of `steps` calls of step() after `warmup` untimed ones."""
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        step()
    e.record()
    torch.cuda.synchronize()
    return s.elapsed_time(e) / steps


def mlp70b_leg(q, dev, peaks, warmup=3, steps=5):
    """Forward + backward of the Llama-2-70B-like MLP projection (W0 28672x8192 NF4 with
    double quant, 8192 tokens, r = 64, alpha = 16). Every operand is larger than L2."""
    from bit_nf4_quantized_05_b200 import dp
    w = workloads.WORKLOADS[QUANT]
    M, N, K, r, alpha = w.M, w.N, w.K, w.r, w.alpha
    inp = workloads.make_inputs(w)
    qw = q.nf4_quantize(inp["W0"].to(dev), double_quant=True)
    x, A, B, dY = (inp[k].to(dev) for k in ("x", "A", "B", "dY"))
    del inp
    h = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    u = torch.empty(M, r, dtype=torch.float32, device=dev)
    dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    flat, dA, dB = dp.grad_buffer(r, K, N, device=dev)
    ws_f = torch.empty(q.fwd_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(q.bwd_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev)

    def step():
        q.qlora_linear_fwd(qw, x, A, B, alpha, h=h, u=u, workspace=ws_f)
        q.qlora_linear_bwd(qw, x, A, B, alpha, dY, u=u, workspace=ws_b, outs=(dX, dA, dB))

    ms = _time_steps(step, warmup, steps)
    q.profiling(True)
    for _ in range(steps):
        step()
    torch.cuda.synchronize()
    q.profiling(False)
    prof = q.profile_read()
    f, b = layer_flops(M, N, K, r)
    g_ms = sum(prof.get(k, (0, 0.0))[1] for k in ("qlora_gemm_fwd", "qlora_gemm_dgrad")) / steps
    g_flops = (2 * M * N * K + 2 * M * N * r) + (2 * M * N * K + 2 * M * K * r)
    del qw, x, A, B, dY, h, u, dX, flat, ws_f, ws_b
    torch.cuda.empty_cache()
    tflops = (f + b) / (ms * 1e-3) / 1e12
    gemm_tflops = g_flops / (g_ms * 1e-3) / 1e12 if g_ms > 0 else None
    return {"workload": f"{QUANT}: W0 {N}x{K} NF4 double quant, x {M}x{K} bf16, r={r}, "
                        f"alpha={alpha:g}, forward+backward",
            "ms_per_step": ms, "tflops": tflops, "frac": tflops / peaks["bf16_tflops"],
            "gemm_tflops": gemm_tflops,
            "gemm_frac": gemm_tflops / peaks["bf16_tflops"] if gemm_tflops else None,
            "peak_tflops": peaks["bf16_tflops"], "steps": steps,
            "kernel_avg_us": {k: 1e3 * t / max(n, 1) for k, (n, t) in prof.items()}}


def stack_leg(q, dev, peaks, warmup=2, steps=3):
    """The LLaMA-13B-like adapter stack: 40 layers x {Q, K, V, O}, each a 5120x5120 NF4
    weight with double quant and its own r = 16 adapters (weights and adapters drawn from the
    per-projection seeds), forward + backward of every projection at 4096 tokens. One batch
    of tokens and output gradients (drawn from the first projection's seed) serves every
    projection. The 160 weights (2.2 GB of codes and scales) far exceed L2."""
    from concurrent.futures import ThreadPoolExecutor
    from bit_nf4_quantized_05_b200 import dp
    w = workloads.WORKLOADS[STACK]
    M, N, K, r, alpha = w.M, w.N, w.K, w.r, w.alpha
    seeds = [workloads.stack_seed(l, p) for l in range(w.layers // 4) for p in range(4)]
    base = workloads.make_inputs(w, seed=seeds[0])
    x, dY = base["x"].to(dev), base["dY"].to(dev)
    del base
    t0 = time.perf_counter()
    projs = []

    def draw(seed):
        return workloads.make_inputs(w, M=0, seed=seed, with_dy=False)

    with ThreadPoolExecutor(max_workers=min(16, max(1, cpu_cores()))) as ex:
        for i in range(0, len(seeds), 16):
            for inp in ex.map(draw, seeds[i:i + 16]):
                qw = q.nf4_quantize(inp["W0"].to(dev), double_quant=True)
                projs.append((qw, inp["A"].to(dev), inp["B"].to(dev)))
    gen_s = time.perf_counter() - t0
    h = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    u = torch.empty(M, r, dtype=torch.float32, device=dev)
    dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    grads = [dp.grad_buffer(r, K, N, device=dev) for _ in projs]
    ws_f = torch.empty(q.fwd_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(q.bwd_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev)

    def step():
        for (qw, A, B), (_, dA, dB) in zip(projs, grads):
            q.qlora_linear_fwd(qw, x, A, B, alpha, h=h, u=u, workspace=ws_f)
            q.qlora_linear_bwd(qw, x, A, B, alpha, dY, u=u, workspace=ws_b, outs=(dX, dA, dB))

    ms = _time_steps(step, warmup, steps)
    f, b = layer_flops(M, N, K, r)
    total = len(projs) * (f + b)
    del projs, grads, x, dY, h, u, dX, ws_f, ws_b
    torch.cuda.empty_cache()
    tflops = total / (ms * 1e-3) / 1e12
    return {"workload": f"{STACK}: {w.layers} projections x (W0 {N}x{K} NF4 double quant, "
                        f"x {M}x{K} bf16, r={r}, alpha={alpha:g}), forward+backward each",
            "ms_per_step": ms, "tflops": tflops, "frac": tflops / peaks["bf16_tflops"],
            "peak_tflops": peaks["bf16_tflops"], "algorithmic_tflop": total / 1e12,
            "steps": steps, "input_generation_s": gen_s}


def cpu_baseline_leg(w, inp, target_s=12.0):
    """The oracle on a bounded sample of the workload's tokens: the sample grows
    (at most 8x per try) until one try takes half of target_s or covers every
    token, so the timed try takes roughly 5 to 20 s on the host."""
    tokens = 16
    qw = oracle_weight(w, inp)
    while True:
        f, t = oracle_sample_step(w, inp, tokens, qw)
        if t >= 0.5 * target_s or tokens >= w.M:
            break
        tokens = int(min(w.M, tokens * min(8.0, max(2.0, target_s / max(t, 1e-3)))))
    return {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
            "sample": f"{tokens} of {w.M} tokens: oracle forward+backward of those tokens "
                      f"({t:.1f} s on the host)"}


if __name__ == "__main__":
    main()
