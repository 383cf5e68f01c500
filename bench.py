#!/usr/bin/env python
"""Benchmark of the QLoRA linear layer (NF4 frozen weight + LoRA adapters) on B200.

One step = the layer's forward and backward on one batch of synthetic tokens,
i.e. h = x W~^T + (alpha/r)(x A^T)B^T, then dX, dA, dB (the adapter gradients
in fp32, all-reduced across ranks when N > 1). Headline workload: the
Llama-2-70B-like MLP projection (W0 28672x8192 NF4 with double quantisation,
8192 tokens per rank, r = 64, alpha = 16), the largest configuration that fits
one GPU. value = algorithmic fwd+bwd FLOP/s over all ranks.

Every rank also reports the end-to-end speed through the public API with host
buffers. At N = 1 the same run adds, as compact entries of "legs": the
LLaMA-13B-like attention projection's step (5120x5120, 2048 tokens), the
160-projection adapter stack, the decode-shaped forward (W0 13824x5120, M in
{1,4,16}) as GB/s of 4-bit weight codes, the full-weight quantisation of the
70B MLP weight, the adapter merge, the multi-adapter forward, the step with
128-element blocks, the steps with LoRA dropout (keep mask given, and drawn in
the kernels from a counter-based generator), and the CPU oracle's speed on a
bounded sample of the headline workload. Per-kernel details go to stderr as
one more JSON line.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                       [--skip-extras] [--leg NAME]
       (N > 1: launch under torch.distributed.run, one rank per GPU)
"""
import argparse
import json
import math
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
MAIN = "llama2_70b_mlp_28672x8192"
ATTN = "llama13b_attn_5120"
DECODE = "decode_mlp_up_13824x5120"
QUANT = "llama2_70b_mlp_28672x8192"
STACK = "llama13b_stack_40x4"
L2_FLUSH_BYTES = 512 << 20
# DRAM bytes (read + write) per launch of the fused GEMM, mean of the forward
# and dgrad launches, per workload, from one ncu capture of the kernels as they
# are now (summary and command under profiles/). None whenever the kernel has
# changed since that capture.
GEMM_TRAFFIC_BYTES = {MAIN: 2.774e9, ATTN: 3.98e7}


def layer_flops(M, N, K, r):
    """Algorithmic FLOPs of one forward and one backward of the layer."""
    fwd = 2 * M * N * K + 2 * M * r * (K + N)
    bwd = 2 * M * N * K + 4 * M * N * r + 4 * M * K * r
    return fwd, bwd


def gemm_flops(M, N, K, r):
    """Algorithmic FLOPs of the fused GEMM launches of one step: the forward
    (x W~^T plus the up-projection stage) and dgrad (dY W~ plus s v A)."""
    return (2 * M * N * K + 2 * M * N * r) + (2 * M * N * K + 2 * M * K * r)


def sig(v, n=4):
    """v rounded to n significant digits (compact JSON)."""
    if v is None or not isinstance(v, (int, float)) or v == 0 or not math.isfinite(v):
        return v
    return round(v, -int(math.floor(math.log10(abs(v)))) + n - 1)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def main_config(w, world):
    """The headline workload as the JSON line's config (both arms)."""
    return {"workload": f"{w.name}: W0 {w.N}x{w.K} NF4 (blocks of 64, double quant), "
                        f"x {w.M}x{w.K} bf16 per rank, r={w.r}, alpha={w.alpha:g}, fwd+bwd",
            "global_batch_tokens": w.M * world, "parallelism": f"dp{world}",
            "l2": "512 MiB buffer written before every timed step (outside the events); "
                  "every operand is larger than L2 as well"}


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
def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count()


class OracleSample:
    """The oracle on the headline workload, on a few tokens per step. The frozen
    weight is quantised and dequantised to its bf16 operand once, before any
    step (the GPU path quantises once too); a step is the oracle's full forward
    and backward of `tokens` tokens (h and dX rows, and their dA/dB terms)."""

    def __init__(self, w, tokens):
        import oracle
        self.w, self.tokens = w, tokens
        inp = workloads.make_inputs(w, M=tokens)
        qw = oracle.quantize(inp["W0"].numpy().reshape(-1), dq=w.double_quant)
        del inp["W0"]
        self.Wt = oracle.dequant_operand(qw, w.N, w.K)
        bits = workloads.bf16_bits
        self.x, self.A, self.B, self.dY = (bits(inp[k]) for k in ("x", "A", "B", "dY"))
        f, b = layer_flops(tokens, w.N, w.K, w.r)
        self.flops = f + b

    def step(self):
        """One step; returns its seconds."""
        import oracle
        w = self.w
        t0 = time.perf_counter()
        oracle.qlora_fwd_rows_op(self.Wt, self.x, self.A, self.B, w.r, w.alpha)
        oracle.qlora_bwd_op(self.Wt, self.x, self.A, self.B, w.r, w.alpha, self.dY)
        return time.perf_counter() - t0

    def describe(self):
        return (f"{self.tokens} of the {self.w.M} tokens per step: the oracle's forward and "
                f"backward of those tokens (h and dX rows, dA and dB over them), the weight "
                f"quantised and dequantised to its bf16 operand once before the steps")


def sample_tokens():
    """Tokens per oracle step: about one per host core (its rows run in parallel)."""
    return int(min(64, max(8, cpu_cores())))


def run_reference(args, rank, world):
    """The oracle as it stands, timed on the host cores (rank 0 only)."""
    if rank != 0:
        return
    w = workloads.WORKLOADS[MAIN]
    smp = OracleSample(w, sample_tokens())
    for _ in range(args.warmup):
        smp.step()
    tot_t = 0.0
    for _ in range(args.steps):
        tot_t += smp.step()
    value = smp.flops * args.steps / tot_t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": main_config(w, world),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                         "sample": smp.describe()},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def cpu_baseline_leg(target_s=12.0):
    """The oracle on the headline workload, timed like the reference arm: steps of
    sample_tokens() tokens until about target_s seconds of steps have run."""
    w = workloads.WORKLOADS[MAIN]
    smp = OracleSample(w, sample_tokens())
    smp.step()                                   # warm-up
    n, t = 0, 0.0
    while n < 2 or t < target_s:
        t += smp.step()
        n += 1
    return {"value": smp.flops * n / t / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(),
            "kind": "oracle", "sample": f"{n} steps ({t:.1f} s); " + smp.describe()}


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------
class LayerRun:
    """One workload's layer on the device: quantised weight, inputs, outputs,
    workspaces and the flat fp32 adapter-gradient buffer."""

    def __init__(self, q, dp, w, dev, block=64):
        self.q, self.dp, self.w = q, dp, w
        inp = workloads.make_inputs(w)
        self.qw = q.nf4_quantize(inp.pop("W0").to(dev), double_quant=w.double_quant, block_size=block)
        self.x, self.A, self.B, self.dY = (inp[k].to(dev) for k in ("x", "A", "B", "dY"))
        self.inp = inp
        M, N, K, r = w.M, w.N, w.K, w.r
        self.h = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        self.u = torch.empty(M, r, dtype=torch.float32, device=dev)
        self.dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
        self.flat, self.dA, self.dB = dp.grad_buffer(r, K, N, device=dev)
        self.ws_f = torch.empty(q.fwd_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev)
        self.ws_b = torch.empty(q.bwd_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev)

    def step(self, world=1):
        q, w = self.q, self.w
        q.qlora_linear_fwd(self.qw, self.x, self.A, self.B, w.alpha, h=self.h, u=self.u, workspace=self.ws_f)
        q.qlora_linear_bwd(self.qw, self.x, self.A, self.B, w.alpha, self.dY, u=self.u,
                           workspace=self.ws_b, outs=(self.dX, self.dA, self.dB))
        self.dp.allreduce_adapter_grads(self.flat, world)


def event_steps(step, steps, flush):
    """Per-step device times (ms): `steps` steps, each bracketed by its own two
    events, the L2 flush between them outside the events."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for s, e in ev:
        flush.zero_()
        s.record()
        step()
        e.record()
    torch.cuda.synchronize()
    return [s.elapsed_time(e) for s, e in ev]


def profiled_steps(q, step, steps, flush):
    """The same steps with the library's per-launch events: {kind: (launches, ms)}."""
    q.profiling(True)
    for _ in range(steps):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    q.profiling(False)
    return q.profile_read()


def gemm_roofline(prof, w, steps, peaks, sustained):
    """Roofline of the fused GEMM (forward and dgrad launches of `steps` steps).
    peak: the measured dense bf16 rate, sustained (a kernel timed inside a long
    run of steps, where the power cap holds the clock down) or burst."""
    g_launch = sum(prof.get(k, (0, 0.0))[0] for k in ("qlora_gemm_fwd", "qlora_gemm_dgrad"))
    g_ms = sum(prof.get(k, (0, 0.0))[1] for k in ("qlora_gemm_fwd", "qlora_gemm_dgrad"))
    g_tflops = steps * gemm_flops(w.M, w.N, w.K, w.r) / (g_ms * 1e-3) / 1e12 if g_ms > 0 else None
    use_sus = sustained and peaks.get("bf16_tflops_sustained")
    peak = peaks["bf16_tflops_sustained"] if use_sus else peaks["bf16_tflops"]
    out = {"bound": "tensor", "achieved": g_tflops, "peak": peak, "unit": "TFLOP/s",
           "frac": (g_tflops / peak) if g_tflops else None,
           "traffic": GEMM_TRAFFIC_BYTES.get(w.name),
           "kernel": "qlora_gemm_pair_kernel (forward and dgrad launches)",
           "peak_source": peaks["source"] + (" bf16 sustained" if use_sus else " bf16 burst"),
           "avg_launch_us": 1e3 * g_ms / max(g_launch, 1)}
    if use_sus:
        out["frac_of_burst"] = g_tflops / peaks["bf16_tflops"] if g_tflops else None
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--skip-extras", action="store_true",
                    help="only the headline fwd+bwd line (no legs, no end-to-end, no oracle)")
    ap.add_argument("--leg", default="all",
                    choices=["all", "attn5120", "decode", "quantize", "stack", "merge", "multi",
                             "block128", "dropout", "dropout_philox", "cpu"],
                    help="run one leg alone and print its JSON (for profiling)")
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
    peaks = load_peaks()
    if args.leg != "all":
        if rank == 0:
            print(json.dumps({"leg": args.leg, **run_leg(args.leg, q, dp, dev, peaks)}), flush=True)
        return
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    w = workloads.WORKLOADS[MAIN]
    M, N, K, r = w.M, w.N, w.K, w.r
    run = LayerRun(q, dp, w, dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step():
        run.step(world)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = q.device_status(dev)
    if st != q.NF4_OK:
        raise RuntimeError(f"device status after warm-up: {q.status_string(st)}")

    barrier()
    torch.cuda.synchronize()
    # Timed region: K steps with only the two step events each (per-launch
    # events would sit between the kernels and stop each launch from
    # overlapping the tail of the one before).
    with ClockSampler(local_rank) as clk:
        per_step = event_steps(step, args.steps, flush)
    barrier()
    # Kernel durations: the same K steps again with the library's per-launch
    # CUDA events (recorded on the stream each kernel is launched on).
    prof = profiled_steps(q, step, args.steps, flush)
    barrier()
    ms = statistics.mean(per_step)
    if world > 1:
        t = torch.tensor([ms], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = float(t.item())
    f_fwd, f_bwd = layer_flops(M, N, K, r)
    value = world * (f_fwd + f_bwd) / (ms * 1e-3) / 1e12
    # the GEMM runs inside back-to-back steps of several milliseconds each, long
    # enough for the 1 kW power cap to set the clock: the sustained peak applies
    roofline = gemm_roofline(prof, w, args.steps, peaks, sustained=True)
    gpu_launches = sum(n for n, _ in prof.values())
    kernels = {k: {"launches": n, "avg_us": 1e3 * t / max(n, 1)} for k, (n, t) in prof.items()}

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; shapes and distributions of the pages' workloads)",
        "config": main_config(w, world),
        "roofline": {k: sig(v) for k, v in roofline.items()},
        "gpu_launches": gpu_launches,
        "clocks": clk.summary(),
    }
    detail = {"main_kernels_us": kernels}

    if not args.skip_extras:
        # every rank takes the same collective steps in the end-to-end leg
        e2e = e2e_leg(q, dp, run, args, dev, world)
        if rank == 0:
            line["e2e"] = {k: sig(v) for k, v in e2e.items()}
    del run, flush
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.skip_extras:
        # single-GPU legs: at N > 1 the other ranks would wait in the closing
        # barrier for minutes, beyond the process group's timeout
        legs = {}
        for name in ("attn5120", "stack", "decode", "quantize", "dropout", "dropout_philox",
                     "block128", "merge", "multi"):
            res = run_leg(name, q, dp, dev, peaks)
            detail[name] = res
            legs[name] = compact_leg(name, res)
        line["legs"] = legs
        line["cpu_baseline"] = cpu_baseline_leg()
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps({"detail": detail}), file=sys.stderr, flush=True)
        print(json.dumps(line), flush=True)


def run_leg(name, q, dp, dev, peaks):
    if name == "cpu":
        return cpu_baseline_leg()
    fn = {"attn5120": attn_leg, "decode": decode_leg, "quantize": quantize_leg, "stack": stack_leg,
          "merge": merge_leg, "multi": multi_leg, "block128": block128_leg, "dropout": dropout_leg,
          "dropout_philox": dropout_philox_leg}[name]
    out = fn(q, dev, peaks)
    torch.cuda.synchronize()
    st = q.device_status(dev)
    if st != q.NF4_OK:
        raise RuntimeError(f"device status after the {name} leg: {q.status_string(st)}")
    return out


def compact_leg(name, res):
    """The few figures of a leg that go on the JSON line."""
    if name == "decode":
        return {m: {"us": sig(v["graph_call_us"]), "gbs": sig(v["gbs_graph_call"]),
                    "frac": sig(v["frac_graph_call"], 3)}
                for m, v in res.items() if m.startswith("M")}
    if name == "quantize":
        return {"us": sig(res["kernel_us"]), "gbs": sig(res["gbs"]), "frac": sig(res["frac"], 3),
                "bf16_in_us": sig(res["bf16_input"]["kernel_us"])}
    if name in ("attn5120", "stack"):
        return {k: sig(res[k], 4 if k != "frac" and k != "gemm_frac" else 3)
                for k in ("ms_per_step", "tflops", "frac", "gemm_frac") if k in res}
    if name in ("dropout", "dropout_philox"):
        return {"ms_per_step": sig(res["ms_per_step"]), "tflops": sig(res["tflops"])}
    if name == "block128":
        return {"step_ms": sig(res["step"]["ms_per_step"]),
                "decode_M1_us": sig(res["decode"]["M1"]["graph_call_us"]),
                "quantize_us": sig(res["quantize"]["kernel_us"])}
    if name == "merge":
        return {"bf16_frac": sig(res["bf16"]["frac"], 3), "fp32_frac": sig(res["fp32"]["frac"], 3)}
    if name == "multi":
        return {"us": sig(res["graph_call_us"]), "frac": sig(res["frac_graph_call"], 3)}
    return {}


def attn_leg(q, dev, peaks, warmup=3, steps=50):
    """The LLaMA-13B-like attention projection's fwd+bwd step (W0 5120x5120 NF4 with
    double quant, 2048 tokens, r = 16, alpha = 32), timed like the headline step."""
    from bit_nf4_quantized_05_b200 import dp
    w = workloads.WORKLOADS[ATTN]
    run = LayerRun(q, dp, w, dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(warmup):
        run.step()
    torch.cuda.synchronize()
    ms = statistics.mean(event_steps(run.step, steps, flush))
    prof = profiled_steps(q, run.step, steps, flush)
    f, b = layer_flops(w.M, w.N, w.K, w.r)
    roof = gemm_roofline(prof, w, steps, peaks, sustained=False)
    del run, flush
    torch.cuda.empty_cache()
    tflops = (f + b) / (ms * 1e-3) / 1e12
    return {"workload": f"{w.name}: W0 {w.N}x{w.K} NF4 double quant, x {w.M}x{w.K} bf16, r={w.r}, "
                        f"alpha={w.alpha:g}, forward+backward",
            "ms_per_step": ms, "tflops": tflops, "frac": tflops / peaks["bf16_tflops"],
            "gemm_tflops": roof["achieved"], "gemm_frac": roof["frac"], "gemm_traffic": roof["traffic"],
            "kernel_avg_us": {k: 1e3 * t / max(n, 1) for k, (n, t) in prof.items()}}


def e2e_leg(q, dp, run, args, dev, world):
    """Same metric through the public API with host buffers: every step copies
    x and dY in from pinned host memory and h, dX and the fp32 adapter
    gradients back out (the frozen weight and the adapters stay resident).
    The copies run as a training input pipeline would: two sets of device
    buffers, step i + 1's inputs copied in on one copy stream while step i
    computes, step i's outputs copied out on another (the other direction of
    the host link). Every step's copies are inside the timed region."""
    w = run.w
    M, N, K, r, alpha = w.M, w.N, w.K, w.r, w.alpha
    hx = run.inp["x"].pin_memory()
    hdY = run.inp["dY"].pin_memory()
    oh = [torch.empty(M, N, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    odX = [torch.empty(M, K, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    ograd = [torch.empty(r * K + N * r, dtype=torch.float32).pin_memory() for _ in range(2)]
    qw, A, B = run.qw, run.A, run.B
    xs = [torch.empty(M, K, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    dYs = [torch.empty(M, N, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    hs = [torch.empty(M, N, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    dXs = [torch.empty(M, K, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    grads = [dp.grad_buffer(r, K, N, device=dev) for _ in range(2)]
    main = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]     # set k's inputs landed
    ev_used = [torch.cuda.Event() for _ in range(2)]   # the step on set k has computed
    ev_out = [torch.cuda.Event() for _ in range(2)]    # set k's outputs copied out
    for k in range(2):
        ev_used[k].record(main)
        ev_out[k].record(main)

    def copy_in(i):
        k = i % 2
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_used[k])                # the step two back is done with set k
            xs[k].copy_(hx, non_blocking=True)
            dYs[k].copy_(hdY, non_blocking=True)
            ev_in[k].record(s_in)

    def compute(i):
        k = i % 2
        main.wait_event(ev_in[k])
        main.wait_event(ev_out[k])                     # set k's previous outputs are out
        flat, dA, dB = grads[k]
        _, u = q.qlora_linear_fwd(qw, xs[k], A, B, alpha, h=hs[k])
        q.qlora_linear_bwd(qw, xs[k], A, B, alpha, dYs[k], u=u, outs=(dXs[k], dA, dB))
        dp.allreduce_adapter_grads(flat, world)
        ev_used[k].record(main)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_used[k])
            oh[k].copy_(hs[k], non_blocking=True)
            odX[k].copy_(dXs[k], non_blocking=True)
            ograd[k].copy_(flat, non_blocking=True)
            ev_out[k].record(s_out)

    def run_steps(n):
        copy_in(0)
        for i in range(n):
            if i + 1 < n:
                copy_in(i + 1)
            compute(i)
        main.wait_stream(s_out)

    steps = max(5, min(args.steps, 20))
    run_steps(3)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(main)
    s_in.wait_stream(main)
    run_steps(steps)
    e.record(main)
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    if world > 1:
        t = torch.tensor([ms], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = float(t.item())
    f, b = layer_flops(M, N, K, r)
    nbytes_in, nbytes_out = hx.nbytes + hdY.nbytes, oh[0].nbytes + odX[0].nbytes + ograd[0].nbytes
    del xs, dYs, hs, dXs, grads
    torch.cuda.empty_cache()
    return {"value": world * (f + b) / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "ms_per_step": ms, "h2d_bytes_per_step": nbytes_in, "d2h_bytes_per_step": nbytes_out}


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
    w = workloads.WORKLOADS[ATTN]
    inp = workloads.make_inputs(w, M=0, with_dy=False)
    W0 = inp["W0"].to(dev)
    copies = [q.nf4_quantize(W0, double_quant=True) for _ in range(4)]
    del W0
    A, B = inp["A"].to(dev), inp["B"].to(dev)
    nb = w.N * w.K // 64
    out = {"workload": f"{ATTN}: W0 {w.N}x{w.K} NF4 double quant, r={w.r}, alpha={w.alpha:g}",
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
    w = workloads.WORKLOADS[ATTN]
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
    return {"workload": f"{ATTN}: W0 {N}x{K} NF4 double quant, x {M}x{K}, r={r}, LoRA dropout p={p}, "
                        f"fwd+bwd", "ms_per_step": ms, "tflops": (f_fwd + f_bwd) / (ms * 1e-3) / 1e12,
            "kernels_us": {k: 1e3 * t / max(n, 1) for k, (n, t) in prof.items()},
            "lora_dX_add": {"bytes": add_bytes, "kernel_us": add_us,
                            "gbs": add_bytes / (add_us * 1e-6) / 1e9 if add_us > 0 else None,
                            "frac": add_bytes / (add_us * 1e-6) / 1e9 / peaks["hbm_gbs"] if add_us > 0 else None}}


def dropout_philox_leg(q, dev, peaks, steps=50, p=0.05):
    """The main workload's forward + backward with LoRA dropout p = 0.05 whose mask the
    kernels draw from Philox4x32-10 (a new offset every step; the backward regenerates the
    forward's mask, nothing is stored): the rank-r kernels draw and apply the mask to the
    landed x tiles, the dgrad GEMM writes dY W~ in fp32 and the adapter-add kernel draws,
    masks, adds and rounds dX once."""
    w = workloads.WORKLOADS[ATTN]
    M, N, K, r, alpha = w.M, w.N, w.K, w.r, w.alpha
    inp = workloads.make_inputs(w)
    qw = q.nf4_quantize(inp["W0"].to(dev), double_quant=w.double_quant)
    x, A, B, dY = (inp[k].to(dev) for k in ("x", "A", "B", "dY"))
    h = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    dA = torch.empty(r, K, dtype=torch.bfloat16, device=dev)
    dB = torch.empty(N, r, dtype=torch.bfloat16, device=dev)
    ws_f = torch.empty(q.fwd_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(int(q.lib.qlora_bwd_dropout_workspace_bytes(M, N, K, r)), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    seed, offset = 20241202, [0]

    def step():
        offset[0] += 1
        _, u = q.qlora_linear_fwd_dropout_philox(qw, x, A, B, alpha, p, seed, offset[0], h=h, workspace=ws_f)
        q.qlora_linear_bwd_dropout_philox(qw, x, A, B, alpha, p, seed, offset[0], dY, u=u, workspace=ws_b,
                                          outs=(dX, dA, dB))

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    ms = statistics.mean(event_steps(step, steps, flush))
    prof = profiled_steps(q, step, steps, flush)
    f_fwd, f_bwd = layer_flops(M, N, K, r)
    del qw, x, A, B, dY, h, dX, dA, dB, ws_f, ws_b, flush, inp
    torch.cuda.empty_cache()
    return {"workload": f"{ATTN}: W0 {N}x{K} NF4 double quant, x {M}x{K}, r={r}, LoRA dropout p={p} "
                        f"drawn in the kernels (Philox4x32-10), fwd+bwd",
            "ms_per_step": ms, "tflops": (f_fwd + f_bwd) / (ms * 1e-3) / 1e12,
            "kernels_us": {k: 1e3 * t / max(n, 1) for k, (n, t) in prof.items()}}


def block128_leg(q, dev, peaks, steps=50):
    """The main workload's fused forward + backward, the decode forward and the
    quantiser with 128-element blocks (the pages' other block size): the same
    kernels with two 64-element steps per scale."""
    from bit_nf4_quantized_05_b200 import dp
    w = workloads.WORKLOADS[ATTN]
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
    return {"step": {"workload": f"{ATTN}: W0 {N}x{K} NF4 (blocks of 128, double quant), x {M}x{K}, "
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


if __name__ == "__main__":
    main()
