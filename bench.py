#!/usr/bin/env python
"""Benchmark of the 4-bit routed-MoE layer forward on B200.

One step is one forward of a Qwen3-30B-A3B-shaped NF4 MoE layer (E=128,
H=2048, I=768, top-8) on a decode batch of T=64 tokens: routing, expert
permute and gather, the grouped gate_up GEMM with in-kernel NF4 dequant and
SwiGLU, the grouped down GEMM and the weighted combine.  Weights are seeded
synthetic N(0, 0.02) values NF4-quantised on the device by the library's
quantiser; activations and router logits are seeded N(0, 1) in bf16.

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle on
the same workload instead (one token per step).  Under torchrun every rank
runs an independent replica of the layer (the forward has no exchange step):
``value`` is the whole-job token rate, timed on the device and taken as the
max over ranks.
"""
import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "4-bit MoE layer tokens/s; decode weight GB/s vs HBM peak; prefill TFLOP/s"
WORKLOAD = "qwen3_30b_a3b_nf4_decode"
T_HEADLINE = 64
L2_BYTES = 126 * 1000 * 1000
KERNELS_PER_STEP = 5      # route (top-k + rank, one block at T<=128), gather, gate_up GEMM, down GEMM, combine
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_digest(name):
    """Digest of one kernel source: a recorded traffic figure is void once its kernel's source changes."""
    h = hashlib.sha256()
    with open(os.path.join(ROOT, "bit_mixture_experts_top_b200", "csrc", name), "rb") as f:
        h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_tag, workload, source):
    """DRAM bytes per launch of the kernel from the committed ncu summary, if it still matches the kernel's
    source file and was taken on this workload."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel_tag)
    if not e or e.get("source") != source or e.get("source_digest") != source_digest(source) \
            or not e.get("workload", "").startswith(workload + " "):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler(threading.Thread):
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle",
               0x2: "applications_clocks_setting"}

    def __init__(self, gpu_index, period_s=0.0002):
        super().__init__(daemon=True)
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period, self.stop_evt, self.err = period_s, threading.Event(), None
        self.first = threading.Event()          # set once the first sample is in (or sampling is impossible)
        self.switch, self.pre = None, 0
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(gpu_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:          # no NVML: report the gap instead of guessing
            self.nv, self.err = None, f"nvml unavailable: {e}"

    def _reasons(self):
        try:
            return self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            return self.nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)

    def run(self):
        if self.nv is None:
            self.first.set()
            return
        while not self.stop_evt.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                bits = self._reasons()
                for b, name in self.REASONS.items():
                    if bits & b and b not in (0x1,):
                        self.reasons.add(name)
            except Exception as e:
                self.err = str(e)
            self.first.set()
            time.sleep(self.period)

    def start(self):
        """Starts sampling and returns once the first sample is in; while it runs the interpreter
        switches threads every 0.2 ms, so a short timed region (whose host thread only enqueues
        graph replays and then waits) still gets several samples."""
        self.switch = sys.getswitchinterval()
        sys.setswitchinterval(2e-4)
        super().start()
        self.first.wait(timeout=1.0)
        self.pre = len(self.samples)            # taken before the region: kept only if nothing follows

    def summary(self):
        self.stop_evt.set()
        self.join(timeout=2)
        if self.switch is not None:
            sys.setswitchinterval(self.switch)
            self.switch = None
        if len(self.samples) > self.pre:
            self.samples = self.samples[self.pre:]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples),
                **({"note": self.err} if self.err else {})}


# every layer configuration the metric is quoted on (the tiny layer is a correctness case only)
CONFIGS = [("qwen3_30b_a3b_nf4_decode", 1), ("qwen3_30b_a3b_nf4_decode", 8), ("qwen3_30b_a3b_nf4_decode", 32),
           ("qwen3_30b_a3b_nf4_decode", 64), ("qwen3_30b_a3b_nf4_lora", 512), ("gptoss_20b_mxfp4", 1),
           ("gptoss_20b_mxfp4", 16), ("gptoss_20b_mxfp4", 4096), ("gptoss_120b_mxfp4_zipf", 16384)]
ROTATE_BYTES = 4 * L2_BYTES      # decode layers rotate over weight copies until this much is touched per pass
MAX_COPIES = 24


def bench_configs(dev, peaks, max_over_ranks, target_s=0.4, only=None):
    """Every configuration of CONFIGS, timed as CUDA-graph replays of the whole forward.

    Decode-sized layers touch less than L2 holds, so one pass replays the layer over several copies of its
    packed stacks (identical bytes at distinct addresses, like consecutive layers of a model) until a pass
    touches ROTATE_BYTES; the time per layer is the pass time over the copies.  The gate_up and down
    launches are timed the same way on their own.  Decode-class layers report weight-stream GB/s against
    the HBM peak, prefill-class ones TFLOP/s (real routed rows only) against the bf16 burst peak."""
    import torch
    from bit_mixture_experts_top_b200 import e4b, layer
    from bit_mixture_experts_top_b200.workloads import WORKLOADS

    rows, built = [], {}
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    for wname, T in CONFIGS:
        if only and f"{wname}:{T}" not in only:
            continue
        w = WORKLOADS[wname]
        key = (w.fmt, w.E, w.H, w.I, w.k, w.exp_range, w.weight_std, w.seed)
        if key not in built:
            built.clear()
            torch.cuda.empty_cache()
            built[key] = layer.synthetic_layer(w, dev)
        base = built[key]
        A, B = layer.synthetic_lora(w, dev)
        lay = layer.MoeLayer(w.E, w.H, w.I, w.k, w.fmt, base.gate_up, base.down, A, B, w.lora_scale)
        x_np, lg_np = layer.synthetic_tokens(w, T)
        x, lg = layer.bits_tensor(x_np, dev), layer.bits_tensor(lg_np, dev)
        out = torch.empty((T, w.H), dtype=torch.bfloat16, device=dev)
        ws = lay.workspace(T, dev)
        lay.forward(x, lg, out)
        torch.cuda.synchronize()
        offs = lay.region(T, e4b.E4B_WS_EXPERT_OFFSETS, torch.int32).cpu().numpy()
        touched = int(np.count_nonzero(np.diff(offs)))
        R = T * w.k
        wbytes = touched * (w.gate_up_bytes_per_expert() + w.down_bytes_per_expert())
        lora_bytes = touched * (w.H + 2 * w.I) * w.lora_rank * 2
        gu_bytes = touched * w.gate_up_bytes_per_expert() + R * w.H * 2 + R * w.I * 2 + lora_bytes
        dn_bytes = touched * w.down_bytes_per_expert() + R * w.I * 2 + R * w.H * 4
        gu_flops = 2 * R * w.H * 2 * w.I + (2 * R * (w.H + 2 * w.I) * w.lora_rank if w.lora_rank else 0)
        dn_flops = 2 * R * w.I * w.H
        tensor = gu_flops / gu_bytes > ridge
        copies = 1 if wbytes >= ROTATE_BYTES else min(MAX_COPIES, -(-ROTATE_BYTES // max(wbytes, 1)))
        layers = [lay]
        for _ in range(copies - 1):
            gu = layer.PackedStack(lay.gate_up.codes.clone(), lay.gate_up.scales.clone(), w.E, 2 * w.I, w.H, w.fmt)
            dn = layer.PackedStack(lay.down.codes.clone(), lay.down.scales.clone(), w.E, w.H, w.I, w.fmt)
            layers.append(layer.MoeLayer(w.E, w.H, w.I, w.k, w.fmt, gu, dn, A, B, w.lora_scale))

        def args_of(l):
            return (l.desc, T, x, lg, l.gate_up.codes, l.gate_up.scales, l.down.codes, l.down.scales, l.lora_A,
                    l.lora_B, l.gu_bias, l.dn_bias, out, ws)

        def graph_of(fn):
            side = torch.cuda.Stream(device=dev)
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                fn()
            torch.cuda.current_stream().wait_stream(side)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn()
            return g

        g_fwd = graph_of(lambda: [e4b.e4b_moe_forward(*args_of(l)) for l in layers])
        g_gu = graph_of(lambda: [e4b.e4b_moe_forward_stage(e4b.E4B_STAGE_GATE_UP, *args_of(l)) for l in layers])
        g_dn = graph_of(lambda: [e4b.e4b_moe_forward_stage(e4b.E4B_STAGE_DOWN, *args_of(l)) for l in layers])

        def per_layer_ms(g, n=None, sampler=None):
            for _ in range(3):
                g.replay()
            torch.cuda.synchronize()
            if n is None:
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                g.replay()
                e1.record()
                torch.cuda.synchronize()
                n = int(min(2000, max(5, target_s * 1e3 / max(e0.elapsed_time(e1), 1e-3))))
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            if sampler:
                sampler.start()
            e0.record()
            for _ in range(n):
                g.replay()
            e1.record()
            torch.cuda.synchronize()
            clk = sampler.summary() if sampler else None
            return max_over_ranks(e0.elapsed_time(e1) / (n * len(layers))), n, clk

        # tensor-bound layers: a short window (a few tens of ms, kernels timed alone: burst peak) first,
        # then the long window's rate against the sustained peak (the power cap engages within it)
        if tensor:
            est, _, _ = per_layer_ms(g_fwd, 3)
            n = int(min(2000, max(3, 30.0 / max(est * len(layers), 1e-3))))
            ms, n, clk = per_layer_ms(g_fwd, n, sampler=ClockSampler(physical_gpu_index(dev.index or 0)))
        else:
            ms, n, clk = per_layer_ms(g_fwd, sampler=ClockSampler(physical_gpu_index(dev.index or 0)))
        gu_ms, _, _ = per_layer_ms(g_gu, n)
        dn_ms, _, _ = per_layer_ms(g_dn, n)
        sustained = None
        if tensor:
            ns = int(min(2000, max(5, target_s * 1e3 / max(ms * len(layers), 1e-3))))
            ms_s, _, clk_s = per_layer_ms(g_fwd, ns, sampler=ClockSampler(physical_gpu_index(dev.index or 0)))
            sustained = {"ms_per_step": ms_s, "layer_tflops": w.flops(T) / (ms_s * 1e-3) / 1e12,
                         "window_s": ns * ms_s * len(layers) * 1e-3, "clocks": clk_s}
            sustained["layer_frac_of_sustained_peak"] = sustained["layer_tflops"] / peaks["bf16_tflops_sustained"]
        if e4b.e4b_device_status(ws) != e4b.E4B_OK:
            raise RuntimeError(f"device status reported an error in config {wname} T={T}")
        active = max(min(R, w.E), 1)
        avg = (R + active - 1) // active
        rec = {"workload": wname, "T": T, "ms_per_step": ms, "tokens_per_s": T / (ms * 1e-3),
               "bound": "tensor" if tensor else "hbm", "touched_experts": touched,
               "kernel": "decode kernel (warp-level MMA)" if avg <= 12 else "tcgen05 tiles",
               "timing": f"{n} graph replays of {len(layers)} layer cop{'y' if len(layers) == 1 else 'ies'} "
                         f"(distinct weight addresses, {wbytes * len(layers) / 1e6:.0f} MB touched per replay)"
                         + (f", a {n * ms * len(layers):.0f} ms window against the burst peak" if tensor else ""),
               "clocks": clk}
        if sustained:
            rec["sustained"] = sustained
        if tensor:
            rec["gate_up"] = {"ms": gu_ms, "flops": gu_flops, "tflops": gu_flops / (gu_ms * 1e-3) / 1e12}
            rec["down"] = {"ms": dn_ms, "flops": dn_flops, "tflops": dn_flops / (dn_ms * 1e-3) / 1e12}
            rec["layer_tflops"] = w.flops(T) / (ms * 1e-3) / 1e12
            for kk in ("gate_up", "down"):
                rec[kk]["frac"] = rec[kk]["tflops"] / peaks["bf16_tflops"]
            rec["layer_frac"] = rec["layer_tflops"] / peaks["bf16_tflops"]
        else:
            rec["gate_up"] = {"ms": gu_ms, "bytes": gu_bytes, "gbs": gu_bytes / (gu_ms * 1e-3) / 1e9}
            rec["down"] = {"ms": dn_ms, "bytes": dn_bytes, "gbs": dn_bytes / (dn_ms * 1e-3) / 1e9}
            rec["layer_weight_gbs"] = wbytes / (ms * 1e-3) / 1e9
            for kk in ("gate_up", "down"):
                rec[kk]["frac"] = rec[kk]["gbs"] / peaks["hbm_gbs"]
            rec["layer_frac"] = rec["layer_weight_gbs"] / peaks["hbm_gbs"]
            rec["layer_tflops"] = w.flops(T) / (ms * 1e-3) / 1e12
        if w.lora_rank:
            rec["training"] = bench_training(lay, layers, w, T, x, lg, wbytes, peaks, max_over_ranks, target_s)
        rows.append(rec)
        del g_fwd, g_gu, g_dn, layers, lay, ws
        torch.cuda.synchronize()
    built.clear()
    torch.cuda.empty_cache()
    return rows


def bench_training(lay, layers, w, T, x, lg, wbytes, peaks, max_over_ranks, target_s):
    """A QLoRA training step on the layer (the forward that keeps what the backward needs, then the backward:
    LoRA factor gradients and dgrad through both frozen stacks), timed as CUDA-graph replays over the same
    weight copies as the forward; the backward streams every touched expert's packed weights once more."""
    import torch
    from bit_mixture_experts_top_b200 import e4b, synth, layer as lmod
    dev = x.device
    ws = lay.train_workspace(T, dev)
    out = torch.empty((T, w.H), dtype=torch.bfloat16, device=dev)
    dout = lmod.bits_tensor(synth.normal_bf16((T, w.H), 1.0, w.seed, f"dout{T}"), dev)
    r = w.lora_rank
    dx = torch.empty((T, w.H), dtype=torch.float32, device=dev)
    dl = torch.empty((T, w.E), dtype=torch.float32, device=dev)
    dA = torch.empty((w.E, w.H, r), dtype=torch.float32, device=dev)
    dB = torch.empty((w.E, r, 2 * w.I), dtype=torch.float32, device=dev)

    def fwd(l):
        e4b.e4b_moe_forward_train(l.desc, T, x, lg, l.gate_up.codes, l.gate_up.scales, l.down.codes, l.down.scales,
                                  l.lora_A, l.lora_B, None, None, out, ws)

    def bwd(l):
        e4b.e4b_moe_backward(l.desc, T, lg, dout, l.gate_up.codes, l.gate_up.scales, l.down.codes, l.down.scales,
                             l.lora_A, l.lora_B, dx, dl, dA, dB, ws)

    def graph_of(fn):
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            fn()
        torch.cuda.current_stream().wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        return g

    g_step = graph_of(lambda: [(fwd(l), bwd(l)) for l in layers])
    g_bwd = graph_of(lambda: [bwd(l) for l in layers])

    def per_layer_ms(g):
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        n = int(min(500, max(5, target_s * 1e3 / max(e0.elapsed_time(e1), 1e-3))))
        e0.record()
        for _ in range(n):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        return max_over_ranks(e0.elapsed_time(e1) / (n * len(layers)))

    step_ms = per_layer_ms(g_step)
    bwd_ms = per_layer_ms(g_bwd)
    if e4b.e4b_device_status(ws) != e4b.E4B_OK:
        raise RuntimeError("device status reported an error in the training step")
    del g_step, g_bwd
    gbs = wbytes / (bwd_ms * 1e-3) / 1e9
    return {"step_ms": step_ms, "tokens_per_s": T / (step_ms * 1e-3), "backward_ms": bwd_ms,
            "backward_weight_gbs": gbs, "backward_frac_of_hbm": gbs / peaks["hbm_gbs"],
            "note": "forward keeping G + backward (dx, dlogits, dA, dB); weight bytes = touched experts' packed "
                    "stacks, streamed once by the backward's two dgrad launches"}


def init_dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def physical_gpu_index(local):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local < len(ids) and ids[local].isdigit():
            return int(ids[local])
    return local


def oracle_tokens_per_s(w, x, logits, rows, reps=1):
    """Times the CPU oracle's forward on `rows` tokens (test infrastructure, baseline only)."""
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from helpers import oracle_lora, oracle_stacks, touched_experts
    from oracle import moe as omoe
    experts = touched_experts(logits[rows], w.k)
    stacks = oracle_stacks(w, experts)
    A, B = oracle_lora(w)
    t0 = time.perf_counter()
    for _ in range(reps):
        omoe.moe_forward(x[rows], logits[rows], w.k, w.fmt, w.E, w.H, w.I, *stacks, lora_A_bits=A, lora_B_bits=B,
                         lora_scale=w.lora_scale)
    dt = (time.perf_counter() - t0) / reps
    return len(rows) / dt, dt, len(experts)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count() or 1


def bench_reference(args, world, rank):
    """--impl reference: the oracle as it stands, one token of the workload per step, on host cores."""
    if rank != 0:
        return 0
    from bit_mixture_experts_top_b200 import layer
    from bit_mixture_experts_top_b200.workloads import WORKLOADS
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from helpers import oracle_stacks, touched_experts
    from oracle import moe as omoe
    w = WORKLOADS[WORKLOAD]
    x, logits = layer.synthetic_tokens(w, T_HEADLINE)
    steps, warmup = args.steps, args.warmup
    rows = [i % T_HEADLINE for i in range(steps + warmup)]
    stacks = oracle_stacks(w, touched_experts(logits[sorted(set(rows))], w.k))
    for i in range(warmup):
        omoe.moe_forward(x[rows[i]:rows[i] + 1], logits[rows[i]:rows[i] + 1], w.k, w.fmt, w.E, w.H, w.I, *stacks)
    t0 = time.perf_counter()
    for i in range(warmup, warmup + steps):
        omoe.moe_forward(x[rows[i]:rows[i] + 1], logits[rows[i]:rows[i] + 1], w.k, w.fmt, w.E, w.H, w.I, *stacks)
    dt = time.perf_counter() - t0
    value = steps / dt
    cores = blas_threads()
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": steps, "warmup": warmup,
        "ms_per_step": dt * 1e3 / steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": f"{WORKLOAD} T={T_HEADLINE} (one token per step)", "E": w.E, "H": w.H, "I": w.I,
                   "k": w.k, "format": w.fmt, "global_batch": 1, "parallelism": "cpu oracle, rank 0 only"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": "one token of the T=64 decode batch per step (8 routed experts decoded in fp64)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


class Replicas:
    """Process-group plumbing of the replicas run: one process per GPU, no data exchange;
    a barrier around the timed region and the max over ranks of every time.  NCCL on GPUs,
    gloo for the CPU tests of this logic; world == 1 needs no process group."""

    def __init__(self, world, rank, backend="nccl", device=None, timeout_s=120):
        import torch
        self.world, self.rank, self.device = world, rank, device
        self.dist = world > 1
        if self.dist:
            import datetime
            import torch.distributed as tdist
            kw = {"device_id": device} if backend == "nccl" else {}
            tdist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
        self._torch = torch

    def barrier(self):
        if self.dist:
            self._torch.distributed.barrier()

    def max_over_ranks(self, v):
        if not self.dist:
            return v
        t = self._torch.tensor([v], dtype=self._torch.float64, device=self.device)
        self._torch.distributed.all_reduce(t, op=self._torch.distributed.ReduceOp.MAX)
        return float(t.item())

    def whole_job_rate(self, units_per_rank, ms_max):
        """Units every rank processed per second of the slowest rank (weak scaling)."""
        return self.world * units_per_rank / (ms_max * 1e-3)

    def emit(self, line):
        if self.rank == 0:
            print(json.dumps(line), flush=True)

    def close(self):
        if self.dist:
            self._torch.distributed.destroy_process_group()


def bench_e4b(args, world, rank, local):
    import torch
    from bit_mixture_experts_top_b200 import e4b, layer
    from bit_mixture_experts_top_b200.workloads import WORKLOADS

    dist = world > 1
    if dist:
        torch.cuda.set_device(local)
    dev = torch.device("cuda", local if dist else 0)
    torch.cuda.set_device(dev)
    rep = Replicas(world, rank, "nccl", dev)
    barrier, max_over_ranks = rep.barrier, rep.max_over_ranks

    w = WORKLOADS[args.workload]
    T = args.tokens
    lay = layer.synthetic_layer(w, dev)
    x_np, lg_np = layer.synthetic_tokens(w, T)
    x = layer.bits_tensor(x_np, dev)
    lg = layer.bits_tensor(lg_np, dev)
    out = torch.empty((T, w.H), dtype=torch.bfloat16, device=dev)
    ws = lay.workspace(T, dev)
    args_fwd = (lay.desc, T, x, lg, lay.gate_up.codes, lay.gate_up.scales, lay.down.codes, lay.down.scales,
                lay.lora_A, lay.lora_B, lay.gu_bias, lay.dn_bias, out, ws)

    def forward():
        e4b.e4b_moe_forward(*args_fwd)

    for _ in range(args.warmup):
        forward()
    torch.cuda.synchronize()
    if e4b.e4b_device_status(ws) != e4b.E4B_OK:
        raise RuntimeError("device status reported an error after warm-up")
    offs = lay.region(T, e4b.E4B_WS_EXPERT_OFFSETS, torch.int32).cpu().numpy()
    touched = int(np.count_nonzero(np.diff(offs)))
    R = T * w.k
    gu_bytes = touched * w.gate_up_bytes_per_expert() + R * w.H * 2 + R * w.I * 2
    dn_bytes = touched * w.down_bytes_per_expert() + R * w.I * 2 + R * w.H * 4
    layer_weight_bytes = touched * (w.gate_up_bytes_per_expert() + w.down_bytes_per_expert())

    # one step = one forward, replayed from a CUDA graph (the library's launches captured as-is)
    def capture(fn):
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            fn()
        torch.cuda.current_stream().wait_stream(side)
        with torch.cuda.graph(g):
            fn()
        return g

    g_fwd = capture(forward)
    # per-stage timing: each stage's graph runs the stage once per copy of the layer's packed stacks
    # (identical bytes at distinct addresses, like consecutive layers of a model, together at least 4x L2),
    # so every gate_up / down launch streams its weights from HBM and the graph launch is spread over the
    # copies; a stage's time is the replay time over the copies
    n_copies = max(2, 1 if layer_weight_bytes >= ROTATE_BYTES
                   else min(MAX_COPIES, -(-ROTATE_BYTES // max(layer_weight_bytes, 1))))
    stage_layers = [(lay.gate_up.codes, lay.gate_up.scales, lay.down.codes, lay.down.scales)] + [
        (lay.gate_up.codes.clone(), lay.gate_up.scales.clone(), lay.down.codes.clone(), lay.down.scales.clone())
        for _ in range(n_copies - 1)]

    def stage_all(st):
        for gc, gs, dc, ds in stage_layers:
            e4b.e4b_moe_forward_stage(st, lay.desc, T, x, lg, gc, gs, dc, ds, lay.lora_A, lay.lora_B, lay.gu_bias,
                                      lay.dn_bias, out, ws)

    g_gu = capture(lambda: stage_all(e4b.E4B_STAGE_GATE_UP))
    g_dn = capture(lambda: stage_all(e4b.E4B_STAGE_DOWN))
    g_small = {nm: capture(lambda st=st: stage_all(st)) for nm, st in
               (("route_ms", e4b.E4B_STAGE_ROUTE), ("gather_ms", e4b.E4B_STAGE_GATHER),
                ("combine_ms", e4b.E4B_STAGE_COMBINE))}
    for _ in range(3):
        g_fwd.replay()
    torch.cuda.synchronize()

    K = args.steps
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(physical_gpu_index(local))
    barrier()
    torch.cuda.synchronize()
    sampler.start()
    with torch.cuda.nvtx.range(f"timed: {K} forwards"):      # NVTX ranges mark the bench's phases for nsys
        t_start.record()
        for _ in range(K):
            g_fwd.replay()
        t_end.record()
        torch.cuda.synchronize()
    clocks = sampler.summary()
    barrier()
    total_ms = t_start.elapsed_time(t_end)
    ms_per_step = max_over_ranks(total_ms / K)

    def time_graph(g, n):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        evs[0].record()
        for i in range(n):
            g.replay()
            evs[i + 1].record()
        torch.cuda.synchronize()
        return statistics.fmean(evs[i].elapsed_time(evs[i + 1]) for i in range(n))

    # the dominant kernel, launch by launch (touched weights per launch exceed L2: no flush needed)
    n_stage = min(K, 500)
    with torch.cuda.nvtx.range("per-stage timing"):
        gu_ms = max_over_ranks(time_graph(g_gu, n_stage) / n_copies)
        dn_ms = max_over_ranks(time_graph(g_dn, n_stage) / n_copies)
        small_ms = {nm: max_over_ranks(time_graph(g, n_stage) / n_copies) for nm, g in g_small.items()}
    if e4b.e4b_device_status(ws) != e4b.E4B_OK:
        raise RuntimeError("device status reported an error in the timed region")
    del g_fwd, g_gu, g_dn, g_small, stage_layers

    # end to end through the public host-to-host call (layer.HostForward): every step copies the
    # inputs from pinned host memory, runs the layer and copies the output back (one graph replay)
    hf = layer.HostForward(lay, T, dev)
    hf.x.copy_(torch.from_numpy(x_np.view(np.int16)))
    hf.logits.copy_(torch.from_numpy(lg_np.view(np.int16)))
    e2e_steps = min(K, 200)
    for _ in range(3):
        hf.run()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.nvtx.range(f"end to end: {e2e_steps} host-to-host forwards"):
        e0.record()
        for _ in range(e2e_steps):
            hf.run()
        e1.record()
        torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps)
    barrier()
    h2d_bytes = int(hf.x.numel() * 2 + hf.logits.numel() * 2)
    d2h_bytes = int(hf.out.numel() * 2)
    del hf

    # the two standalone format kernels on their full stacks (inputs larger than L2, timed per launch)
    formats = {}
    if args.workload == WORKLOAD and not args.no_formats:
        gen = torch.Generator(device=dev)
        gen.manual_seed(0)
        n_q = 128 * 2048 * 1536                      # the Qwen3-shaped gate_up stack, fp32 N(0, 0.02)
        xq = torch.empty(n_q, dtype=torch.float32, device=dev).normal_(0.0, 0.02, generator=gen)
        cq = torch.empty(n_q // 2, dtype=torch.uint8, device=dev)
        aq = torch.empty(n_q // 64, dtype=torch.float32, device=dev)
        n_d = 32 * 2880 * 5760                       # the gpt-oss-20b-shaped gate_up stack
        cd = torch.randint(0, 256, (n_d // 2,), dtype=torch.uint8, device=dev, generator=gen)
        sd = torch.randint(121, 129, (n_d // 32,), dtype=torch.uint8, device=dev, generator=gen)
        od = torch.empty(n_d, dtype=torch.int16, device=dev)

        def time_calls(fn, n=20):
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
            evs[0].record()
            for i in range(n):
                fn()
                evs[i + 1].record()
            torch.cuda.synchronize()
            return statistics.fmean(evs[i].elapsed_time(evs[i + 1]) for i in range(n))

        q_ms = max_over_ranks(time_calls(lambda: e4b.e4b_quantize_nf4(xq, n_q, cq, aq)))
        d_ms = max_over_ranks(time_calls(lambda: e4b.e4b_dequant_mxfp4(cd, sd, n_d, od)))
        q_bytes = n_q * 4 + n_q // 2 + n_q // 64 * 4
        d_bytes = n_d // 2 + n_d // 32 + n_d * 2
        formats = {"quantize_nf4": {"shape": [128, 2048, 1536], "ms": q_ms, "bytes": q_bytes,
                                    "gbs": q_bytes / (q_ms * 1e-3) / 1e9},
                   "dequant_mxfp4": {"shape": [32, 2880, 5760], "ms": d_ms, "bytes": d_bytes,
                                     "gbs": d_bytes / (d_ms * 1e-3) / 1e9}}
        del xq, cq, aq, cd, sd, od

    peaks, peak_kind = load_peaks()
    configs = []
    if args.workload == WORKLOAD and not args.no_configs:
        with torch.cuda.nvtx.range("every configuration"):
            configs = bench_configs(dev, peaks, max_over_ranks,
                                    only=set(args.only_config.split(",")) if args.only_config else None)
    for f in formats.values():
        f["frac_of_hbm"] = f["gbs"] / peaks["hbm_gbs"]
    # the library's kernel choice (tokens_per_tile 0): the decode kernel at <= 12 rows per routed expert
    active = min(R, w.E)
    decode_kernel = (R + active - 1) // active <= 12
    # decode shapes are bound by the weight stream, prefill shapes by the tensor cores
    gu_flops = 2 * R * w.H * 2 * w.I + (2 * R * (w.H + 2 * w.I) * w.lora_rank if w.lora_rank else 0)
    tensor_bound = gu_flops / gu_bytes > peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if tensor_bound:
        roof = {"bound": "tensor", "achieved": gu_flops / (gu_ms * 1e-3) / 1e12, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "algorithmic_flops_per_launch": gu_flops}
    else:
        roof = {"bound": "hbm", "achieved": gu_bytes / (gu_ms * 1e-3) / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "algorithmic_bytes_per_launch": gu_bytes}
    roof["frac"] = roof["achieved"] / roof["peak"]
    value = rep.whole_job_rate(T, ms_per_step)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{args.workload} T={T}", "E": w.E, "H": w.H, "I": w.I, "k": w.k, "format": w.fmt,
                   "global_batch": T * world, "tokens_per_gpu": T, "parallelism": f"replicas x{world}",
                   "l2": f"inputs larger than L2: {layer_weight_bytes / 1e6:.0f} MB of touched expert weights "
                         f"per step vs {L2_BYTES / 1e6:.0f} MB L2, no flush"},
        "roofline": {"kernel": ("skinny_gemm gate_up (decode kernel: codes decoded in registers, warp-level MMA, "
                                "SwiGLU)" if decode_kernel else
                                "grouped_gemm gate_up (tcgen05, dequant to tensor memory, SwiGLU)"),
                     **roof, "peak_kind": peak_kind,
                     "traffic": recorded_traffic("gate_up", f"{args.workload} T={T}",
                                                 "skinny_gemm.cu" if decode_kernel else "grouped_gemm.cu"),
                     "avg_launch_ms": gu_ms,
                     "avg_launch_timing": f"{n_stage} replays of a graph holding the launch once per copy of the "
                                          f"packed stacks ({n_copies} copies at distinct addresses), per launch"},
        "kernels": {"gate_up_ms": gu_ms, "down_ms": dn_ms, **small_ms,
                    "down_gbs": dn_bytes / (dn_ms * 1e-3) / 1e9,
                    "layer_weight_gbs": layer_weight_bytes / (ms_per_step * 1e-3) / 1e9,
                    "touched_experts": touched},
        "e2e": {"value": rep.whole_job_rate(T, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes,
                "path": "layer.HostForward.run: torch copies the inputs from pinned host tensors to the device, "
                        "the library's forward runs, torch copies the output back to a pinned host tensor; "
                        "one CUDA graph replay and a synchronize per step"},
        "standalone_kernels": formats,
        "configs": configs,
        "gpu_launches": K * KERNELS_PER_STEP,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ns = min(T, 64)     # a bounded sample of the batch for prefill shapes
        tps, dt, ne = oracle_tokens_per_s(w, x_np, lg_np, np.arange(ns), reps=2)
        what = f"the whole T={T} batch" if ns == T else f"the first {ns} of the T={T} tokens"
        line["cpu_baseline"] = {"value": tps, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                                "sample": f"{what} ({ne} experts decoded in fp64), "
                                          f"timed twice, {dt:.1f} s per forward"}
    rep.emit(line)
    rep.close()
    return 0


def main():
    from bit_mixture_experts_top_b200.workloads import WORKLOADS
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["e4b", "reference"], default="e4b")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing")
    ap.add_argument("--no-formats", action="store_true", help="skip timing the standalone format kernels")
    ap.add_argument("--no-configs", action="store_true", help="skip timing every configuration of the metric")
    ap.add_argument("--only-config", default=None,
                    help="time only these configurations (comma-separated workload:T, e.g. qwen3_30b_a3b_nf4_lora:512)")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=WORKLOAD,
                    help="synthetic layer to time (default: the headline decode workload)")
    ap.add_argument("--tokens", type=int, default=None, help="tokens per step (default: the workload's largest)")
    args = ap.parse_args()
    if args.tokens is None:
        args.tokens = T_HEADLINE if args.workload == WORKLOAD else WORKLOADS[args.workload].tokens[-1]
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world, rank, local = init_dist()
    if args.impl == "reference":
        return bench_reference(args, world, rank)
    return bench_e4b(args, world, rank, local)


if __name__ == "__main__":
    sys.exit(main())
