#!/usr/bin/env python
"""Throughput of one QLoRA training step of the grouped NF4 expert block.

A step is one pass of the whole hot path over one batch: routing and
permutation, the grouped NF4+LoRA forward (gate_up with the SiLU-gated
epilogue, down, combine), the input gradient (down dgrad with the SwiGLU
backward, gate_up dgrad, un-permute) and the LoRA weight gradients -- the
four C-ABI calls of libe4b.so.  Default workload: E=128, H=2048, I=768,
top-8, T=8192 tokens per GPU, LoRA r=64, alpha=128, Zipf(1.1) routing.
A forward-only workload (``--workload decode``: 16 tokens) times the serving
call e4b_moe_serve_fwd (routing + forward, nothing kept for a backward)
replayed from a CUDA graph.

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle on
bounded token samples of the same workload instead.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
"""

from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-block fwd+bwd tokens/s and TFLOP/s at 1 B200; % of tensor/HBM roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NVML_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
                0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
                0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["e4b", "reference"], default="e4b")
    ap.add_argument("--workload", default="train")
    ap.add_argument("--cpu-sample-tokens", type=int, default=24,
                    help="tokens of the oracle's cpu_baseline sample")
    ap.add_argument("--ref-tokens", type=int, default=1, help="tokens per step of the reference arm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sub-workloads", default=",".join(SUB_WORKLOADS),
                    help="comma-separated workloads timed beside the headline one (1 GPU); '' for none")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in PEAKS_FALLBACK}, "measured"
    except Exception:
        return dict(PEAKS_FALLBACK), "fallback"


def nf4_gemm_source_hash():
    """Hash of the grouped NF4 GEMM kernel's source text: gemm.cu from its namespace to the next
    kernel's section (the kernel, its parameters and its constants)."""
    import hashlib
    gemm = open(os.path.join(ROOT, "grouped_nf4_expert_b200", "csrc", "gemm.cu"), "rb").read()
    i = gemm.index(b"namespace nf4g {")
    j = gemm.index(b"// LoRA projection: out[rows, r]", i)
    return hashlib.sha256(gemm[i:j]).hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per step of the nf4_gemm launches from the committed ncu summary, if the kernel
    source still hashes to what was profiled; else None."""
    import re
    sha = nf4_gemm_source_hash()
    try:
        text = open(os.path.join(ROOT, "profiles", "nf4_gemm_train_ncu.md")).read()
    except OSError:
        return None
    m_t = re.search(r"^traffic_bytes_per_step: (\d+)", text, re.M)
    m_s = re.search(r"^source_sha256_16: ([0-9a-f]+)", text, re.M)
    if m_t and m_s and m_s.group(1) == sha:
        return int(m_t.group(1))
    return None


def step_flops(cfg):
    """Algorithmic FLOPs of one step of the workload's passes (forward, input gradient, LoRA weight
    gradients): routed slots only, 2 FLOP per MAC."""
    N, H, I, r = cfg.N, cfg.H, cfg.I, cfg.r
    lora = 2.0 * N * r * (2 * H + 3 * I)     # one pass's LoRA products (projections and K=r terms)
    flops = 6.0 * N * H * I + lora           # forward: gate_up + down
    if "dgrad" in cfg.passes:
        flops += 6.0 * N * H * I + lora      # dgrad down + gate_up
    if "wgrad" in cfg.passes:
        flops += lora                        # the four weight-gradient products
    return flops


def fwd_flops(cfg):
    """Algorithmic FLOPs of the forward alone (gate_up, down and the forward LoRA terms)."""
    N, H, I, r = cfg.N, cfg.H, cfg.I, cfg.r
    return 6.0 * N * H * I + 2.0 * N * r * (2 * H + 3 * I)


def nf4_gemm_flop_total(gflops, kern):
    """FLOPs of the grouped NF4 GEMM launches the profiler recorded (each mode's work per launch times
    its launches): the modes a workload does not run count nothing."""
    return sum(f * kern[n][0] for n, f in gflops.items() if n in kern)


def stream_bytes(cfg, touched):
    """Algorithmic HBM bytes of the two streaming forward launches: the NF4 codes and
    fp32 block scales of every expert the batch routes to, each read once."""
    per_weight = 0.5 + 4.0 / 64
    return {"nf4_stream_fwd_gate_up": touched * 2 * cfg.I * cfg.H * per_weight,
            "nf4_stream_fwd_down": touched * cfg.H * cfg.I * per_weight}


def serve_bytes(cfg, touched):
    """Algorithmic HBM bytes of the one-launch serving forward: the NF4 codes and fp32 block scales
    of both stacks of every expert the batch routes to, each read once."""
    return {"nf4_serve": sum(stream_bytes(cfg, touched).values())}


def router_bwd_bytes(cfg):
    """Algorithmic HBM bytes of one router-backward launch: per token its k expert-output rows and
    its upstream-gradient row (bf16), its ids, weights and rows (int32/fp32), and its [E] fp32
    logit-gradient row written."""
    T, k, H, E = cfg.T, cfg.top_k, cfg.H, cfg.E
    return T * (k + 1) * H * 2 + T * k * 12 + T * E * 4


def quantize_bytes(n):
    """Algorithmic HBM bytes of quantising n bf16 weights: read once, NF4 codes and fp32 block
    scales written once."""
    return n * 2 + n // 2 + (n // 64) * 4


def nf4_gemm_flops(cfg):
    """Algorithmic FLOPs of the four grouped NF4 GEMM launches of one step."""
    N, H, I, r = cfg.N, cfg.H, cfg.I, cfg.r
    return {
        "nf4_gemm_fwd_gate_up": 2.0 * N * H * 2 * I + 2.0 * N * r * 2 * I,
        "nf4_gemm_fwd_down": 2.0 * N * I * H + 2.0 * N * r * H,
        "nf4_gemm_dgrad_down": 2.0 * N * H * I + 2.0 * N * r * I,
        "nf4_gemm_dgrad_gate_up": 2.0 * N * 2 * I * H + 2.0 * N * r * H,
    }


class ClockSampler:
    """Samples SM clock, power and clock-event reasons of one GPU through NVML."""

    def __init__(self, torch_device, period_s=0.01):
        self.samples, self.period, self.ok = [], period_s, False
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(torch_device).uuid).replace("GPU-", "")
            self.h = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == uuid:
                    self.h = h
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = self.h is not None
        except Exception as exc:  # clocks are reported as unavailable, never guessed
            self.err = repr(exc)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:
                    reasons = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                watts = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                self.samples.append((mhz, reasons, watts))
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
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        mhz = [s[0] for s in self.samples]
        mask = 0
        for s in self.samples:
            mask |= s[1]
        reasons = [name for bit, name in NVML_REASONS.items() if mask & bit and bit != 0x1]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples), "power_w_max": max(s[2] for s in self.samples)}


# --------------------------------------------------------------------------- oracle legs

def oracle_sample_step(prob, tokens):
    """The CPU oracle as it stands on a token sample: forward + backward (dx and the
    sample's LoRA-gradient contributions), dequantising the base in both passes;
    the forward alone for a forward-only workload."""
    import numpy as np

    import oracle
    from grouped_nf4_expert_b200 import inputs
    cfg = prob.cfg
    f = lambda b: inputs.bits_to_f32(b).astype(np.float64)  # noqa: E731
    ex = oracle.Experts(prob.gate_up_nf4, prob.gate_up_absmax, prob.down_nf4, prob.down_absmax,
                        f(prob.A_gu), f(prob.B_gu), f(prob.A_d), f(prob.B_d))
    x, dY = f(prob.x), f(prob.dY)
    oracle.moe_forward(x, prob.logits, ex, cfg.top_k, cfg.alpha, tokens=tokens)
    if cfg.passes != ("fwd",):
        oracle.moe_backward(x, prob.logits, dY, ex, cfg.top_k, cfg.alpha, tokens=tokens, grad_experts=[])


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(prob, n_tokens):
    import numpy as np
    n_tokens = min(n_tokens, prob.cfg.T)
    toks = np.sort(np.random.default_rng(7).choice(prob.cfg.T, size=n_tokens, replace=False))
    t0 = time.perf_counter()
    oracle_sample_step(prob, toks)
    dt = time.perf_counter() - t0
    return {"value": n_tokens / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": "%d random tokens of the %s workload, %s, float64 numpy, %.1f s" % (
                n_tokens, prob.cfg.name, passes_text(prob.cfg), dt)}


def passes_text(cfg):
    return ("forward only" if cfg.passes == ("fwd",)
            else "forward + backward (input gradient and their LoRA-gradient terms)")


def run_reference(args):
    from grouped_nf4_expert_b200 import inputs
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cfg = inputs.CONFIGS[args.workload]
    prob = inputs.make_problem(cfg)
    import numpy as np
    rng = np.random.default_rng(11)
    times = []
    args.ref_tokens = min(args.ref_tokens, cfg.T)
    for i in range(args.warmup + args.steps):
        toks = np.sort(rng.choice(cfg.T, size=args.ref_tokens, replace=False))
        t0 = time.perf_counter()
        oracle_sample_step(prob, toks)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    total = sum(times)
    value = args.ref_tokens * args.steps / total
    cores = blas_threads()
    sample = "%d random tokens per step of the %s workload, %s, float64 numpy" % (
        args.ref_tokens, cfg.name, passes_text(cfg))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(cfg, args.gpus),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(cfg, world):
    """The workload's identity, the same dict in both arms' lines (the GPU arm's call sequence and graph
    use are top-level keys of its own record)."""
    return {"workload": "%s: %s" % (cfg.name, cfg.note), "E": cfg.E, "H": cfg.H, "I": cfg.I,
            "top_k": cfg.top_k, "tokens_per_gpu": cfg.T, "global_batch": cfg.T * world, "r": cfg.r,
            "alpha": cfg.alpha, "routing": cfg.routing, "nf4_blocksize": 64, "parallelism": "dp%d" % world,
            "passes": list(cfg.passes),
            "l2": "GPU arm: flushed between timed steps by a 256 MiB write; reference arm: host memory"}


# --------------------------------------------------------------------------- GPU arm

# Workloads measured beside the headline one in the same run (each its own passes, timed the same way).
SUB_WORKLOADS = ("mixtral", "finegrained", "decode", "tiny")
# Oracle sample per workload for its cpu_baseline: tokens, chosen so each takes seconds on host cores.
SUB_CPU_TOKENS = {"mixtral": 1, "finegrained": 2, "decode": 2, "tiny": 32, "train": 24, "tiny_b0": 32}


class Ctx:
    """Device, ranks, peaks and the timing helpers shared by every workload of one run."""

    def __init__(self, args, dev, world, rank):
        import torch
        import torch.distributed as dist
        self.args, self.dev, self.world, self.rank = args, dev, world, rank
        self.torch, self.dist = torch, dist
        self.flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)  # 2x the 126 MB L2
        self.peaks, self.peak_src = load_peaks()

    def sync_all(self):
        self.torch.cuda.synchronize(self.dev)
        if self.world > 1:
            self.dist.barrier()

    def timed(self, K, body, flush_l2=True):
        """Device time of K calls of body() (ms, summed over per-call CUDA events; max over ranks)."""
        torch = self.torch
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        self.sync_all()
        for i in range(K):
            if flush_l2:
                self.flush.fill_(i & 0xFF)  # evict the previous step's working set from L2
            evs[i][0].record()
            body()
            evs[i][1].record()
        self.sync_all()
        ms = sum(a.elapsed_time(b) for a, b in evs)
        if self.world > 1:
            t = torch.tensor([ms], dtype=torch.float64, device=self.dev)
            self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
            ms = float(t.item())
        return ms

    def capture(self, body):
        """A CUDA graph of body() (the serving step: the library allocates and synchronises nothing),
        and the number of library launches it holds."""
        from grouped_nf4_expert_b200 import e4b
        torch = self.torch
        torch.cuda.synchronize(self.dev)
        g = torch.cuda.CUDAGraph()
        n0 = e4b.e4b_launch_count()
        with torch.cuda.graph(g):
            body()
        n = e4b.e4b_launch_count() - n0
        torch.cuda.synchronize(self.dev)
        return g, n


def tensor_roofline(ctx, kern, gflops, steps, traffic):
    """The grouped NF4 GEMM launches against the dense bf16 tensor peak.  The timed regions are well
    under a second at full clocks, so the fraction is taken against the measured burst GEMM peak;
    the fraction of the sustained (power-capped, seconds-long) figure is given beside it."""
    peaks = ctx.peaks
    nf4_ms = sum(kern.get(n, (0, 0.0))[1] for n in gflops)
    nf4_launches = sum(kern.get(n, (0, 0.0))[0] for n in gflops)
    nf4_flop = nf4_gemm_flop_total(gflops, kern)
    achieved = nf4_flop / (nf4_ms / 1e3) / 1e12 if nf4_ms > 0 else None
    modes = [n[len("nf4_gemm_"):].replace("_", " ", 1) for n in gflops if n in kern]
    per_mode = {}
    for n, f in gflops.items():
        if n in kern and kern[n][1] > 0:
            a = f * kern[n][0] / (kern[n][1] / 1e3) / 1e12
            per_mode[n] = {"achieved": a, "frac": a / peaks["bf16_tflops"],
                           "avg_launch_ms": kern[n][1] / kern[n][0]}
    return {"kernel": "nf4_gemm (%s)" % ", ".join(modes), "bound": "tensor",
            "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": (achieved / peaks["bf16_tflops"]) if achieved else None,
            "peak_source": "%s bf16_tflops (burst: the timed region is well under a second at full clocks)"
                           % ctx.peak_src,
            "frac_of_sustained": (achieved / peaks["bf16_tflops_sustained"]) if achieved else None,
            "traffic": traffic,
            "traffic_unit": "DRAM bytes per step of the nf4_gemm launches (ncu)",
            "launches": nf4_launches, "avg_launch_ms": nf4_ms / max(nf4_launches, 1),
            "algorithmic_flop_per_step": nf4_flop / steps, "per_mode": per_mode}


def pipelined_e2e(ctx, K, blk, base, lora, d, ins, outs, houts, do_wgrad, grads):
    """Device time (ms, max over ranks) of K training steps end to end through the public calls: every
    step's inputs come from pinned host memory (`ins`) and its results (`outs`) go back to pinned host
    memory, on two copy streams, so that step i+1's copy-in and step i's copy-out overlap the compute
    of their neighbours.  Timed from the first copy-in to the last copy-out."""
    import torch
    from grouped_nf4_expert_b200 import parallel
    dev = ctx.dev
    cs = torch.cuda.current_stream(dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    dins = [(d.x, d.logits, d.dY), tuple(t.clone() for t in (d.x, d.logits, d.dY))]
    stage = [[torch.empty_like(t) for t in outs] for _ in range(2)]
    hsets = [houts, [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]]
    in_ready = [torch.cuda.Event() for _ in range(K)]
    done = [torch.cuda.Event() for _ in range(K)]
    out_done = [torch.cuda.Event() for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def copy_in(i):
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(done[i - 2])  # step i-2 used this input set
            for dst, src in zip(dins[i % 2], ins):
                dst.copy_(src, non_blocking=True)
            in_ready[i].record(s_in)

    ctx.sync_all()
    t0.record(s_in)
    copy_in(0)
    for i in range(K):
        if i + 1 < K:
            copy_in(i + 1)
        cs.wait_event(in_ready[i])
        x, logits, dy = dins[i % 2]
        blk.e4b_route_permute(logits, x, gather=False)
        blk.e4b_grouped_nf4_lora_fwd(base, lora, x=x)
        blk.e4b_grouped_nf4_lora_dgrad(base, lora, dy)
        if do_wgrad:
            blk.e4b_lora_wgrad()
            if ctx.world > 1:
                parallel.allreduce_lora_grads(grads)
        if i >= 2:
            cs.wait_event(out_done[i - 2])  # step i-2's results have left this staging set
        for dst, src in zip(stage[i % 2], outs):
            dst.copy_(src, non_blocking=True)
        done[i].record(cs)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done[i])
            for dst, src in zip(hsets[i % 2], stage[i % 2]):
                dst.copy_(src, non_blocking=True)
            out_done[i].record(s_out)
    t1.record(s_out)
    ctx.sync_all()
    ms = t0.elapsed_time(t1)
    if ctx.world > 1:
        t = torch.tensor([ms], dtype=torch.float64, device=dev)
        ctx.dist.all_reduce(t, op=ctx.dist.ReduceOp.MAX)
        ms = float(t.item())
    return ms


def measure(ctx, cfg, headline):
    """Times one workload's step (its own passes) and returns its record."""
    import torch
    from grouped_nf4_expert_b200 import e4b, inputs, parallel
    from grouped_nf4_expert_b200 import device as dv

    args, dev, world, rank = ctx.args, ctx.dev, ctx.world, ctx.rank
    peaks, peak_src = ctx.peaks, ctx.peak_src
    prob = inputs.make_problem(cfg, data_rank=rank)
    d = dv.upload(prob, dev)
    blk = e4b.Block(dv.dims_of(cfg), cfg.T, dev)
    base, lora = d.base(), d.lora()
    grads = (blk.lora_grads,)  # dA_gu, dB_gu, dA_d, dB_d are views of this one buffer: one all-reduce

    fwd_only = cfg.passes == ("fwd",)  # a forward-only workload: the serving forward alone
    do_wgrad = "wgrad" in cfg.passes

    def step():
        if fwd_only:  # routing + forward for inference, nothing kept for a backward
            blk.e4b_moe_serve_fwd(d.logits, d.x, base, lora)
            return
        blk.e4b_route_permute(d.logits, d.x, gather=False)  # the forward gathers x with its first projection
        blk.e4b_grouped_nf4_lora_fwd(base, lora, x=d.x)
        blk.e4b_grouped_nf4_lora_dgrad(base, lora, d.dY)
        if do_wgrad:
            blk.e4b_lora_wgrad()
            if world > 1:  # data parallel: sum the LoRA gradients of all ranks (NCCL over NVLink)
                parallel.allreduce_lora_grads(grads)

    for _ in range(max(args.warmup, 3)):
        step()
    st = blk.check_device_error()
    if st != e4b.E4B_OK:
        raise RuntimeError("device error after warm-up: %s" % e4b.STATUS.get(st, st))

    # ---- main timed region (the serving step replays a CUDA graph of the call)
    graphs = []
    if fwd_only:
        g_step, per_step = ctx.capture(step)
        graphs.append(g_step)
        with ClockSampler(dev) as clocks:
            total_ms = ctx.timed(args.steps, g_step.replay)
        launches = per_step * args.steps
    else:
        launches0 = e4b.e4b_launch_count()
        with ClockSampler(dev) as clocks:
            total_ms = ctx.timed(args.steps, step)
        launches = e4b.e4b_launch_count() - launches0
    st = blk.check_device_error()
    if st != e4b.E4B_OK:
        raise RuntimeError("device error in the timed region: %s" % e4b.STATUS.get(st, st))
    ms_per_step = total_ms / args.steps
    value = cfg.T * world * args.steps / (total_ms / 1e3)
    flops = step_flops(cfg)

    # ---- per-kernel device times over a second timed region (library profiler, events on the launch stream)
    e4b.e4b_profiler_enable(True)
    prof_ms = ctx.timed(args.steps, step)
    e4b.e4b_profiler_enable(False)
    kern = e4b.e4b_profiler_read()
    kern_total = sum(v[1] for v in kern.values())
    roofline = tensor_roofline(ctx, kern, nf4_gemm_flops(cfg), args.steps,
                               profiled_traffic() if cfg.name == "train" else None)
    touched = int((blk.counts > 0).sum().item())
    sbytes = serve_bytes(cfg, touched) if "nf4_serve" in kern else stream_bytes(cfg, touched)
    st_ms = sum(kern.get(n, (0, 0.0))[1] for n in sbytes)
    if st_ms > 0:  # the weight-streaming forward ran: it is HBM-bound by design
        st_launches = sum(kern.get(n, (0, 0.0))[0] for n in sbytes)
        st_bytes = sum(sbytes.values()) * args.steps
        ach = st_bytes / (st_ms / 1e3) / 1e9
        per_mode = {}
        for n in sbytes:
            if n in kern and kern[n][0] > 0:
                launch_ms = kern[n][1] / kern[n][0]  # one launch of each per step
                per_mode[n] = {"achieved": sbytes[n] / (launch_ms / 1e3) / 1e9, "avg_launch_ms": launch_ms,
                               "algorithmic_bytes": sbytes[n]}
        for v in per_mode.values():
            v["frac"] = v["achieved"] / peaks["hbm_gbs"]
        name = ("nf4_serve (x scatter + p_gu, gate_up, p_d, down, combine in one launch)" if "nf4_serve" in sbytes
                else "nf4_stream (fwd gate_up, fwd down)")
        roofline = {"kernel": name, "bound": "hbm", "achieved": ach,
                    "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": ach / peaks["hbm_gbs"],
                    "peak_source": "%s hbm_gbs" % peak_src, "traffic": None,
                    "traffic_unit": "DRAM bytes per launch (ncu), see profiles/",
                    "launches": st_launches, "avg_launch_ms": st_ms / max(st_launches, 1),
                    "algorithmic_bytes_per_step": sum(sbytes.values()), "per_mode": per_mode}
    if cfg.name.startswith("tiny"):
        roofline = dict(roofline, note="latency-bound at this size (a few MFLOP per step): reported, not a target")
    per_kernel = {n: {"launches_per_step": v[0] / args.steps, "ms_per_step": v[1] / args.steps,
                      "share": v[1] / kern_total if kern_total else None} for n, v in kern.items()}

    # ---- end to end through the public API with host buffers
    pin = lambda t: torch.empty(t.shape, dtype=t.dtype, pin_memory=True)  # noqa: E731
    hx, hl, hdy = pin(d.x), pin(d.logits), pin(d.dY)
    hx.copy_(d.x)
    hl.copy_(d.logits)
    hdy.copy_(d.dY)
    outs = [blk.y] if fwd_only else [blk.y, blk.dx] + ([blk.lora_grads] if do_wgrad else [])
    houts = [pin(t) for t in outs]
    ins = (hx, hl) if fwd_only else (hx, hl, hdy)
    h2d = sum(t.numel() * t.element_size() for t in ins)
    d2h = sum(t.numel() * t.element_size() for t in houts)

    def e2e_step():
        d.x.copy_(hx, non_blocking=True)
        d.logits.copy_(hl, non_blocking=True)
        if not fwd_only:
            d.dY.copy_(hdy, non_blocking=True)
        step()
        for h, t in zip(houts, outs):
            h.copy_(t, non_blocking=True)

    if fwd_only:  # the whole serving step, copies included, as one graph
        g_e2e, _ = ctx.capture(e2e_step)
        graphs.append(g_e2e)
        e2e_ms = ctx.timed(args.steps, g_e2e.replay)
        e2e_how = "each step: copy-in, the serving call, copy-out, one CUDA graph"
    else:
        e2e_ms = pipelined_e2e(ctx, args.steps, blk, base, lora, d, ins, outs, houts, do_wgrad, grads)
        e2e_how = ("training loop: step i+1's inputs are copied in and step i's results copied out on two copy "
                   "streams while the compute stream runs (inputs and results double-buffered on the device; "
                   "each step's results are first copied to a device staging buffer on the compute stream)")
    e2e = {"value": cfg.T * world * args.steps / (e2e_ms / 1e3), "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / args.steps,
           "schedule": e2e_how}

    rec = {
        "value": value, "unit": "tokens/s", "ms_per_step": ms_per_step,
        "config": workload_config(cfg, world),
        "call": ("e4b_moe_serve_fwd" if fwd_only else
                 "route_permute + lora_fwd + lora_dgrad" + (" + lora_wgrad" if do_wgrad else "")),
        "cuda_graph": fwd_only,
        "tflops": flops * world / (ms_per_step / 1e3) / 1e12,
        "step_flop_per_gpu": flops,
        "roofline": roofline,
        "kernels": per_kernel,
        "profiled_ms_per_step": prof_ms / args.steps,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks.summary(),
    }
    if "dgrad" in cfg.passes or fwd_only:
        rec["routed_experts"] = int((blk.counts > 0).sum().item())

    # ---- the rows next to the path, each timed alone (HBM-bound by design).  Both read more than the
    # 126 MB L2 per launch, so they are timed back to back without the flush (whose dirty lines would
    # be written back during the next launch).
    if headline:
        next_rows = {}
        if not fwd_only:  # router backward (for a trained router) on this step's forward outputs
            d_logits = torch.empty((cfg.T, cfg.E), dtype=torch.float32, device=dev)
            rb_ms = ctx.timed(args.steps, lambda: blk.e4b_router_backward(d.dY, d_logits),
                              flush_l2=False) / args.steps
            rb_b = router_bwd_bytes(cfg)
            next_rows["router_backward"] = {
                "launch_ms": rb_ms, "algorithmic_bytes": rb_b, "achieved": rb_b / (rb_ms / 1e3) / 1e9,
                "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": rb_b / (rb_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                "bound": "hbm", "l2": "not flushed: > 300 MB read per launch",
                "note": "d(logits) [T,E] from dY and the forward's y_perm"}
            del d_logits
        nq = cfg.E * 2 * cfg.I * cfg.H  # the workload's gate_up stack, bf16 N(0, sigma_w)
        gq = torch.Generator(device=dev).manual_seed(1234 + rank)
        wq = (torch.randn(nq, generator=gq, device=dev) * cfg.sigma_w).to(torch.bfloat16)
        pq = torch.empty(nq // 2, dtype=torch.uint8, device=dev)
        aq = torch.empty(nq // 64, dtype=torch.float32, device=dev)
        q_ms = ctx.timed(args.steps, lambda: e4b.e4b_nf4_quantize(wq, pq, aq), flush_l2=False) / args.steps
        q_b = quantize_bytes(nq)
        next_rows["nf4_quantize"] = {
            "launch_ms": q_ms, "weights": nq, "algorithmic_bytes": q_b, "achieved": q_b / (q_ms / 1e3) / 1e9,
            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": q_b / (q_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
            "bound": "hbm", "l2": "not flushed: > 800 MB read per launch",
            "note": "bf16 gate_up stack [E,2I,H] -> packed NF4 + fp32 absmax"}
        del wq, pq, aq
        rec["next_rows"] = next_rows
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n_tok = args.cpu_sample_tokens if headline else SUB_CPU_TOKENS.get(cfg.name, 1)
        rec["cpu_baseline"] = cpu_baseline(prob, n_tok)
    del graphs, blk, d
    torch.cuda.empty_cache()
    return rec


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    from grouped_nf4_expert_b200 import build, e4b, inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    e4b.lib()

    ctx = Ctx(args, dev, world, rank)
    cfg = inputs.CONFIGS[args.workload]
    head = measure(ctx, cfg, headline=True)
    line = {
        "metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": head["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
    }
    line.update({k: v for k, v in head.items() if k not in line and k not in ("unit",)})
    # The other workloads, each timed the same way in the same run (one GPU: a data-parallel run times
    # the headline step only, since every rank would hold its GPU for them).
    subs = [w for w in (args.sub_workloads.split(",") if args.sub_workloads else []) if w and w != args.workload]
    if world == 1 and subs:
        line["workloads"] = {w: measure(ctx, inputs.CONFIGS[w], headline=False) for w in subs}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
