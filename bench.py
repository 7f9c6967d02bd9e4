#!/usr/bin/env python
"""Throughput of the DeepSeekMoE layer forward pass on B200.

One step = one full forward pass of the layer (router, scan/permute, gate/up GEMM with
SwiGLU, down GEMM, combine, balance statistics) over one batch of T tokens already
resident in HBM.  Default workload: the DeepSeekMoE-16B-shaped layer at prefill
(T=16384, d=2048, 2 shared + 64 routed experts of width 1408, top-6, bf16).

  python bench.py [--gpus N --steps K --warmup W] [--config NAME] [--impl ours|reference]

Multi-GPU (torchrun, one process per GPU): every rank runs its own T tokens (data
parallel, weights replicated, weak scaling); the only exchange is the all-reduce of the
per-expert counts and affinity sums for the global balance loss.
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s and expert-GEMM TFLOP/s (% BF16 peak), 16B-shaped, 1 B200"
L2_BYTES = 126 * 2 ** 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNELS = ("router", "scan", "permute", "gate_up_gemm", "down_gemm", "combine")
# kernel-by-kernel timing at burst clocks: forwards timed, and the pause before and after
KERNEL_BURST_FORWARDS = 8
KERNEL_REST_S = 1.0


def parse_args():
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=400)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--config", default="16b_prefill")
    p.add_argument("--tokens", type=int, default=None,
                   help="override the token count T of the workload (profiling captures)")
    p.add_argument("--e2e-steps", type=int, default=20)
    p.add_argument("--cpu-seconds", type=float, default=15.0,
                   help="target CPU time of the oracle baseline sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-graph", action="store_true",
                   help="launch the forward eagerly instead of replaying captured CUDA graphs")
    p.add_argument("--sustained-seconds", type=float, default=3.0,
                   help="after the timed steps, run forwards back to back this long and report "
                        "the power-capped (sustained) throughput beside the value; 0 skips it")
    p.add_argument("--backward", type=int, default=0, metavar="K",
                   help="also time K forward + backward steps (input, router and weight "
                        "gradients) after the forward measurements and add a 'backward' "
                        "object to the line; bf16 prefill-sized layers only")
    p.add_argument("--expert-parallel", action="store_true",
                   help="time the expert-parallel forward instead (routed experts split over the "
                        "ranks, token rows exchanged by all-to-all; one rank: local copies) and "
                        "print its line; not the headline")
    p.add_argument("--dry-run", action="store_true",
                   help="CPU check of the multi-rank plumbing (gloo): rank discovery, the "
                        "global balance loss's exchange on synthetic per-rank statistics and "
                        "max-over-ranks timing; no GPU and no forward pass, value null")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return {k: float(pk[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def peak_regime(clk: dict | None, timed_s: float) -> str:
    """Which measured bf16 peak a tensor-bound kernel is held against: 'sustained' (the
    seconds-long loop under the 1 kW power cap) when the run was power-capped -- timed for at
    least half a second with sw_power_cap seen and the median SM clock below 90% of its
    maximum -- else 'burst' (the peak of a GEMM timed alone at full clock)."""
    if not clk or not clk.get("sm_mhz") or not clk.get("sm_max_mhz"):
        return "burst"
    capped = "sw_power_cap" in clk.get("reasons", []) and clk["sm_mhz"] < 0.9 * clk["sm_max_mhz"]
    return "sustained" if capped and timed_s >= 0.5 else "burst"


PEAK_KEY = {"burst": "bf16_tflops", "sustained": "bf16_tflops_sustained"}


def choose_kernel_timing(regime: str, no_graph: bool, burst_kt, post_kt):
    """The per-kernel timing pass held against the timed region's peak: the one measured in
    the same clock regime.  burst_kt / post_kt = (summed ms per kernel, forwards, clocks) of
    the pass before the timed region (after a pause) and of the pass right after it (or,
    with no_graph, of the timed steps themselves).  Returns (ms, forwards, clocks, text)."""
    ms, n, clk = post_kt
    if no_graph:
        return ms, n, clk, "CUDA events between the library's kernels over the timed steps"
    if regime == "burst" and burst_kt is not None:
        ms, n, clk = burst_kt
        return ms, n, clk, (f"CUDA events between the library's kernels over {n} eager forwards "
                            f"after a {KERNEL_REST_S:.0f} s pause before the timed region (burst "
                            "clocks, as in the timed region)")
    return ms, n, clk, (f"CUDA events between the library's kernels over {n} eager forwards "
                        "right after the timed region (its clock regime)")


def workload_desc(w, n_gpus: int) -> dict:
    return {"workload": f"{w.name}: T={w.T} d={w.d} shared={w.n_shared} routed={w.n_routed} "
                        f"inter={w.inter} top_k={w.top_k} {w.dtype}"
                        f"{(' (gate/up and down e4m3)' if getattr(w, 'down_e4m3', False) else ' (gate/up e4m3)') if getattr(w, 'gate_up_e4m3', False) else ''}",
            "T_per_gpu": w.T, "d": w.d, "n_shared": w.n_shared, "n_routed": w.n_routed,
            "inter": w.inter, "top_k": w.top_k, "global_batch": w.T * n_gpus,
            "parallelism": f"dp{n_gpus}"}


# --------------------------------------------------------------------------- work model
SMALL_BATCH_MAX_T = 128   # the library streams weights (weights-on-M GEMMs) up to this T


def algorithmic_work(w, active_experts: int | None = None) -> dict:
    """Per-launch algorithmic work of each kernel (selected experts only, no padding).

    Prefill-sized layers: the expert GEMMs are tensor-bound (FLOPs).  Decode-sized layers
    (T <= 128, weights-on-M GEMMs): they are bound by streaming the weights of the experts
    that received tokens (bytes), plus the shared experts.
    """
    es = 2 if w.dtype == "bf16" else 4
    T, d, I, K, ks, nr = w.T, w.d, w.inter, w.top_k, w.n_shared, w.n_routed
    passes = ks + K
    work = {
        "router": ("hbm", T * d * es + nr * d * es + T * K * 12),
        "scan": ("latency", 0),
        "permute": ("hbm", T * d * es + T * K * d * es + T * K * 12),
        "gate_up_gemm": ("tensor", 4.0 * T * d * I * passes),
        "down_gemm": ("tensor", 2.0 * T * d * I * passes),
        "combine": ("hbm", T * d * es * (2 + (1 if ks else 0) + K) + T * K * 8),
    }
    if w.dtype == "bf16" and T <= SMALL_BATCH_MAX_T and d % 128 == 0:
        # one kernel runs both GEMMs (its slot is the gate/up one; the down slot stays empty)
        n = (nr if active_experts is None else active_experts) + ks
        work["gate_up_gemm"] = ("hbm", n * 2 * I * d * es + T * passes * (d + I) * es
                                + n * I * d * es + T * passes * (I + d) * es)
        work["down_gemm"] = ("fused", 0)
    return work


def _code_only(src: str) -> str:
    """C/C++ source without comments and whitespace (comment edits keep the digest)."""
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "".join(src.split())


def csrc_digest() -> str:
    h = hashlib.sha1()
    d = os.path.join(ROOT, "mixture_experts_layer_65_b200", "csrc")
    for f in sorted(os.listdir(d)):
        with open(os.path.join(d, f), encoding="utf-8") as fh:
            h.update(f.encode() + _code_only(fh.read()).encode())
    return h.hexdigest()


def ncu_traffic(kernel: str, config: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernels are unchanged."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        tab = json.load(f)
    if tab.get("csrc_sha1") != csrc_digest():
        return None
    ent = tab.get("kernels", {}).get(config, {}).get(kernel)
    return None if ent is None else float(ent["dram_bytes_per_launch"])


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi's clock, power and throttle-reason samples (every `period_ms`), each
    tagged with nvidia-smi's own timestamp, so that a summary can keep only the samples
    taken inside a measured window."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, period_ms: int = 20, device: int = 0):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(device), f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", str(period_ms)],
                                      stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.p = None

    @staticmethod
    def now() -> datetime.datetime:
        return datetime.datetime.now()

    def stop(self, window: tuple | None = None) -> dict:
        """Summary of the samples inside `window` (two `now()` marks), or of all samples
        when none falls inside it (then "window": "all samples")."""
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        try:
            out = self.p.communicate(timeout=10)[0]
        except subprocess.TimeoutExpired:
            self.p.kill()
            out = self.p.communicate()[0]
        rows = []
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f")
                rows.append((ts, float(f[2]), float(f[3]), float(f[4]), f[6:10]))
            except ValueError:
                continue
        inside = [r for r in rows if window and window[0] <= r[0] <= window[1]]
        use = inside or rows
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in use for n, v in zip(names, r[4]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": max(r[2] for r in use),
                "samples": len(use), "window": "timed window" if inside else "all samples",
                "power_w_max": max(r[3] for r in use), "reasons": reasons}


# --------------------------------------------------------------------------- CPU oracle
def oracle_tokens_per_s(w, seconds: float) -> tuple[float, dict]:
    """Time the fp64 oracle (as it stands) on a bounded token sample of the workload."""
    import numpy as np
    import threadpoolctl

    from oracle import moe_oracle as O

    def run(n):
        t0 = time.perf_counter()
        O.moe_forward(w.u[:n], w.centroids, w.w_gate, w.w_up, w.w_down, w.n_shared, w.top_k,
                      w.alpha1, bias=w.logit_bias, gate_up_e4m3=w.gate_up_e4m3,
                      down_e4m3=w.down_e4m3)
        return time.perf_counter() - t0

    # grow the sample until one call takes about `seconds` (the oracle has a per-call cost
    # for widening the experts it touches, so the rate depends on the sample size)
    n = min(w.T, 64)
    while True:
        dt = run(n)
        if dt >= 0.5 * seconds or n >= w.T:
            break
        n = int(min(w.T, max(2 * n, n * 0.8 * seconds / max(dt, 1e-6))))
    info = threadpoolctl.threadpool_info()
    threads = max([i.get("num_threads", 1) for i in info] or [1])
    desc = {"kind": "oracle", "cores": threads,
            "sample": f"first {n} of {w.T} tokens of the same layer (routing + all experts, fp64 "
                      f"NumPy/{info[0]['internal_api'] if info else 'BLAS'}); {dt:.1f} s",
            "value": n / dt, "unit": "tokens/s"}
    _ = np
    return n / dt, desc


# --------------------------------------------------------------------------- reference arm
def run_reference(args, rank: int, world: int):
    if rank != 0:
        return
    from mixture_experts_layer_65_b200 import workloads as W
    w = W.make_workload(args.config, **({"T": args.tokens} if args.tokens else {}))
    from oracle import moe_oracle as O
    budget = 120.0 / max(1, args.steps + args.warmup)

    t0 = time.perf_counter()
    O.moe_forward(w.u[:16], w.centroids, w.w_gate, w.w_up, w.w_down, w.n_shared, w.top_k,
                  w.alpha1, bias=w.logit_bias, gate_up_e4m3=w.gate_up_e4m3,
                      down_e4m3=w.down_e4m3)
    per_tok = (time.perf_counter() - t0) / 16
    n = int(max(1, min(w.T, budget / max(per_tok, 1e-9))))
    times = []
    for i in range(args.warmup + args.steps):
        s = (i * n) % max(1, w.T - n + 1)
        t0 = time.perf_counter()
        O.moe_forward(w.u[s:s + n], w.centroids, w.w_gate, w.w_up, w.w_down, w.n_shared,
                      w.top_k, w.alpha1, bias=w.logit_bias, gate_up_e4m3=w.gate_up_e4m3,
                      down_e4m3=w.down_e4m3)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    tot = sum(times)
    value = n * len(times) / tot
    import threadpoolctl
    info = threadpoolctl.threadpool_info()
    threads = max([i.get("num_threads", 1) for i in info] or [1])
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tot / len(times), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_desc(w, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": f"{n} tokens per step of the {w.name} layer (fp64 oracle)"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- expert parallel
class _LocalComm:
    """The expert-parallel forward's collectives for a single rank: the row exchange is a copy
    and the sums over ranks are the rank's own values."""

    def all_to_all_single(self, out, inp, out_splits=None, in_splits=None):
        out.copy_(inp)

    def all_reduce(self, t):
        pass


def run_expert_parallel(args, rank: int, world: int, local_rank: int):
    """Tokens/s of the expert-parallel forward (`expert_parallel.ep_forward` over the library's
    moe_ep_* calls): each rank holds n_routed / world routed experts and the shared ones and
    routes its own T tokens; eager launches (the forward reads the exchange's split sizes on
    the host), CUDA-event timing, max over ranks."""
    import torch
    import torch.distributed as dist

    from mixture_experts_layer_65_b200 import workloads as W
    from mixture_experts_layer_65_b200.expert_parallel import (DistComm, ep_forward,
                                                              lib_backend_from_workload)
    from mixture_experts_layer_65_b200.layer import to_device_tensor

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = W.make_workload(args.config, **({"T": args.tokens} if args.tokens else {}))
    if w.dtype != "bf16" or getattr(w, "gate_up_e4m3", False) or w.n_routed % world:
        print(f"bench.py: --expert-parallel takes bf16 layers whose routed experts split evenly "
              f"over the ranks ({w.name}: {w.dtype}, {w.n_routed} routed, {world} ranks)",
              file=sys.stderr)
        sys.exit(2)
    be = lib_backend_from_workload(w, rank, world, device=dev, recv_capacity=w.T * w.top_k * world)
    u = torch.roll(to_device_tensor(w.u, dev), shifts=rank * 997, dims=0).contiguous()
    comm = DistComm() if world > 1 else _LocalComm()
    stream = torch.cuda.current_stream(dev)
    for _ in range(max(3, args.warmup)):
        ep_forward(be, u, comm)
    torch.cuda.synchronize()
    be.device_status()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        ep_forward(be, u, comm)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    be.device_status()
    if world > 1:
        t = torch.tensor([ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    be.close()
    if rank != 0:
        return
    print(json.dumps({
        "mode": "expert_parallel", "metric": METRIC, "value": world * w.T * args.steps / (ms * 1e-3),
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": dict(workload_desc(w, world), parallelism=f"ep{world}"),
        "launch": "eager (the exchange's split sizes are read on the host each step)",
        "collectives": "NCCL all_to_all_single / all_reduce" if world > 1 else "one rank: local copies"}),
        flush=True)


# --------------------------------------------------------------------------- our arm
def run_ours(args, rank: int, world: int, local_rank: int):
    import numpy as np
    import torch
    import torch.distributed as dist

    from mixture_experts_layer_65_b200 import workloads as W
    from mixture_experts_layer_65_b200.layer import MoELayer, to_device_tensor
    from mixture_experts_layer_65_b200.parallel import global_balance_loss, global_token_count

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = W.make_workload(args.config, **({"T": args.tokens} if args.tokens else {}))
    layer = MoELayer.from_workload(w, dev)
    es = 2 if w.dtype == "bf16" else 4
    u_bytes = w.T * w.d * es
    n_buf = int(min(8, max(2, math.ceil(2 * L2_BYTES / u_bytes))))
    base = to_device_tensor(w.u, dev)
    # distinct token batches per rank and per buffer (row rotations of the seeded batch)
    ubufs = [torch.roll(base, shifts=(rank * n_buf + i) * 997, dims=0).contiguous()
             for i in range(n_buf)]
    del base
    out = layer.alloc_outputs()
    if world > 1:
        psum = torch.empty(w.n_routed, dtype=torch.float32, device=dev)
        cnt_g = torch.empty(w.n_routed, dtype=torch.int32, device=dev)
        aux_g = torch.empty(1, dtype=torch.float32, device=dev)
        n_global = global_token_count(w.T, dev)   # once: the per-rank token count is fixed

    stream = torch.cuda.current_stream(dev)
    # one captured CUDA graph per input buffer: the kernel launches of a forward are
    # replayed without host launch overhead (the layer's inputs/outputs stay fixed)
    graphs = None
    if not args.no_graph:
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            for ub in ubufs:
                layer.forward(ub, out)
        stream.wait_stream(side)
        torch.cuda.synchronize()
        graphs = []
        for ub in ubufs:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                layer.forward(ub, out)
            graphs.append(g)
        torch.cuda.synchronize()

    def step(i, eager=False):
        if graphs is not None and not eager:
            graphs[i % n_buf].replay()
        else:
            layer.forward(ubufs[i % n_buf], out)
        if world > 1:   # balance loss of the global batch: all-reduce counts and sums
            global_balance_loss(layer, out, psum, cnt_g, aux_g, n_global=n_global)

    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize()
    layer.device_status()

    def kernel_pass(n):
        # per-kernel durations: CUDA events between the kernels of n eager forwards
        layer.timing_begin(n)
        for i in range(n):
            step(i, eager=True)
        torch.cuda.synchronize()
        return layer.timing_end()

    # Per-kernel durations at the clocks of a short run.  A GPU at ~1 kW reaches its power
    # cap within ~0.1 s of back-to-back forwards, so kernels timed after the timed steps run
    # at lower clocks than a short timed region did: after a pause, a few eager forwards are
    # timed kernel by kernel (with their own clock samples), then another pause.
    burst_kt = None
    if graphs is not None:
        if world > 1:
            dist.barrier()
        ksamp = ClockSampler(period_ms=10, device=local_rank) if rank == 0 else None
        time.sleep(KERNEL_REST_S)
        kt0 = ClockSampler.now()
        km, kn = kernel_pass(min(args.steps, KERNEL_BURST_FORWARDS))
        burst_kt = (km, kn, ksamp.stop((kt0, ClockSampler.now())) if ksamp else None)
        time.sleep(KERNEL_REST_S)
    if world > 1:
        dist.barrier()
    clocks = ClockSampler(device=local_rank) if rank == 0 else None
    time.sleep(0.3 if clocks else 0.0)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if graphs is None:
        layer.timing_begin(args.steps)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_start = ClockSampler.now()
    ev0.record(stream)
    for i in range(args.steps):
        step(i)
    ev1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = ev0.elapsed_time(ev1)
    t_end = ClockSampler.now()
    if graphs is not None:
        # per-kernel durations right after the timed steps (the clock regime a long timed
        # region ends in)
        kernel_ms, n_rec = kernel_pass(min(args.steps, 100))
    else:
        kernel_ms, n_rec = layer.timing_end()
    clk = clocks.stop((t_start, t_end)) if clocks else None
    if world > 1:
        t = torch.tensor([ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    layer.device_status()

    # end to end through the public host-buffer call (pinned host memory): a stream of
    # batches through moe_forward_host_pipelined, which overlaps each step's host->device
    # and device->host copies with the neighbouring steps' forwards
    # (after a pause, so that it starts in the clock regime the timed steps started in; the
    # sustained loop comes after it)
    e2e_ms, e2e_clk = None, None
    if args.e2e_steps > 0:
        u_hosts = [ubufs[i % len(ubufs)].cpu().pin_memory() for i in range(2)]
        host_outs = [layer.host_outputs() for _ in range(2)]
        for i in range(2):
            layer.forward_host_pipelined(u_hosts[i], host_outs[i], stream)
        layer.pipeline_wait(stream)
        torch.cuda.synchronize()
        esamp = ClockSampler(device=local_rank) if rank == 0 else None
        time.sleep(KERNEL_REST_S)
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        et0 = ClockSampler.now()
        e0.record(stream)
        for i in range(args.e2e_steps):
            layer.forward_host_pipelined(u_hosts[i % 2], host_outs[i % 2], stream)
        layer.pipeline_wait(stream)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_clk = esamp.stop((et0, ClockSampler.now())) if esamp else None
        e2e_ms = e0.elapsed_time(e1)
        if world > 1:
            t = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e2e_ms = float(t.item())
        layer.device_status()

    # sustained regime: forwards back to back for about --sustained-seconds, so that the
    # GPU settles under its power cap; reported beside the value with its own clocks
    sustained = None
    if args.sustained_seconds > 0:
        n_sus = max(1, int(args.sustained_seconds / max(ms * 1e-3 / args.steps, 1e-6)))
        if world > 1:
            dist.barrier()
        sampler = ClockSampler(period_ms=100, device=local_rank) if rank == 0 else None
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ts0 = ClockSampler.now()
        s0.record(stream)
        for i in range(n_sus):
            step(i)
        s1.record(stream)
        torch.cuda.synchronize()
        sus_ms = s0.elapsed_time(s1)
        if world > 1:
            t = torch.tensor([sus_ms], dtype=torch.float64, device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            sus_ms = float(t.item())
        sustained = {"value": world * w.T * n_sus / (sus_ms * 1e-3), "unit": "tokens/s",
                     "steps": n_sus, "seconds": sus_ms * 1e-3,
                     "clocks": sampler.stop((ts0, ClockSampler.now())) if sampler else None}
        layer.device_status()

    bwd = None
    if args.backward > 0:
        bwd = time_backward(args, layer, ubufs, out, stream, dev, world, local_rank, rank)

    if rank != 0:
        return
    del graphs
    peaks, peak_src = load_peaks()
    if bwd is not None:
        regime_b = peak_regime(bwd.pop("_clk"), bwd["seconds"])
        peak_b = peaks[PEAK_KEY[regime_b]]
        bwd.update(peak_regime=regime_b, frac=bwd["gemm_tflops"] / peak_b,
                   frac_of_burst=bwd["gemm_tflops"] / peaks["bf16_tflops"],
                   frac_of_sustained=bwd["gemm_tflops"] / peaks["bf16_tflops_sustained"])
    # hold tensor-bound kernels against the peak of the timed region's clock regime, with
    # the kernel durations measured in that regime: the pass before the timed steps for a
    # short (burst-clock) region, the pass right after them for a power-capped one
    regime = peak_regime(clk, ms * 1e-3)
    kernel_ms, n_rec, kernel_clk, timing_desc = choose_kernel_timing(
        regime, args.no_graph, burst_kt, (kernel_ms, n_rec, clk))
    work = algorithmic_work(w, int((out.expert_counts > 0).sum().item()))
    per_kernel = {}
    # e4m3 gate/up variant: that GEMM's peak is the measured bf16 peak times the nominal
    # dense e4m3 : bf16 ratio (4.5 : 2.25 PFLOP/s), and the token rows are quantised (one
    # extra kernel, timed in the permute slot)
    e4m3 = bool(getattr(w, "gate_up_e4m3", False))
    e4m3_down = bool(getattr(w, "down_e4m3", False))
    tensor_ratio = {k: (2.0 if ((e4m3 and k == "gate_up_gemm") or (e4m3_down and k == "down_gemm"))
                        else 1.0) for k in KERNELS}
    if e4m3:
        work["permute"] = ("hbm", w.T * w.d * 3 + w.T * 4)   # quantise: bf16 in, e4m3 + scale out
    # with a shared group the paired bf16 GEMM copies the routed rows itself (its copy
    # warps run beside the shared group's tiles), and so does the decode-sized gate/up GEMM
    # (its epilogue warps, after the scan has placed the rows): no permute kernel is launched
    fused_permute = (layer.kernels_per_forward - (1 if e4m3 else 0) -
                     ((1 + (w.n_shared > 0)) if e4m3_down else 0)) <= len(KERNELS) - 1
    for k in KERNELS:
        kind, amount = work[k]
        avg_ms = kernel_ms[k] / max(1, n_rec)
        ent = {"avg_ms": avg_ms, "share": kernel_ms[k] / max(1e-12, sum(kernel_ms.values()))}
        if kind == "fused":
            ent.update(fused_into="gate_up_gemm (one decode FFN kernel runs both GEMMs)")
        elif k == "permute" and fused_permute and not e4m3:
            # paired path: the gate/up GEMM's copy warps; decode-sized layers: the scan places
            # the rows and the gate/up GEMM's epilogue warps copy them
            ent.update(fused_into="gate_up_gemm" if w.T > 128 else "scan + gate_up_gemm")
        elif kind == "tensor":
            ach = amount / (avg_ms * 1e-3) / 1e12
            ent.update(bound="tensor", achieved=ach, unit="TFLOP/s",
                       frac=ach / (tensor_ratio[k] * peaks[PEAK_KEY[regime]]),
                       frac_of_burst=ach / (tensor_ratio[k] * peaks["bf16_tflops"]),
                       frac_of_sustained=ach / (tensor_ratio[k] * peaks["bf16_tflops_sustained"]))
            if tensor_ratio[k] != 1.0:
                ent.update(operands="e4m3", peak_note="measured bf16 peak x 2 (nominal dense e4m3/bf16)")
            if k == "down_gemm" and e4m3_down:
                ent.update(slot_includes="the activations' e4m3 quantisation before the GEMM")
        elif kind == "hbm":
            ach = amount / (avg_ms * 1e-3) / 1e9
            ent.update(bound="hbm", achieved=ach, unit="GB/s", frac=ach / peaks["hbm_gbs"])
        per_kernel[k] = ent
    dominant = max(KERNELS, key=lambda k: kernel_ms[k])
    dk = per_kernel[dominant]
    bound = dk.get("bound", "latency")
    tensor_peak = f"bf16 {regime}" + ("" if tensor_ratio[dominant] == 1.0 else " x 2 for e4m3 operands")
    roofline = {"kernel": dominant, "bound": bound, "achieved": dk.get("achieved"),
                "peak": (tensor_ratio[dominant] * peaks[PEAK_KEY[regime]] if bound == "tensor"
                         else peaks["hbm_gbs"]),
                "unit": dk.get("unit"), "frac": dk.get("frac"),
                "peak_source": f"{peak_src} ({'HBM copy' if bound != 'tensor' else tensor_peak}; "
                               f"clock regime of the kernel timing: {regime})",
                "traffic": ncu_traffic(dominant, w.name), "algorithmic_per_launch": work[dominant][1]}
    # a kernel held against a plain copy or cuBLAS can read a little above 1; far above
    # means the timed kernel is not doing the work it is credited with
    roofline["frac_le_1"] = bool(roofline["frac"] is None or roofline["frac"] <= 1.0)
    if not roofline["frac_le_1"]:
        print(f"bench.py: warning: roofline frac {roofline['frac']:.3f} > 1 for {dominant}",
              file=sys.stderr)
    gemm_flops = 6.0 * w.T * w.d * w.inter * (w.n_shared + w.top_k)
    gemm_ms = (kernel_ms["gate_up_gemm"] + kernel_ms["down_gemm"]) / max(1, n_rec)
    gemm_tflops = gemm_flops / (gemm_ms * 1e-3) / 1e12
    # fraction of peak = time at peak / measured time (each GEMM at its operands' peak)
    ideal = {key: sum(work[k][1] / (tensor_ratio[k] * peaks[key] * 1e12)
                      for k in ("gate_up_gemm", "down_gemm"))
             for key in ("bf16_tflops_sustained", "bf16_tflops")}
    value = world * w.T * args.steps / (ms * 1e-3)
    tk = w.T * w.top_k
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": ("bf16 (expert GEMMs on e4m3 operands)" if e4m3_down else
                  "bf16 (gate/up GEMM on e4m3 operands)" if e4m3 else w.dtype),
        "data": "synthetic (seeded N(0,1) tokens, N(0,0.02) random-init experts, no trained weights)",
        "config": dict(workload_desc(w, world),
                       l2=f"inputs rotate over {n_buf} token buffers "
                          f"({n_buf * u_bytes / 2**20:.0f} MiB > 126 MiB L2); expert weights "
                          f"{layer.device_bytes / 2**30:.2f} GiB with workspace"),
        "expert_gemm_tflops": gemm_tflops,
        "expert_gemm_frac_of_peak": ideal[PEAK_KEY[regime]] / (gemm_ms * 1e-3),
        "expert_gemm_peak_regime": regime,
        "expert_gemm_frac_of_burst_peak": ideal["bf16_tflops"] / (gemm_ms * 1e-3),
        "expert_gemm_frac_of_sustained_peak": ideal["bf16_tflops_sustained"] / (gemm_ms * 1e-3),
        "roofline": roofline,
        "kernels": per_kernel,
        "e2e": None if e2e_ms is None else {
            "value": world * w.T * args.e2e_steps / (e2e_ms * 1e-3), "unit": "tokens/s",
            "h2d_bytes_per_step": u_bytes, "d2h_bytes_per_step": u_bytes + tk * 8 + w.n_routed * 4 + 4,
            "api": "moe_forward_host_pipelined (two steps in flight), then moe_pipeline_wait",
            "clocks": e2e_clk},
        "gpu_launches": args.steps * (layer.kernels_per_forward + (1 if world > 1 else 0)),
        "launch": "eager" if args.no_graph else "CUDA graph replay (one graph per input buffer)",
        "kernel_timing": timing_desc,
        "kernel_timing_clocks": kernel_clk,
        "clocks": clk,
        "sustained": sustained,
    }
    if bwd is not None:
        line["backward"] = bwd
    if world == 1 and not args.no_cpu_baseline:
        _, desc = oracle_tokens_per_s(w, args.cpu_seconds)
        line["cpu_baseline"] = desc
    print(json.dumps(line), flush=True)


def time_backward(args, layer, ubufs, out, stream, dev, world, local_rank, rank):
    """K forward + backward steps (eager forwards: the captured graphs predate the backward's
    bookkeeping), each on the next token buffer with a fixed seeded upstream gradient dh and
    d_aux = 1; CUDA events on the launching stream around each backward and around the
    whole loop, max over ranks.  The backward's GEMM work is 16·T·d·I·(K_s + K') FLOPs:
    dHmid (2), the recomputed gate/up (4), dX (4), dW_gate/up (4) and dW_down (2), selected
    experts only; the router's dl·e GEMM and the SIMT kernels are not counted."""
    import torch
    import torch.distributed as dist

    layer.backward_prepare()
    g = torch.Generator(device=dev).manual_seed(1234 + rank)
    dh = (torch.randn(layer.T, layer.d, device=dev, generator=g) * 0.01).to(layer.torch_dtype)
    n_buf = len(ubufs)

    def one(i, evs=None):
        layer.forward(ubufs[i % n_buf], out)
        if evs is not None:
            evs[0].record(stream)
        grads = layer.backward(ubufs[i % n_buf], out, dh, d_aux=1.0)
        if evs is not None:
            evs[1].record(stream)
        return grads

    for i in range(3):
        one(i)
    torch.cuda.synchronize()
    layer.device_status()
    if world > 1:
        dist.barrier()
    k = args.backward
    clocks = ClockSampler(device=local_rank) if rank == 0 else None
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(k)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ts = ClockSampler.now()
    t0.record(stream)
    for i in range(k):
        one(i, evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop((ts, ClockSampler.now())) if clocks else None
    total_ms = t0.elapsed_time(t1)
    bwd_ms = sum(a.elapsed_time(b) for a, b in evs)
    if world > 1:
        t = torch.tensor([total_ms, bwd_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms, bwd_ms = (float(x) for x in t.tolist())
    layer.device_status()
    flops = 16.0 * layer.T * layer.d * layer.inter * (layer.n_shared + layer.top_k)
    return {"steps": k, "seconds": total_ms * 1e-3,
            "fwd_bwd_ms_per_step": total_ms / k, "bwd_ms_per_step": bwd_ms / k,
            "fwd_bwd_tokens_per_s": world * layer.T * k / (total_ms * 1e-3),
            "bwd_gemm_tflop_per_step": flops / 1e12,
            "gemm_tflops": flops / (bwd_ms / k * 1e-3) / 1e12,
            "gradients": "du, d_centroids, d_bias, d_w_gate, d_w_up, d_w_down (fp32)",
            "timing": "CUDA events around each backward call (eager forwards in between)",
            "clocks": clk, "_clk": clk}


def relaunch_under_torchrun(args) -> int:
    """`--gpus N` (N > 1) outside a launcher: start N ranks of this script with torchrun,
    one process per GPU, rendezvous on 127.0.0.1; returns their exit status."""
    import socket
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={args.gpus}", "--master-addr", "127.0.0.1",
           f"--master-port={port}", os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def run_dry(args, rank: int, world: int):
    """The multi-rank plumbing on CPU (gloo): every rank makes synthetic per-expert counts
    and affinity sums for its T tokens (seeded by its rank), the global balance loss runs
    through the same host logic as a GPU run (parallel.global_balance_loss, here with the
    loss formula on the CPU), the exchange is timed as the max over ranks, and rank 0
    prints one line with value null."""
    import types

    import numpy as np
    import torch
    import torch.distributed as dist

    from mixture_experts_layer_65_b200 import workloads as W
    from mixture_experts_layer_65_b200.parallel import global_balance_loss, global_token_count

    spec = dict(W.CONFIGS[args.config])
    T, nr, K, alpha1 = int(spec["T"]), int(spec["n_routed"]), int(spec["top_k"]), float(spec["alpha1"])
    rng = np.random.default_rng(rank)
    counts = torch.from_numpy(rng.multinomial(T * K, np.full(nr, 1.0 / nr)).astype(np.int32))
    psum = torch.from_numpy((rng.dirichlet(np.ones(nr)) * T).astype(np.float32))
    layer = types.SimpleNamespace(T=T, alpha1=alpha1, expert_psum=lambda buf: buf.copy_(psum))
    out = types.SimpleNamespace(expert_counts=counts)

    def cpu_loss(c, p, n, a, o):
        o.fill_(a * float(((c.double() / n) * (p.double() / n)).sum()))
        return o

    cnt_g, psum_g, aux_g = torch.empty_like(counts), torch.empty_like(psum), torch.empty(1)
    n_global = global_token_count(T, "cpu")
    for _ in range(max(3, args.warmup)):
        global_balance_loss(layer, out, psum_g, cnt_g, aux_g, n_global=n_global, loss_fn=cpu_loss)
    dist.barrier()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        global_balance_loss(layer, out, psum_g, cnt_g, aux_g, n_global=n_global, loss_fn=cpu_loss)
    dt = torch.tensor([time.perf_counter() - t0], dtype=torch.float64)
    dist.all_reduce(dt, op=dist.ReduceOp.MAX)
    if rank == 0:
        print(json.dumps({"metric": METRIC, "value": None, "unit": "tokens/s", "n_gpus": world,
                          "steps": args.steps, "warmup": max(3, args.warmup),
                          "ms_per_step": 1e3 * float(dt.item()) / max(1, args.steps),
                          "dry_run": True, "backend": "gloo", "global_tokens": n_global,
                          "aux_loss": float(aux_g.item()),
                          "config": {"workload": args.config, "parallelism": f"dp{world}"}}),
              flush=True)


def main():
    args = parse_args()
    env_world = os.environ.get("WORLD_SIZE")
    if env_world is None and args.gpus > 1:
        sys.exit(relaunch_under_torchrun(args))
    world = int(env_world or "1")
    if world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but the launcher started {world} ranks "
              "(WORLD_SIZE); they must agree", file=sys.stderr)
        sys.exit(2)
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    import torch.distributed as dist
    if args.dry_run:
        if world > 1:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
        try:
            if world > 1:
                run_dry(args, rank, world)
            else:
                print(json.dumps({"metric": METRIC, "value": None, "n_gpus": 1, "dry_run": True}))
        finally:
            if world > 1:
                dist.destroy_process_group()
        return
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=None)
    try:
        if args.expert_parallel:
            run_expert_parallel(args, rank, world, local_rank)
        else:
            run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
