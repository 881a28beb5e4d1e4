#!/usr/bin/env python
"""Throughput of the gated delta-rule layer on B200; prints ONE JSON line on rank 0.

Headline workload (the metric's decode configuration): 64 independent sequences, one token
each per step, Qwen3-Next layer shape (H_k=16 key heads -> H_v=32 value heads, d_k=d_v=128),
fp32 recurrent state per slot, bf16 x / conv state / output. One step = gdn_conv_step +
gdn_decode_step over the 64 tokens. Also measured in the same run and reported under
"prefill": B=1, T=4096 chunked prefill through gdn_layer_prefill (the front inside the
prefill's first kernel, chunk 64), with the two-call path (gdn_conv_step +
gdn_chunked_prefill) timed beside it.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]

With N > 1 (torchrun, one process per GPU) every rank runs an independent replica of the
workload (the layer has no exchange step); value = tokens of all ranks / max-over-ranks time.
--impl reference times the fp64 CPU oracle on the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDN tokens/s (decode, prefill) on 1 B200; % of HBM / tensor roofline"
UNIT = "tokens/s"
N_SEQS = 64
X_STEPS = 256          # distinct synthetic decode inputs (the workload's 256 steps)
PREFILL_T = 4096
L2_BYTES = 126 * 1024 * 1024

# Algorithmic bytes per decoded token for the decode kernel (gdn_decode_step):
# fp32 state read + write (32 heads x 128 x 128 x 4 B x 2), fp32 q,k (2 x 16 x 128 x 4),
# fp32 v (32 x 128 x 4), g and beta (2 x 32 x 4), bf16 o (32 x 128 x 2).
DECODE_KERNEL_BYTES_PER_TOKEN = 4_194_304 + 16_384 + 16_384 + 256 + 8_192
# Whole decode step per token: state r+w + bf16 conv state r+w (2 x 3 x 8192 x 2) + bf16 x
# (8192 x 2) + a,b (2 x 32 x 4) + bf16 o.
DECODE_STEP_BYTES_PER_TOKEN = 4_194_304 + 98_304 + 16_384 + 256 + 8_192
# Chunked prefill, B=1, T=4096: bf16 x + a,b + conv w + bf16 o + final fp32 state + conv
# state; FLOPs per (chunk, head) = 5 * 2 C^2 d + 3 * 2 C d^2 + C^3 / 3 with C=64, d=128.
PREFILL_STEP_BYTES = 67_108_864 + 1_048_576 + 131_072 + 33_554_432 + 2_097_152 + 49_152
PREFILL_FLOP_PER_CHUNK_HEAD = 5 * 2 * 64 * 64 * 128 + 3 * 2 * 64 * 128 * 128 + 64 ** 3 // 3


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=256)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--prefill-iters", type=int, default=20)
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


# ---------------------------------------------------------------------------- helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                source="fallback")


def kernel_source_hash(files):
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, "gated_deltanet_linear_19_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, files):
    """DRAM bytes per launch from the committed ncu summary, if the kernel is unchanged."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(kernel)
    if not d or d.get("src_sha256_16") != kernel_source_hash(files):
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.002):
        self.samples, self.reasons, self.ok = [], set(), False
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.ok:
            self._t.join()

    def summary(self, others=()):
        s = list(self.samples)
        for o in others:
            s += o.samples
        reasons = set(self.reasons)
        for o in others:
            reasons |= o.reasons
        return {"sm_mhz": (statistics.median(s) if s else None), "sm_max_mhz": self.max_mhz,
                "samples": len(s), "reasons": sorted(reasons - {"gpu_idle"})}


# ---------------------------------------------------------------------------- replicas

def reduce_max(x: float, world: int, device) -> float:
    """Max of a per-rank number over all ranks (the job time is the slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, world: int, total_ms: float) -> float:
    """Whole-job units per second: every rank runs an independent replica of the workload."""
    return world * units_per_rank / (total_ms * 1e-3)


# ---------------------------------------------------------------------------- reference arm

def run_reference(args):
    import oracle
    import synthetic
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = synthetic.decode(steps=max(1, min(X_STEPS, args.steps + args.warmup)))
    threads = oracle.default_threads()
    # bound the run to a few minutes: estimate one step, then sample sequences if needed
    t0 = time.perf_counter()
    oracle.decode_steps(dict(w, slot_ids=w["slot_ids"][:8], x=w["x"][:1, :8], a=w["a"][:1, :8],
                             b=w["b"][:1, :8]), 1, threads=threads)
    per_seq = (time.perf_counter() - t0) / 8
    budget = 150.0
    n_sample = int(max(1, min(N_SEQS, budget / max(per_seq * (args.steps + args.warmup), 1e-9))))
    ws = dict(w, slot_ids=w["slot_ids"][:n_sample])
    nx = w["x"].shape[0]
    S = None
    cst = None
    dtimes = []

    def step(s, S, cst):
        ws_s = dict(ws, x=w["x"][s % nx:s % nx + 1, :n_sample], a=w["a"][s % nx:s % nx + 1, :n_sample],
                    b=w["b"][s % nx:s % nx + 1, :n_sample])
        r = oracle.decode_steps(ws_s, 1, threads=threads, S0=S, conv_state0=cst)
        return r["S"], r["conv_state"]

    for s in range(args.warmup):
        S, cst = step(s, S, cst)
    t0 = time.perf_counter()
    for s in range(args.steps):
        S, cst = step(args.warmup + s, S, cst)
    dt = time.perf_counter() - t0
    value = n_sample * args.steps / dt
    sample = (f"{args.steps} decode steps x {n_sample} of {N_SEQS} sequences, all 32 heads, "
              "fp64 oracle (front + per-token recurrence)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "decode: 64 seqs x 1 token/step, Qwen3-Next GDN layer "
                                   "(H_k=16->H_v=32, d=128), fp32 state",
                       "n_seqs": N_SEQS},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------- our arm

def cpu_baseline(seconds: float):
    """fp64 oracle decode steps on the host cores for about `seconds` (rank 0, N=1 only)."""
    import oracle
    import synthetic
    w = synthetic.decode(steps=64)
    threads = oracle.default_threads()
    S = cst = None
    steps = 0
    t0 = time.perf_counter()
    while True:
        ws = dict(w, x=w["x"][steps:steps + 1], a=w["a"][steps:steps + 1],
                  b=w["b"][steps:steps + 1])
        r = oracle.decode_steps(ws, 1, threads=threads, S0=S, conv_state0=cst)
        S, cst = r["S"], r["conv_state"]
        steps += 1
        dt = time.perf_counter() - t0
        if dt >= seconds or steps >= w["x"].shape[0]:
            break
    return {"value": N_SEQS * steps / dt, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{steps} decode steps x {N_SEQS} sequences x 32 heads (fp64 oracle, "
                      f"{dt:.1f} s)"}


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    import synthetic
    import gated_deltanet_linear_19_b200 as gdn
    from gated_deltanet_linear_19_b200.layer import GDNLayer

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x: float) -> float:
        return reduce_max(x, world, dev)

    peaks = load_peaks()
    # ------------------------------------------------------------------ decode workload
    w = synthetic.decode(seed=synthetic.SEED_BASE + 1 + 1000 * rank, steps=X_STEPS)
    d = w["dims"]
    dims = gdn.Dims(n_slots=d["n_slots"], H_k=d["H_k"], H_v=d["H_v"], d_k=d["d_k"],
                    d_v=d["d_v"], d_conv=d["d_conv"])
    layer = GDNLayer(dims, torch.from_numpy(w["conv_w"]), torch.from_numpy(w["A_log"]),
                     torch.from_numpy(w["dt_bias"]), eps=w["eps"], q_scale=w["q_scale"],
                     device=dev)
    layer.state.copy_(torch.from_numpy(w["state"]))
    layer.conv_state.copy_(torch.from_numpy(w["conv_state"]).view(torch.bfloat16))
    x_all = torch.from_numpy(w["x"]).view(torch.bfloat16).to(dev)
    a_all = torch.from_numpy(w["a"]).to(dev)
    b_all = torch.from_numpy(w["b"]).to(dev)
    slots = torch.from_numpy(w["slot_ids"]).to(dev)
    cu = torch.arange(N_SEQS + 1, dtype=torch.int32, device=dev)
    q, k, v, g, beta = gdn.front_outputs(dims, N_SEQS, torch.float32, dev)
    o = torch.empty((N_SEQS, dims.H_v, dims.d_v), dtype=torch.bfloat16, device=dev)

    def front(s):
        gdn.conv_step(dims, x_all[s % X_STEPS], layer.conv_w, layer.conv_state, cu, slots,
                      a_all[s % X_STEPS], b_all[s % X_STEPS], layer.A_log, layer.dt_bias,
                      q, k, v, g, beta, eps=layer.eps, q_scale=layer.q_scale)

    def core():
        gdn.decode_step(dims, q, k, v, g, beta, layer.state, slots, o)

    dec_ws = torch.empty(gdn.decode_workspace_size(dims, N_SEQS), dtype=torch.uint8, device=dev)

    def layer_step(s):
        # the timed step: gdn_layer_decode (front, then the decode kernel, which streams the
        # state in while the front runs)
        gdn.layer_decode(dims, x_all[s % X_STEPS], layer.conv_w, layer.conv_state, slots,
                         a_all[s % X_STEPS], b_all[s % X_STEPS], layer.A_log, layer.dt_bias,
                         layer.state, o, eps=layer.eps, q_scale=layer.q_scale, workspace=dec_ws)

    K, W = args.steps, args.warmup
    for s in range(W):
        layer_step(s)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    # (a) the dominant kernel's own duration: an eager pass of K steps with events around
    # every gdn_decode_step launch (the events also keep front and decode from overlapping)
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    for s in range(K):
        front(W + s)
        ev0[s].record()
        core()
        ev1[s].record()
    torch.cuda.synchronize()
    dec_ms = [a.elapsed_time(b) for a, b in zip(ev0, ev1)]
    dec_kernel_ms = statistics.mean(dec_ms)
    # (b) the timed region: K steps (gdn_layer_decode each: front + decode) captured in one
    # CUDA graph, so the host adds no gaps; the front lets the decode grid start early
    # (programmatic launch)
    graph = torch.cuda.CUDAGraph()
    cap_stream = torch.cuda.Stream()
    cap_stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap_stream):
        with torch.cuda.graph(graph, stream=cap_stream):
            for s in range(K):
                layer_step(W + K + s)
    torch.cuda.current_stream().wait_stream(cap_stream)
    graph.replay()  # warm replay (untimed)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk_dec:
        start.record()
        graph.replay()
        end.record()
        torch.cuda.synchronize()
    barrier()
    total_ms = max_over_ranks(start.elapsed_time(end))
    del graph
    value = job_throughput(N_SEQS * K, world, total_ms)
    launches = 2 * K

    # ------------------------------------------------------------------ e2e through the API
    # each step's inputs x | a | b packed in one pinned host row, moved by one H2D copy into
    # one device buffer that the decode call sees as three tensors
    x_bytes = N_SEQS * dims.conv_dim * 2
    ab_bytes = N_SEQS * dims.H_v * 4
    step_bytes = x_bytes + 2 * ab_bytes
    packed_h = torch.empty((X_STEPS, step_bytes), dtype=torch.uint8).pin_memory()
    for i in range(X_STEPS):
        packed_h[i, :x_bytes] = torch.from_numpy(w["x"][i]).view(torch.uint8).reshape(-1)
        packed_h[i, x_bytes:x_bytes + ab_bytes] = \
            torch.from_numpy(np.ascontiguousarray(w["a"][i], np.float32)).view(torch.uint8).reshape(-1)
        packed_h[i, x_bytes + ab_bytes:] = \
            torch.from_numpy(np.ascontiguousarray(w["b"][i], np.float32)).view(torch.uint8).reshape(-1)
    packed_d = torch.empty(step_bytes, dtype=torch.uint8, device=dev)
    xs = packed_d[:x_bytes].view(torch.bfloat16).view(N_SEQS, dims.conv_dim)
    as_ = packed_d[x_bytes:x_bytes + ab_bytes].view(torch.float32).view(N_SEQS, dims.H_v)
    bs = packed_d[x_bytes + ab_bytes:].view(torch.float32).view(N_SEQS, dims.H_v)
    o_h = torch.empty((N_SEQS, dims.H_v, dims.d_v), dtype=torch.bfloat16).pin_memory()

    def e2e_step(s):
        i = s % X_STEPS
        packed_d.copy_(packed_h[i], non_blocking=True)
        out = layer.decode(xs, as_, bs, slots)
        o_h.copy_(out, non_blocking=True)

    for s in range(W):
        e2e_step(s)
    torch.cuda.synchronize()
    barrier()
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    e_start.record()
    for s in range(K):
        e2e_step(W + s)
    e_end.record()
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end))
    h2d = step_bytes
    d2h = o_h.numel() * 2
    e2e = {"value": job_throughput(N_SEQS * K, world, e2e_ms), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    assert gdn.device_status() == 0

    dec_bytes = DECODE_KERNEL_BYTES_PER_TOKEN * N_SEQS
    achieved = dec_bytes / (dec_kernel_ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"],
                "traffic": ncu_traffic("decode", ["decode.cu", "gdn_common.cuh"]),
                "kernel": "decode_kernel", "algorithmic_bytes_per_launch": dec_bytes,
                "kernel_ms_avg": dec_kernel_ms, "kernel_timing": "CUDA events around each "
                "gdn_decode_step launch in an eager pass of the same K steps",
                "peak_source": peaks["source"]}
    step_bytes = DECODE_STEP_BYTES_PER_TOKEN * N_SEQS
    step_gbs = step_bytes / (total_ms / K * 1e-3) / 1e9

    # ------------------------------------------------------------------ prefill workload
    prefill = None
    clk_pf = None
    if not args.no_prefill:
        del x_all, packed_h
        pw = synthetic.prefill(seed=synthetic.SEED_BASE + 2 + 1000 * rank, T=PREFILL_T)
        pl = GDNLayer(dims, torch.from_numpy(pw["conv_w"]), torch.from_numpy(pw["A_log"]),
                      torch.from_numpy(pw["dt_bias"]), eps=pw["eps"], q_scale=pw["q_scale"],
                      device=dev)
        px = torch.from_numpy(pw["x"]).view(torch.bfloat16).to(dev)
        pa = torch.from_numpy(pw["a"]).to(dev)
        pb = torch.from_numpy(pw["b"]).to(dev)
        pcu = torch.from_numpy(pw["cu_seqlens"]).to(dev)
        pslots = torch.from_numpy(pw["slot_ids"]).to(dev)
        preset = torch.ones(1, dtype=torch.uint8, device=dev)
        fq, fk, fv, fg, fb = gdn.front_outputs(dims, PREFILL_T, pl.prefill_qkv_dtype, dev)
        po = torch.empty((PREFILL_T, dims.H_v, dims.d_v), dtype=torch.bfloat16, device=dev)
        need = gdn.prefill_workspace_size(dims, PREFILL_T, 1, 64, pl.prefill_qkv_dtype)
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
        flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

        def pf_front():
            gdn.conv_step(dims, px, pl.conv_w, pl.conv_state, pcu, pslots, pa, pb, pl.A_log,
                          pl.dt_bias, fq, fk, fv, fg, fb, eps=pl.eps, q_scale=pl.q_scale,
                          reset=preset)

        def pf_core():
            gdn.chunked_prefill(dims, fq, fk, fv, fg, fb, pl.state, pslots, pcu, po, chunk=64,
                                reset=preset, workspace=ws if need else None)

        def pf_layer():
            # the timed prefill: gdn_layer_prefill, the front inside the prep kernel
            gdn.layer_prefill(dims, px, pl.conv_w, pl.conv_state, pcu, pslots, pa, pb, pl.A_log,
                              pl.dt_bias, pl.state, po, eps=pl.eps, q_scale=pl.q_scale,
                              chunk=64, reset=preset, workspace=ws)

        for _ in range(3):
            pf_layer()
            pf_front()
            pf_core()
        torch.cuda.synchronize()
        assert gdn.device_status() == 0
        n = args.prefill_iters
        e = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
        e2 = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n)]
        barrier()
        with ClockSampler(local) as clk_pf:
            for i in range(n):
                flush.zero_()                   # evict L2 between iterations
                e[i][0].record()
                pf_layer()
                e[i][1].record()
            for i in range(n):                  # the two-call path, for comparison
                flush.zero_()
                e2[i][0].record()
                pf_front()
                e2[i][1].record()
                pf_core()
                e2[i][2].record()
            torch.cuda.synchronize()
        barrier()
        step_ms = max_over_ranks(statistics.mean(a[0].elapsed_time(a[1]) for a in e))
        two_call_ms = statistics.mean(a[0].elapsed_time(a[2]) for a in e2)
        core_ms = statistics.mean(a[1].elapsed_time(a[2]) for a in e2)
        front_ms = statistics.mean(a[0].elapsed_time(a[1]) for a in e2)
        flops = PREFILL_FLOP_PER_CHUNK_HEAD * (PREFILL_T // 64) * dims.H_v
        t_hbm = PREFILL_STEP_BYTES / (peaks["hbm_gbs"] * 1e9)
        t_tc = flops / (peaks["bf16_tflops"] * 1e12)
        bound = "hbm" if t_hbm >= t_tc else "tensor"
        t_roof = max(t_hbm, t_tc)
        prefill = {
            "workload": "chunked prefill B=1, T=4096, Qwen3-Next GDN layer (H_k=16->H_v=32, "
                        "d=128), chunk 64, bf16 x -> conv/SiLU/L2 (fp16 operands) -> bf16 o, "
                        "fp32 state; L2 flushed between iterations",
            "path": "gdn_layer_prefill (front inside the prep kernel; prep + scan launches)",
            "value": job_throughput(PREFILL_T, world, step_ms), "unit": UNIT,
            "ms_per_step": step_ms,
            "two_call_path": {"ms_per_step": two_call_ms, "front_ms": front_ms,
                              "core_ms": core_ms,
                              "calls": "gdn_conv_step + gdn_chunked_prefill"},
            "roofline": {"bound": bound, "t_roofline_us": t_roof * 1e6,
                         "frac": t_roof / (step_ms * 1e-3),
                         "hbm_gbs_achieved": PREFILL_STEP_BYTES / (step_ms * 1e-3) / 1e9,
                         "tflops_achieved": flops / (step_ms * 1e-3) / 1e12,
                         "algorithmic_bytes": PREFILL_STEP_BYTES, "algorithmic_flops": flops,
                         "peaks": {"hbm_gbs": peaks["hbm_gbs"],
                                   "bf16_tflops": peaks["bf16_tflops"]}},
            "gpu_launches": 2 * n,  # prep (with the front), scan
        }
        launches_pf = 2 * n

    clocks = clk_dec.summary([clk_pf] if clk_pf is not None else [])
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": "decode: 64 seqs x 1 token/step, Qwen3-Next GDN layer "
                               "(H_k=16->H_v=32, d_k=d_v=128), fp32 state, bf16 x/conv/o; "
                               "step = gdn_layer_decode (front + decode step)",
                   "n_seqs": N_SEQS, "global_batch": world * N_SEQS, "seq_len": 1,
                   "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (128 MiB fp32 state pool per rank)",
                   "timed_region": "K steps replayed from one CUDA graph"},
        "roofline": roofline,
        "step_hbm_gbs": step_gbs,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
        "prefill": prefill,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
