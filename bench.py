#!/usr/bin/env python
"""Throughput of the gated delta-rule layer on B200; prints ONE JSON line on rank 0.

Headline workload (the metric's decode configuration): 64 independent sequences, one token
each per step, Qwen3-Next layer shape (H_k=16 key heads -> H_v=32 value heads, d_k=d_v=128),
fp32 recurrent state per slot, bf16 x / conv state / output. One step = gdn_layer_decode
(the front, then the single-token step) over the 64 tokens. Also measured in the same run:
"prefill" (and "prefill_roofline"): B=1, T=4096 chunked prefill through gdn_layer_prefill
(chunk 64), with the two-call path (gdn_conv_step + gdn_chunked_prefill) timed beside it;
"varlen_prefill": 16 packed sequences of lengths U[128, 8192] with non-contiguous slots and
nonzero initial states; "long_context": 4 x 65536 prefill from zero states, then 512 decode
steps at batch 4; "cpu_baseline" / "cpu_baseline_prefill": the fp64 oracle on the host.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]
  python bench.py --profile-run NAME   (one workload, untimed, for profiler captures)

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
# Any packed prefill at the Qwen3-Next layer shape: per token bf16 x (8192 x 2) + a, b
# (2 x 32 x 4) + bf16 o (32 x 128 x 2); per sequence the fp32 state (2 MiB) written, and read
# unless the sequence is reset, the bf16 conv state (3 x 8192 x 2) likewise; once the conv
# weights (8192 x 4 x 4). For B=1, T=4096 with reset this is PREFILL_STEP_BYTES.
PF_BYTES_PER_TOKEN = 16_384 + 256 + 8_192
PF_STATE_BYTES = 2_097_152
PF_CONV_BYTES = 49_152
PF_WEIGHT_BYTES = 131_072


def prefill_algorithmic(lengths, reset: bool, H_v: int = 32):
    """Algorithmic bytes and FLOPs of one packed prefill call (sequence lengths, reset flag)."""
    T = sum(lengths)
    per_seq = (PF_STATE_BYTES + PF_CONV_BYTES) * (1 if reset else 2)
    nbytes = T * PF_BYTES_PER_TOKEN + len(lengths) * per_seq + PF_WEIGHT_BYTES
    chunks = sum((L + 63) // 64 for L in lengths)
    return nbytes, PREFILL_FLOP_PER_CHUNK_HEAD * chunks * H_v


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
    ap.add_argument("--no-varlen", action="store_true", help="skip the 16-sequence varlen prefill")
    ap.add_argument("--no-long", action="store_true",
                    help="skip the 4 x 65536 prefill and its 512 decode steps")
    ap.add_argument("--no-next", action="store_true",
                    help="skip the gated decode, multi-token and mixed-batch measurements")
    ap.add_argument("--profile-run", choices=PROFILE_RUNS, default=None,
                    help="run one workload a few times, untimed, and exit (a small, bounded "
                         "command for profiler captures of its kernels)")
    return ap.parse_args()


# workload -> (what runs); each fits in well under 1 GB of device memory
PROFILE_RUNS = {
    "decode64": "4 layer-decode steps of 64 sequences (front kernel + decode kernel)",
    "decode4": "4 layer-decode steps of 4 sequences (the one-kernel layer decode)",
    "prefill4096": "2 layer prefills, B=1, T=4096 (prep + tile scan)",
    "prefill4096_head": "2 layer prefills, B=1, T=4096, with the whole-head scan",
    "multitoken": "2 layer prefills of 64 sequences x 4 tokens (front of the short sequences, "
                  "token-by-token kernel)",
}


def profile_run(name: str) -> int:
    import torch

    import synthetic
    import gated_deltanet_linear_19_b200 as gdn
    from gated_deltanet_linear_19_b200.layer import GDNLayer

    dev = torch.device("cuda", 0)
    if name.startswith("decode"):
        B = 64 if name == "decode64" else 4
        w = synthetic.decode(steps=4, n_seqs=B)
    elif name == "multitoken":
        w = synthetic.packed([4] * 64, synthetic.SEED_BASE + 60, slots=list(range(64)),
                             state_std=0.02, conv_std=1.0, n_slots=64)
    else:
        w = synthetic.prefill(T=PREFILL_T)
    d = w["dims"]
    dims = gdn.Dims(n_slots=d["n_slots"], H_k=d["H_k"], H_v=d["H_v"], d_k=d["d_k"],
                    d_v=d["d_v"], d_conv=d["d_conv"])
    layer = GDNLayer(dims, torch.from_numpy(w["conv_w"]), torch.from_numpy(w["A_log"]),
                     torch.from_numpy(w["dt_bias"]), eps=w["eps"], q_scale=w["q_scale"],
                     device=dev)
    layer.state.copy_(torch.from_numpy(w["state"]))
    slots = torch.from_numpy(w["slot_ids"]).to(dev)
    x = torch.from_numpy(w["x"]).view(torch.bfloat16).to(dev)
    a = torch.from_numpy(w["a"]).to(dev)
    b = torch.from_numpy(w["b"]).to(dev)
    if name.startswith("decode"):
        layer.conv_state.copy_(torch.from_numpy(w["conv_state"]).view(torch.bfloat16))
        for s in range(4):
            layer.decode(x[s], a[s], b[s], slots)
    elif name == "multitoken":
        layer.conv_state.copy_(torch.from_numpy(w["conv_state"]).view(torch.bfloat16))
        cu = torch.from_numpy(w["cu_seqlens"]).to(dev)
        for _ in range(2):
            layer.prefill(x, a, b, cu, slots)
    else:
        cu = torch.from_numpy(w["cu_seqlens"]).to(dev)
        reset = torch.ones(1, dtype=torch.uint8, device=dev)
        flags = gdn.GDN_PREFILL_TC_HEAD_SCAN if name.endswith("_head") else \
            gdn.GDN_PREFILL_TC_TILE_SCAN
        for _ in range(2):
            layer.prefill(x, a, b, cu, slots, reset=reset, flags=flags)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    print(f"profile run {name}: {PROFILE_RUNS[name]}: ok")
    return 0


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


def cpu_baseline_prefill():
    """fp64 oracle (front + per-token recurrence) on the B=1, T=4096 prefill workload: with one
    thread on 2 of the 16 key heads (4 of 32 value heads) and with all host threads on all
    heads; tokens/s scaled to the whole layer (rank 0, N=1 only)."""
    import oracle
    import synthetic
    w = synthetic.prefill(T=PREFILL_T)
    threads = oracle.default_threads()
    t0 = time.perf_counter()
    oracle.layer(w, threads=1, k_heads=[0, 1])
    t1 = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.layer(w, threads=threads)
    tn = time.perf_counter() - t0
    return {"one_thread": {"value": PREFILL_T / (t1 * 8), "unit": UNIT, "cores": 1,
                           "kind": "oracle",
                           "sample": f"T=4096, 4 of 32 value heads in {t1:.1f} s, scaled x8"},
            "all_threads": {"value": PREFILL_T / tn, "unit": UNIT, "cores": threads,
                            "kind": "oracle", "sample": f"T=4096, all 32 heads in {tn:.1f} s"}}


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.profile_run:
        return profile_run(args.profile_run)

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
    launches = gdn.layer_decode_launches(dims, N_SEQS) * K

    # ------------------------------------------------------------------ e2e through the API
    # the host-buffer decode pipeline (gdn_decode_pipe_step, one C-ABI call per step): each
    # step's x | a | b | slot ids sit in one pinned host row, copied in (one copy) on the
    # pipeline's input stream, and the output is copied back to pinned host memory on
    # its output stream, every step; the copies overlap the neighbouring steps' compute (two
    # staging sets), while the steps stay in order on the compute stream.
    comp = torch.cuda.current_stream()
    pipe = layer.decode_pipe(N_SEQS, stream=comp)
    row_bytes = pipe.packed_bytes                    # x | a | b | slot ids: one copy per step
    ox, oa, ob, osl = pipe.packed_offsets
    packed_h = torch.zeros((X_STEPS, row_bytes), dtype=torch.uint8).pin_memory()

    def bytes_of(arr, dtype):
        return torch.from_numpy(np.ascontiguousarray(arr, dtype)).view(torch.uint8).reshape(-1)
    sl_row = bytes_of(w["slot_ids"], np.int32)
    for i in range(X_STEPS):
        xr = torch.from_numpy(w["x"][i]).view(torch.uint8).reshape(-1)
        packed_h[i, ox:ox + xr.numel()] = xr
        ar, br = bytes_of(w["a"][i], np.float32), bytes_of(w["b"][i], np.float32)
        packed_h[i, oa:oa + ar.numel()] = ar
        packed_h[i, ob:ob + br.numel()] = br
        packed_h[i, osl:osl + sl_row.numel()] = sl_row
    o_h = [torch.empty((N_SEQS, dims.H_v, dims.d_v), dtype=torch.bfloat16).pin_memory()
           for _ in range(2)]
    rows = [packed_h[i].data_ptr() for i in range(X_STEPS)]
    o_ptrs = [o.data_ptr() for o in o_h]

    def e2e_step(s):
        pipe.step_packed_ptr(rows[s % X_STEPS], None, o_ptrs[s % 2])

    # warm-up: W steps, and one pass over every pinned input row (the first copy out of a
    # freshly pinned row costs more than later ones; a serving loop reuses its pinned buffers)
    WE = max(W, X_STEPS)
    for s in range(WE):
        e2e_step(s)
    pipe.flush()
    torch.cuda.synchronize()
    barrier()
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    e_start.record(comp)
    for s in range(K):
        e2e_step(WE + s)
    pipe.flush()                                    # the last outputs are in host memory
    e_end.record(comp)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end))
    h2d = row_bytes
    d2h = o_h[0].numel() * 2
    e2e = {"value": job_throughput(N_SEQS * K, world, e2e_ms), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "ms_per_step": e2e_ms / K,
           "path": "gdn_decode_pipe_step_packed per step (GDNLayer.decode_pipe): pinned H2D "
                   "of one row of x, a, b and the slot ids and D2H of o every step, on the "
                   "pipeline's copy streams, overlapped with the neighbouring steps"}
    pipe.close()
    assert gdn.device_status() == 0

    dec_bytes = DECODE_KERNEL_BYTES_PER_TOKEN * N_SEQS
    achieved = dec_bytes / (dec_kernel_ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"],
                "traffic": ncu_traffic("decode", ["decode.cu", "gdn_common.cuh"]),
                "traffic_note": "ncu DRAM read + write bytes inside one launch; part of the "
                                "state it writes is still in L2 when it ends and reaches DRAM "
                                "during the next launch",
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

    # ------------------------------------------------------------------ varlen and long prefill
    # Inputs generated on the device (seeded; the same shapes and distributions as the
    # parity tests' synthetic workloads): inputs of these sizes exceed L2, so no flush.
    gen = torch.Generator(device=dev)

    def packed_inputs(lengths, seed, a_mean=0.0, b_std=1.0):
        gen.manual_seed(seed)
        T = int(sum(lengths))
        n = len(lengths)
        x = torch.randn((T, dims.conv_dim), generator=gen, device=dev).to(torch.bfloat16)
        a = torch.randn((T, dims.H_v), generator=gen, device=dev) + a_mean
        b = torch.randn((T, dims.H_v), generator=gen, device=dev) * b_std
        cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32,
                          device=dev)
        return x, a, b, cu, T, n

    def time_packed(lengths, seed, *, reset, slots_list, n_slots, a_mean=0.0, b_std=1.0,
                    iters=3, name=""):
        """gdn_layer_prefill over one packed batch; returns (ms per call, layer)."""
        pdims = gdn.Dims(n_slots=n_slots, H_k=dims.H_k, H_v=dims.H_v, d_k=dims.d_k,
                         d_v=dims.d_v, d_conv=dims.d_conv)
        L = GDNLayer(pdims, torch.from_numpy(pw_conv_w), torch.from_numpy(pw_A_log),
                     torch.from_numpy(pw_dt_bias), eps=1e-6, q_scale=dims.d_k ** -0.5,
                     device=dev)
        gen.manual_seed(seed)
        if not reset:
            L.state.normal_(0.0, 0.02, generator=gen)
            L.conv_state.copy_(torch.randn(L.conv_state.shape, generator=gen, device=dev))
        x, a, b, cu, T, n = packed_inputs(lengths, seed + 1, a_mean=a_mean, b_std=b_std)
        slots_t = torch.tensor(slots_list, dtype=torch.int32, device=dev)
        rs = torch.ones(n, dtype=torch.uint8, device=dev) if reset else None
        o_ = torch.empty((T, dims.H_v, dims.d_v), dtype=torch.bfloat16, device=dev)
        need_ = gdn.prefill_workspace_size(pdims, T, n, 64, torch.float16)
        ws_ = torch.empty(max(need_, 16), dtype=torch.uint8, device=dev)

        def call():
            gdn.layer_prefill(pdims, x, L.conv_w, L.conv_state, cu, slots_t, a, b, L.A_log,
                              L.dt_bias, L.state, o_, eps=L.eps, q_scale=L.q_scale, chunk=64,
                              reset=rs, workspace=ws_)
        call()
        torch.cuda.synchronize()
        assert gdn.device_status() == 0, name
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(iters)]
        for i in range(iters):
            ev[i][0].record()
            call()
            ev[i][1].record()
        torch.cuda.synchronize()
        ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in ev)
        del x, a, b, o_, ws_
        return max_over_ranks(ms), L, slots_t

    def pf_record(workload, lengths, reset, ms, launches_per_call, iters):
        nbytes, flops = prefill_algorithmic(lengths, reset, dims.H_v)
        t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
        t_tc = flops / (peaks["bf16_tflops"] * 1e12)
        t_roof = max(t_hbm, t_tc)
        T = int(sum(lengths))
        return {"workload": workload, "value": job_throughput(T, world, ms), "unit": UNIT,
                "ms_per_call": ms, "tokens": T, "sequences": len(lengths),
                "roofline": {"bound": "hbm" if t_hbm >= t_tc else "tensor",
                             "t_roofline_us": t_roof * 1e6, "frac": t_roof / (ms * 1e-3),
                             "algorithmic_bytes": nbytes, "algorithmic_flops": flops,
                             "hbm_gbs_achieved": nbytes / (ms * 1e-3) / 1e9,
                             "tflops_achieved": flops / (ms * 1e-3) / 1e12,
                             "peak_source": peaks["source"]},
                "gpu_launches": launches_per_call * iters}

    sms = torch.cuda.get_device_properties(dev).multi_processor_count

    def layer_launches(lengths):
        """Kernels one gdn_layer_prefill call launches: for more than one sequence (or at most
        16 tokens) the short-sequence kernel (few sequences) or front + token-by-token kernel
        (many), then the record and scan kernels unless T_total <= 16."""
        n, T = len(lengths), sum(lengths)
        short = 0
        if n > 1 or T <= 16:
            short = 1 if n * dims.H_v * (dims.d_v // 32) <= 8 * sms else 2
        return short + (2 if T > 16 else 0)

    varlen = None
    long_ctx = None
    if not args.no_prefill:
        pw_conv_w, pw_A_log, pw_dt_bias = pw["conv_w"], pw["A_log"], pw["dt_bias"]
        del pl, px, po, ws, fq, fk, fv, fg, fb, flush
        torch.cuda.empty_cache()
    if not args.no_prefill and not args.no_varlen:
        # 16 sequences, lengths U[128, 8192], slots = the first 16 of a seeded permutation of
        # 0..63, nonzero initial recurrent and conv states
        lengths = [int(v) for v in synthetic.varlen_lengths(seed=synthetic.SEED_BASE + 3)]
        perm = np.random.default_rng(synthetic.SEED_BASE + 3).permutation(64)[:16].tolist()
        ms, L3, _ = time_packed(lengths, synthetic.SEED_BASE + 3 + 1000 * rank, reset=False,
                                slots_list=perm, n_slots=64, iters=5, name="varlen")
        varlen = pf_record("varlen packed prefill: 16 sequences, lengths U[128, 8192] "
                           f"(sum {sum(lengths)}), non-contiguous slots, nonzero initial "
                           "states, through gdn_layer_prefill", lengths, False, ms,
                           layer_launches(lengths), 5)
        del L3
        torch.cuda.empty_cache()
    if not args.no_prefill and not args.no_long:
        # 4 x 65536 prefill from zero states, a ~ N(2, 1), b ~ N(0, 2^2); then 512 decode
        # steps at batch 4 from the resulting states, replayed from one CUDA graph
        lengths = [65536] * 4
        ms, L4, slots4 = time_packed(lengths, synthetic.SEED_BASE + 4 + 1000 * rank, reset=True,
                                     slots_list=[0, 1, 2, 3], n_slots=4, a_mean=2.0, b_std=2.0,
                                     iters=3, name="long")
        long_ctx = {"prefill": pf_record("long-context prefill: 4 x 65536 tokens from zero "
                                         "states, strongly decaying gates, through "
                                         "gdn_layer_prefill", lengths, True, ms,
                                         layer_launches(lengths), 3)}
        gen.manual_seed(synthetic.SEED_BASE + 40)
        steps4 = 512
        xd = torch.randn((steps4, 4, dims.conv_dim), generator=gen, device=dev).to(torch.bfloat16)
        ad = torch.randn((steps4, 4, dims.H_v), generator=gen, device=dev)
        bd = torch.randn((steps4, 4, dims.H_v), generator=gen, device=dev)
        od = torch.empty((4, dims.H_v, dims.d_v), dtype=torch.bfloat16, device=dev)
        wsd = torch.empty(gdn.decode_workspace_size(L4.dims, 4), dtype=torch.uint8, device=dev)

        def dstep(i):
            gdn.layer_decode(L4.dims, xd[i], L4.conv_w, L4.conv_state, slots4, ad[i], bd[i],
                             L4.A_log, L4.dt_bias, L4.state, od, eps=L4.eps, q_scale=L4.q_scale,
                             workspace=wsd)
        for i in range(3):
            dstep(i)
        torch.cuda.synchronize()
        g4 = torch.cuda.CUDAGraph()
        cs4 = torch.cuda.Stream()
        cs4.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cs4):
            with torch.cuda.graph(g4, stream=cs4):
                for i in range(steps4):
                    dstep(i)
        torch.cuda.current_stream().wait_stream(cs4)
        g4.replay()  # warm replay (untimed): the graph's first launch also uploads it
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g4.replay()
        e1.record()
        torch.cuda.synchronize()
        assert gdn.device_status() == 0
        dms = max_over_ranks(e0.elapsed_time(e1)) / steps4
        dbytes = DECODE_STEP_BYTES_PER_TOKEN * 4
        long_ctx["decode"] = {
            "workload": "512 decode steps at batch 4 from the long prefill's states, "
                        "gdn_layer_decode per step, replayed from one CUDA graph",
            "value": job_throughput(4, world, dms), "unit": UNIT, "ms_per_step": dms,
            "roofline": {"bound": "hbm", "algorithmic_bytes_per_step": dbytes,
                         "achieved": dbytes / (dms * 1e-3) / 1e9, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": dbytes / (dms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                         "peak_source": peaks["source"]},
            "gpu_launches": gdn.layer_decode_launches(L4.dims, 4) * steps4}
        del g4, L4, xd, ad, bd
        torch.cuda.empty_cache()


    # ------------------------------------------------------------------ scope rows f1 - f4
    # f1: the decode step with the output gate; f3: the tiled-GQA / fused beta-alpha layout
    # (decode and a T=4096 prefill); f2: 64 sequences
    # of 4 tokens each (speculative / multi-token steps) and f4: 60 single-token sequences with
    # 4 prompts of 1024 tokens in one call, both through gdn_conv_step + gdn_chunked_prefill,
    # which sends sequences of at most 16 tokens to the token-by-token kernel and the rest to
    # the chunked kernels. Inputs drawn on the device (seeded).
    next_rows = None
    if not args.no_next:
        next_rows = {}
        gen.manual_seed(synthetic.SEED_BASE + 50)
        nst = 16
        xg = torch.randn((nst, N_SEQS, dims.conv_dim), generator=gen, device=dev).to(torch.bfloat16)
        ag = torch.randn((nst, N_SEQS, dims.H_v), generator=gen, device=dev)
        bg = torch.randn((nst, N_SEQS, dims.H_v), generator=gen, device=dev)
        zg = torch.randn((nst, N_SEQS, dims.H_v, dims.d_v), generator=gen,
                         device=dev).to(torch.bfloat16)
        nw = 1.0 + 0.1 * torch.randn(dims.d_v, generator=gen, device=dev)
        og = torch.empty((N_SEQS, dims.H_v, dims.d_v), dtype=torch.bfloat16, device=dev)

        def gstep(i):
            gdn.layer_decode(dims, xg[i % nst], layer.conv_w, layer.conv_state, slots,
                             ag[i % nst], bg[i % nst], layer.A_log, layer.dt_bias, layer.state,
                             og, eps=layer.eps, q_scale=layer.q_scale, workspace=dec_ws,
                             gate=gdn.OutGate(zg[i % nst], nw, 1e-6))
        for i in range(W):
            gstep(i)
        torch.cuda.synchronize()
        gg = torch.cuda.CUDAGraph()
        csg = torch.cuda.Stream()
        csg.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(csg):
            with torch.cuda.graph(gg, stream=csg):
                for i in range(K):
                    gstep(i)
        torch.cuda.current_stream().wait_stream(csg)
        gg.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        gg.replay()
        e1.record()
        torch.cuda.synchronize()
        assert gdn.device_status() == 0
        gms = max_over_ranks(e0.elapsed_time(e1)) / K
        gbytes = (DECODE_STEP_BYTES_PER_TOKEN + dims.H_v * dims.d_v * 2) * N_SEQS
        next_rows["f1_gated_decode"] = {
            "workload": "decode, 64 sequences, with the output gate RMSNorm(o) * w * SiLU(z) "
                        "(bf16 z) through gdn_layer_decode: front, decode (fp32 o), gate "
                        "kernels; graph of K steps",
            "value": job_throughput(N_SEQS, world, gms), "unit": UNIT, "ms_per_step": gms,
            "roofline": {"bound": "hbm", "algorithmic_bytes_per_step": gbytes,
                         "achieved": gbytes / (gms * 1e-3) / 1e9, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s",
                         "frac": gbytes / (gms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                         "peak_source": peaks["source"]},
            "gpu_launches": gdn.layer_decode_launches(dims, N_SEQS, gated=True) * K}

        # f3: the tiled-GQA / fused beta-alpha layout (value head h reads key head h % H_k;
        # the gate inputs as one [T][H_k][2 r] array, b = NULL): the 64-sequence decode step
        # (graph of K steps) and one B=1, T=4096 layer prefill (L2 flushed)
        dims3 = gdn.Dims(n_slots=dims.n_slots, H_k=dims.H_k, H_v=dims.H_v, d_k=dims.d_k,
                         d_v=dims.d_v, d_conv=dims.d_conv,
                         layout=gdn.GDN_GQA_TILED | gdn.GDN_GATES_MIXED_BA)
        rr = dims.H_v // dims.H_k
        bag = torch.randn((nst, N_SEQS, dims.H_k, 2 * rr), generator=gen, device=dev)

        def step3(i):
            gdn.layer_decode(dims3, xg[i % nst], layer.conv_w, layer.conv_state, slots,
                             bag[i % nst], None, layer.A_log, layer.dt_bias, layer.state, og,
                             eps=layer.eps, q_scale=layer.q_scale, workspace=dec_ws)
        for i in range(W):
            step3(i)
        torch.cuda.synchronize()
        g3 = torch.cuda.CUDAGraph()
        cs3 = torch.cuda.Stream()
        cs3.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cs3):
            with torch.cuda.graph(g3, stream=cs3):
                for i in range(K):
                    step3(i)
        torch.cuda.current_stream().wait_stream(cs3)
        g3.replay()
        torch.cuda.synchronize()
        e0.record()
        g3.replay()
        e1.record()
        torch.cuda.synchronize()
        assert gdn.device_status() == 0
        ms3 = max_over_ranks(e0.elapsed_time(e1)) / K
        dbytes3 = DECODE_STEP_BYTES_PER_TOKEN * N_SEQS
        f3 = {"decode": {
            "workload": "decode, 64 sequences, tiled GQA + fused beta/alpha gate layout, "
                        "gdn_layer_decode (front + decode kernels); graph of K steps",
            "value": job_throughput(N_SEQS, world, ms3), "unit": UNIT, "ms_per_step": ms3,
            "roofline": {"bound": "hbm", "algorithmic_bytes_per_step": dbytes3,
                         "achieved": dbytes3 / (ms3 * 1e-3) / 1e9, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": dbytes3 / (ms3 * 1e-3) / 1e9 / peaks["hbm_gbs"],
                         "peak_source": peaks["source"]},
            "gpu_launches": gdn.layer_decode_launches(dims3, N_SEQS) * K}}
        del g3, bag
        if not args.no_prefill:
            gen.manual_seed(synthetic.SEED_BASE + 55)
            T3 = PREFILL_T
            x3 = torch.randn((T3, dims.conv_dim), generator=gen, device=dev).to(torch.bfloat16)
            a3 = torch.randn((T3, dims.H_k, 2 * rr), generator=gen, device=dev)
            cu3 = torch.tensor([0, T3], dtype=torch.int32, device=dev)
            sl3 = torch.zeros(1, dtype=torch.int32, device=dev)
            rs3 = torch.ones(1, dtype=torch.uint8, device=dev)
            o3 = torch.empty((T3, dims.H_v, dims.d_v), dtype=torch.bfloat16, device=dev)
            ws3 = torch.empty(gdn.prefill_workspace_size(dims3, T3, 1, 64, torch.float16),
                              dtype=torch.uint8, device=dev)
            flush3 = torch.empty(64 << 20, dtype=torch.float32, device=dev)

            def call3():
                gdn.layer_prefill(dims3, x3, layer.conv_w, layer.conv_state, cu3, sl3, a3, None,
                                  layer.A_log, layer.dt_bias, layer.state, o3, eps=layer.eps,
                                  q_scale=layer.q_scale, chunk=64, reset=rs3, workspace=ws3)
            for _ in range(3):
                call3()
            torch.cuda.synchronize()
            assert gdn.device_status() == 0
            ts3 = []
            for _ in range(5):
                flush3.zero_()
                e0.record()
                call3()
                e1.record()
                torch.cuda.synchronize()
                ts3.append(e0.elapsed_time(e1))
            ms3p = max_over_ranks(statistics.median(ts3))
            f3["prefill"] = pf_record(
                "chunked prefill B=1, T=4096, tiled GQA + fused beta/alpha gate layout, through "
                "gdn_layer_prefill (L2 flushed)", [T3], True, ms3p, layer_launches([T3]), 5)
            del x3, a3, o3, ws3, flush3
        next_rows["f3_layouts"] = f3
        del gg, xg, ag, bg, zg

        def packed_call(lengths, seed, flags=0, iters=10, layer_path=True):
            """ms per call of one packed batch through gdn_layer_prefill (layer_path) or
            gdn_conv_step + gdn_chunked_prefill, on the decode layer's pools"""
            x, a, b, cu, T, n = packed_inputs(lengths, seed)
            sl = torch.arange(n, dtype=torch.int32, device=dev)
            q2, k2, v2, g2, b2 = gdn.front_outputs(dims, T, torch.float16, dev)
            o2 = torch.empty((T, dims.H_v, dims.d_v), dtype=torch.bfloat16, device=dev)
            need2 = gdn.prefill_workspace_size(dims, T, n, 64, torch.float16, flags)
            ws2 = torch.empty(max(need2, 16), dtype=torch.uint8, device=dev)

            def call():
                if layer_path:
                    gdn.layer_prefill(dims, x, layer.conv_w, layer.conv_state, cu, sl, a, b,
                                      layer.A_log, layer.dt_bias, layer.state, o2, eps=layer.eps,
                                      q_scale=layer.q_scale, chunk=64, workspace=ws2,
                                      flags=flags)
                    return
                gdn.conv_step(dims, x, layer.conv_w, layer.conv_state, cu, sl, a, b,
                              layer.A_log, layer.dt_bias, q2, k2, v2, g2, b2, eps=layer.eps,
                              q_scale=layer.q_scale)
                gdn.chunked_prefill(dims, q2, k2, v2, g2, b2, layer.state, sl, cu, o2, chunk=64,
                                    workspace=ws2, flags=flags)
            for _ in range(3):
                call()
            torch.cuda.synchronize()
            assert gdn.device_status() == 0
            ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(iters)]
            for i in range(iters):
                ev[i][0].record()
                call()
                ev[i][1].record()
            torch.cuda.synchronize()
            return max_over_ranks(statistics.mean(p0.elapsed_time(p1) for p0, p1 in ev))

        for key, lengths, flags, launches2, text in (
                ("f2_multi_token", [4] * 64, gdn.GDN_PREFILL_RECURRENT, 2,
                 "64 sequences x 4 tokens (speculative / multi-token step), nonzero states, "
                 "through gdn_layer_prefill with GDN_PREFILL_RECURRENT (every sequence at most "
                 "16 tokens: front of the short sequences + token-by-token kernel only)"),
                ("f4_mixed_batch", [1] * 60 + [1024] * 4, 0, 4,
                 "mixed batch in one call: 60 single-token sequences + 4 prompts of 1024 "
                 "tokens, nonzero states, through gdn_layer_prefill (front of the short "
                 "sequences + token-by-token kernel for the single tokens, record and scan "
                 "kernels for the prompts)")):
            seed = synthetic.SEED_BASE + 60 + len(next_rows)
            ms = packed_call(lengths, seed, flags=flags)
            nl = layer_launches(lengths) - (2 if flags else 0)  # the promise skips 2 kernels
            rec = pf_record(text, lengths, False, ms, nl, 10)
            ms2 = packed_call(lengths, seed, flags=flags, layer_path=False)
            rec["two_call_path"] = {
                "ms_per_call": ms2, "launches_per_call": launches2,
                "calls": "gdn_conv_step + gdn_chunked_prefill" +
                         (" with GDN_PREFILL_RECURRENT" if flags else " (routes by length)")}
            next_rows[key] = rec
        torch.cuda.empty_cache()

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
        # the prefill roofline at top level (B=1, T=4096 through gdn_layer_prefill)
        "prefill_roofline": (dict(prefill["roofline"], value=prefill["value"],
                                  ms_per_step=prefill["ms_per_step"])
                             if prefill is not None else None),
        "varlen_prefill": varlen,
        "long_context": long_ctx,
        "scope_next_rows": next_rows,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
        if not args.no_prefill:
            line["cpu_baseline_prefill"] = cpu_baseline_prefill()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
