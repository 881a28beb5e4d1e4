"""Seeded synthetic workloads for the gated delta-rule layer (Qwen3-Next layer shapes).

This module holds random-number generation and data-format packing only (fp32 -> bf16
rounding to nearest-even, packing of sequences with cu_seqlens); none of the layer's
arithmetic. Both the CUDA tests/bench and the CPU oracle read the same arrays from here.

Workloads (per-head shapes d_k = d_v, GQA H_v = r * H_k):

* ``tiny``    B=1, T=64, H=2, d=32, fp32 q|k|v|a|b ~ N(0,1), no conv, chunk 16.
* ``decode``  64 sequences x 1 token per step, H_k=16 -> H_v=32, d=128, bf16 x ~ N(0,1),
              fp32 state ~ N(0, 0.02^2), bf16 conv state ~ N(0,1), conv w ~ N(0, 0.5^2).
* ``prefill`` B=1, T=4096, same shapes, zero initial states (reset), chunk 64.
* ``varlen``  16 sequences, lengths ~ U[128, 8192], slots = seeded permutation of 0..63.
* ``long``    B=4 x T=65536 with a ~ N(2,1), b ~ N(0, 2^2), then decode steps.

Readings: "N(0, s)" in the workload text is taken as standard deviation s; A_log =
log(U[1,16]); dt_bias ~ N(0,1); eps = 1e-6; q_scale = 1/sqrt(d_k).
"""
from __future__ import annotations

import math

import numpy as np

SEED_BASE = 1000


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def _normal_f32(g: np.random.Generator, shape, std=1.0, mean=0.0, chunk=1 << 24):
    """Standard normals as float32, generated in slices to bound host memory."""
    out = np.empty(shape, dtype=np.float32)
    flat = out.reshape(-1)
    for s in range(0, flat.size, chunk):
        e = min(flat.size, s + chunk)
        flat[s:e] = g.standard_normal(e - s, dtype=np.float32)
    if std != 1.0:
        flat *= np.float32(std)
    if mean != 0.0:
        flat += np.float32(mean)
    return out


def _normal_bf16(g, shape, std=1.0):
    out = np.empty(shape, dtype=np.uint16)
    flat = out.reshape(-1)
    step = 1 << 24
    for s in range(0, flat.size, step):
        e = min(flat.size, s + step)
        v = g.standard_normal(e - s, dtype=np.float32)
        if std != 1.0:
            v *= np.float32(std)
        flat[s:e] = f32_to_bf16_bits(v)
    return out


GQA_TILED = 1        # layout flags (the C header's GDN_GQA_TILED, GDN_GATES_MIXED_BA)
GATES_MIXED_BA = 2


def dims(H_k=16, H_v=32, d_k=128, d_v=128, d_conv=4, n_slots=64, layout=0):
    return dict(H_k=H_k, H_v=H_v, d_k=d_k, d_v=d_v, d_conv=d_conv, n_slots=n_slots,
                conv_dim=2 * H_k * d_k + H_v * d_v, layout=layout)


def to_mixed_ba(a, b, H_k):
    """Pack separate gate inputs a, b [..., H_v] into the fused beta/alpha layout
    [..., H_k, 2 r]: per key head the r beta logits, then the r alphas (value heads hk r + j)."""
    a = np.asarray(a, np.float32)
    b = np.asarray(b, np.float32)
    H_v = a.shape[-1]
    r = H_v // H_k
    lead = a.shape[:-1]
    m = np.empty(lead + (H_k, 2 * r), np.float32)
    m[..., :r] = b.reshape(lead + (H_k, r))
    m[..., r:] = a.reshape(lead + (H_k, r))
    return m


def _apply_gate_layout(w):
    if w["dims"].get("layout", 0) & GATES_MIXED_BA:
        w["a"] = to_mixed_ba(w["a"], w["b"], w["dims"]["H_k"])
        w["b"] = None
    return w


def _gate_params(g, H_v):
    A_log = np.log(g.uniform(1.0, 16.0, size=H_v)).astype(np.float32)
    dt_bias = g.standard_normal(H_v).astype(np.float32)
    return A_log, dt_bias


def tiny(seed: int = SEED_BASE + 0, T: int = 64, H: int = 2, d: int = 32) -> dict:
    """B=1 fp32 workload without conv: x is [q | k | v] per token."""
    g = rng(seed)
    dm = dims(H_k=H, H_v=H, d_k=d, d_v=d, d_conv=0, n_slots=1)
    x = _normal_f32(g, (T, dm["conv_dim"]))
    a = _normal_f32(g, (T, H))
    b = _normal_f32(g, (T, H))
    A_log, dt_bias = _gate_params(g, H)
    return dict(name="tiny", dims=dm, x=x, x_dtype="f32", conv_w=None, conv_state=None,
                conv_state_dtype=None, a=a, b=b, A_log=A_log, dt_bias=dt_bias,
                state=np.zeros((1, H, d, d), np.float32), slot_ids=np.zeros(1, np.int32),
                cu_seqlens=np.array([0, T], np.int32), reset=np.ones(1, np.uint8),
                eps=1e-6, q_scale=1.0 / math.sqrt(d), chunk=16)


def _pool(g, dm, state_std, conv_std):
    S = _normal_f32(g, (dm["n_slots"], dm["H_v"], dm["d_k"], dm["d_v"]), std=state_std) \
        if state_std > 0 else np.zeros((dm["n_slots"], dm["H_v"], dm["d_k"], dm["d_v"]),
                                       np.float32)
    rows = dm["d_conv"] - 1
    cs = _normal_bf16(g, (dm["n_slots"], rows, dm["conv_dim"]), std=conv_std) \
        if conv_std > 0 else np.zeros((dm["n_slots"], rows, dm["conv_dim"]), np.uint16)
    return S, cs


def decode(seed: int = SEED_BASE + 1, n_seqs: int = 64, steps: int = 256, **dkw) -> dict:
    """n_seqs sequences, one token each per step, ``steps`` steps.

    x [steps, n_seqs, conv_dim] bf16 bits, a/b [steps, n_seqs, H_v] fp32, slots 0..n_seqs-1.
    """
    g = rng(seed)
    dm = dims(**dkw)
    if dm["n_slots"] < n_seqs:
        dm["n_slots"] = n_seqs
    A_log, dt_bias = _gate_params(g, dm["H_v"])
    conv_w = _normal_f32(g, (dm["conv_dim"], dm["d_conv"]), std=0.5)
    S, cs = _pool(g, dm, 0.02, 1.0)
    x = _normal_bf16(g, (steps, n_seqs, dm["conv_dim"]))
    a = _normal_f32(g, (steps, n_seqs, dm["H_v"]))
    b = _normal_f32(g, (steps, n_seqs, dm["H_v"]))
    return _apply_gate_layout(dict(
        name="decode", dims=dm, x=x, x_dtype="bf16", conv_w=conv_w, conv_state=cs,
        conv_state_dtype="bf16", a=a, b=b, A_log=A_log, dt_bias=dt_bias, state=S,
        slot_ids=np.arange(n_seqs, dtype=np.int32), steps=steps, n_seqs=n_seqs,
        cu_seqlens=np.arange(n_seqs + 1, dtype=np.int32), reset=None,
        eps=1e-6, q_scale=1.0 / math.sqrt(dm["d_k"])))


def packed(lengths, seed: int, *, slots=None, state_std=0.0, conv_std=0.0, reset=False,
           a_mean=0.0, a_std=1.0, b_std=1.0, name="packed", chunk=64, **dkw) -> dict:
    """Sequences of the given lengths packed into one token stream (cu_seqlens)."""
    g = rng(seed)
    dm = dims(**dkw)
    lengths = [int(L) for L in lengths]
    n = len(lengths)
    if slots is None:
        slots = np.arange(n, dtype=np.int32)
    slots = np.asarray(slots, dtype=np.int32)
    dm["n_slots"] = max(dm["n_slots"], int(slots.max()) + 1)
    A_log, dt_bias = _gate_params(g, dm["H_v"])
    conv_w = _normal_f32(g, (dm["conv_dim"], dm["d_conv"]), std=0.5) if dm["d_conv"] > 0 \
        else None
    S, cs = _pool(g, dm, state_std, conv_std)
    T = int(sum(lengths))
    cu = np.zeros(n + 1, np.int32)
    cu[1:] = np.cumsum(lengths)
    x = _normal_bf16(g, (T, dm["conv_dim"]))
    a = _normal_f32(g, (T, dm["H_v"]), std=a_std, mean=a_mean)
    b = _normal_f32(g, (T, dm["H_v"]), std=b_std)
    rs = np.full(n, 1 if reset else 0, np.uint8)
    return _apply_gate_layout(dict(
        name=name, dims=dm, x=x, x_dtype="bf16", conv_w=conv_w, conv_state=cs,
        conv_state_dtype="bf16", a=a, b=b, A_log=A_log, dt_bias=dt_bias, state=S,
        slot_ids=slots, cu_seqlens=cu, reset=rs, eps=1e-6,
        q_scale=1.0 / math.sqrt(dm["d_k"]), chunk=chunk))


def prefill(seed: int = SEED_BASE + 2, T: int = 4096, **dkw) -> dict:
    """B=1, T tokens, zero initial recurrent and conv state (reset), chunk 64."""
    return packed([T], seed, reset=True, name="prefill", **dkw)


def varlen_lengths(seed: int = SEED_BASE + 3, n: int = 16, lo: int = 128, hi: int = 8192):
    g = rng(seed + 7919)
    return g.integers(lo, hi + 1, size=n).tolist()


def varlen(seed: int = SEED_BASE + 3, n: int = 16, lo: int = 128, hi: int = 8192,
           **dkw) -> dict:
    """n sequences with lengths ~ U[lo, hi], non-contiguous slots, nonzero initial states."""
    lengths = varlen_lengths(seed, n, lo, hi)
    g = rng(seed + 104729)
    perm = g.permutation(64).astype(np.int32)
    return packed(lengths, seed, slots=perm[:n], state_std=0.02, conv_std=1.0,
                  name="varlen", **dkw)


def long_context(seed: int = SEED_BASE + 4, B: int = 4, T: int = 65536, **dkw) -> dict:
    """B sequences of T tokens with strongly decaying gates: a ~ N(2,1), b ~ N(0, 2^2)."""
    return packed([T] * B, seed, reset=True, a_mean=2.0, a_std=1.0, b_std=2.0,
                  name="long", **dkw)
