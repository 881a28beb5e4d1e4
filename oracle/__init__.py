"""fp64 CPU oracle for the gated delta-rule layer -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package. The CUDA library never calls it and shares no code with it.

The arithmetic lives in ``gdn_oracle.cpp`` (plain fp64 loops, one function per step of the
method, each citing the page it follows). This module only builds that file with the host
C++ compiler, loads it with ctypes and marshals numpy arrays:

* ``front``      -- conv1d over [conv_state; x] + SiLU + q|k|v split + L2 norm + q scale +
                    gates (ik_llama.cpp src/llama-delta-net.cpp, build_layer_attn_linear_core;
                    qwen3next.cpp build_layer_attn_linear for the gate).
* ``recurrence`` -- the per-token gated delta rule (qwen3next.cpp,
                    build_delta_net_autoregressive), the definition the GPU is compared to.
* ``chunked``    -- the chunked WY/UT restatement (qwen3next.cpp, removed single-chunk path
                    and build_delta_net_chunking), used only to pin chunked == recurrent.
* ``gated_norm`` -- the output gate after the delta rule: RMS norm of each (token, value head)
                    row of o times the norm weight, times SiLU(z) (ik_llama.cpp
                    build_layer_attn_linear_core: llm_build_norm(..., ssm_norm, LLM_NORM_RMS)
                    then ggml_fused_mul_unary(z, ., SILU)), plain numpy in fp64.

``layer`` / ``decode_steps`` follow either weight family's layout (ik_llama.cpp
build_layer_attn_linear_core / build_layer_attn_linear): the key heads repeated to the value
heads grouped or tiled, and the gate inputs separate or as the fused beta/alpha projection.
Both are data movement done here before the fp64 routines run.

Parity status: every function is pinned by the CPU tests in ``tests/test_oracle_pins.py``
(closed forms, special cases, a hand-worked example, brute force on tiny inputs, identities).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile gdn_oracle.cpp into liboracle.so next to it (g++, -O2, no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread",
           "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I = ctypes.c_int
            L = ctypes.c_int64
            D = ctypes.c_double
            lib.oracle_front.argtypes = [L, I, P, P, I, I, I, I, I, P, P, P, P, P, P, P, D, D,
                                         P, P, P, P, P, I]
            lib.oracle_front.restype = I
            lib.oracle_recurrence.argtypes = [L, I, P, I, I, I, I, P, P, P, P, P, P, P, I]
            lib.oracle_recurrence.restype = I
            lib.oracle_chunked.argtypes = [L, I, P, I, I, I, I, P, P, P, P, P, P, P, I, I]
            lib.oracle_chunked.restype = I
            _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact decode of bf16 bit patterns (uint16) to float64."""
    u32 = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u32.view(np.float32).astype(np.float64)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def front(x, conv_w, conv_state, cu_seqlens, a, b, A_log, dt_bias, *, H_k, H_v, d_k, d_v,
          d_conv, eps, q_scale, reset=None, threads=None):
    """Front of the layer for packed sequences.

    x [T, conv_dim] (float), conv_w [conv_dim, d_conv], conv_state [n_seqs, d_conv-1, conv_dim]
    (per sequence, already gathered by slot), a/b [T, H_v], A_log/dt_bias [H_v].
    Returns dict(q [T,H_k,d_k], k, v [T,H_v,d_v], g [T,H_v], beta, conv_state (new)).
    """
    lib = _load()
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    n_seqs = cu.shape[0] - 1
    T = int(cu[-1])
    x = _f64(x)
    conv_dim = 2 * H_k * d_k + H_v * d_v
    assert x.shape == (T, conv_dim)
    rows = max(d_conv - 1, 0)
    st = np.zeros((n_seqs, rows, conv_dim)) if conv_state is None else _f64(conv_state).copy()
    w = _f64(conv_w) if d_conv > 0 else None
    rs = None if reset is None else np.ascontiguousarray(reset, dtype=np.uint8)
    q = np.empty((T, H_k, d_k)); k = np.empty((T, H_k, d_k)); v = np.empty((T, H_v, d_v))
    g = np.empty((T, H_v)); beta = np.empty((T, H_v))
    rc = lib.oracle_front(T, n_seqs, _ptr(cu), _ptr(rs), H_k, H_v, d_k, d_v, d_conv,
                          _ptr(x), _ptr(w), _ptr(st), _ptr(_f64(a)), _ptr(_f64(b)),
                          _ptr(_f64(A_log)), _ptr(_f64(dt_bias)), float(eps), float(q_scale),
                          _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                          int(threads or default_threads()))
    assert rc == 0
    return dict(q=q, k=k, v=v, g=g, beta=beta, conv_state=st)


def _core(fn_name, q, k, v, g, beta, S0, cu_seqlens, extra=(), threads=None):
    lib = _load()
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    n_seqs = cu.shape[0] - 1
    q = _f64(q); k = _f64(k); v = _f64(v); g = _f64(g); beta = _f64(beta)
    T, H_k, d_k = q.shape
    _, H_v, d_v = v.shape
    assert T == int(cu[-1]) and H_v % H_k == 0
    S = np.zeros((n_seqs, H_v, d_k, d_v)) if S0 is None else _f64(S0).copy()
    assert S.shape == (n_seqs, H_v, d_k, d_v)
    o = np.zeros((T, H_v, d_v))
    fn = getattr(lib, fn_name)
    rc = fn(T, n_seqs, _ptr(cu), H_k, H_v, d_k, d_v, _ptr(q), _ptr(k), _ptr(v), _ptr(g),
            _ptr(beta), _ptr(S), _ptr(o), *extra, int(threads or default_threads()))
    assert rc == 0
    return o, S


def recurrence(q, k, v, g, beta, S0, cu_seqlens, threads=None):
    """Per-token gated delta rule. Returns (o [T,H_v,d_v], S_final [n_seqs,H_v,d_k,d_v])."""
    return _core("oracle_recurrence", q, k, v, g, beta, S0, cu_seqlens, (), threads)


def chunked(q, k, v, g, beta, S0, cu_seqlens, C, threads=None):
    """Chunked WY/UT restatement with chunk length C (pins chunked == recurrent)."""
    return _core("oracle_chunked", q, k, v, g, beta, S0, cu_seqlens, (int(C),), threads)


GQA_TILED = 1       # value head h reads key head h % H_k (else h // (H_v / H_k))
GATES_MIXED_BA = 2  # gate inputs as the fused beta/alpha projection [T, H_k, 2 r]


def _layout(dims) -> int:
    return int(dims.get("layout", 0))


def _v_heads_of(dims, hk):
    """Value heads that read key head hk (ik_llama.cpp build_layer_attn_linear_core: the
    repeat of q and k to the value heads, grouped on the fused ssm_beta_alpha path, tiled by
    ggml_repeat_4d on the path with separate alpha / beta weights)."""
    H_k, H_v = dims["H_k"], dims["H_v"]
    r = H_v // H_k
    if _layout(dims) & GQA_TILED:
        return [hk + i * H_k for i in range(r)]
    return [hk * r + i for i in range(r)]


def split_mixed_ba(mixed, H_k, H_v):
    """The fused beta/alpha projection [T, H_k, 2 r] -> (a, b), each [T, H_v]: per key head the
    first r values are the beta logits and the next r the alphas of value heads hk r + j
    (ik_llama.cpp build_layer_attn_linear, the two views of mixed_ba_reshaped)."""
    r = H_v // H_k
    m = np.asarray(mixed, dtype=np.float64).reshape(-1, H_k, 2 * r)
    b = m[:, :, :r].reshape(-1, H_v)
    a = m[:, :, r:].reshape(-1, H_v)
    return a, b


def _gates(inputs, T=None):
    """(a, b) [.., H_v] of a workload in either gate layout."""
    dims = inputs["dims"]
    if _layout(dims) & GATES_MIXED_BA:
        a, b = split_mixed_ba(inputs["a"], dims["H_k"], dims["H_v"])
        shape = np.asarray(inputs["a"]).shape[:-2] + (dims["H_v"],)
        return a.reshape(shape), b.reshape(shape)
    return np.asarray(inputs["a"]), np.asarray(inputs["b"])


def _repeat_tiled(q, k, H_v):
    """q, k [T, H_k', d] -> [T, H_v', d] with value head h reading key head h % H_k' (the
    tiled ggml_repeat_4d), so that the recurrence runs with one key head per value head."""
    H_k = q.shape[1]
    idx = [h % H_k for h in range(H_v)]
    return q[:, idx], k[:, idx]


def _channels(dims, k_heads):
    """Channel indices (q | k | v order) of the selected k-heads and their v-heads."""
    H_k, H_v, d_k, d_v = dims["H_k"], dims["H_v"], dims["d_k"], dims["d_v"]
    v_heads = [h for hk in k_heads for h in _v_heads_of(dims, hk)]
    if _layout(dims) & GQA_TILED:
        v_heads = sorted(v_heads)
    qc = [hk * d_k + i for hk in k_heads for i in range(d_k)]
    kc = [H_k * d_k + hk * d_k + i for hk in k_heads for i in range(d_k)]
    vc = [2 * H_k * d_k + h * d_v + j for h in v_heads for j in range(d_v)]
    return np.array(qc + kc + vc, dtype=np.int64), v_heads


def _decode_x(bits_or_f, dtype, ch=None):
    a = np.asarray(bits_or_f)
    if ch is not None:
        a = a[..., ch]
    return bf16_bits_to_f64(a) if dtype == "bf16" else _f64(a)


def layer(inputs: dict, threads=None, k_heads=None):
    """Front + recurrence over one packed synthetic workload (see ``synthetic``).

    Gathers the conv and recurrent states by slot, runs the oracle and returns
    dict(o [T, H_v', d_v], S [n_seqs, H_v', d_k, d_v], conv_state [n_seqs, rows, C'],
    q, k, v, g, beta, v_heads, channels). ``k_heads`` restricts the run to those key heads,
    their value heads and their channels (sampled parity on large workloads); by default
    every head is run.
    """
    dims = inputs["dims"]
    H_k, H_v, d_k, d_v, d_conv = (dims[n] for n in ("H_k", "H_v", "d_k", "d_v", "d_conv"))
    k_heads = list(range(H_k)) if k_heads is None else sorted(k_heads)
    ch, v_heads = _channels(dims, k_heads)
    cu = inputs["cu_seqlens"]
    slots = inputs["slot_ids"]
    reset = inputs.get("reset")
    x = _decode_x(inputs["x"], inputs["x_dtype"], ch)
    conv_state = None
    conv_w = None
    if d_conv > 0:
        conv_state = _decode_x(inputs["conv_state"][slots], inputs["conv_state_dtype"], ch)
        conv_w = _f64(inputs["conv_w"])[ch]
    ga, gb = _gates(inputs)
    fr = front(x, conv_w, conv_state, cu, ga[:, v_heads], gb[:, v_heads],
               np.asarray(inputs["A_log"])[v_heads],
               np.asarray(inputs["dt_bias"])[v_heads], H_k=len(k_heads), H_v=len(v_heads),
               d_k=d_k, d_v=d_v, d_conv=d_conv, eps=inputs["eps"], q_scale=inputs["q_scale"],
               reset=reset, threads=threads)
    S0 = _f64(inputs["state"])[slots][:, v_heads]
    if reset is not None:
        S0[np.asarray(reset, dtype=bool)] = 0.0
    qq, kk = fr["q"], fr["k"]
    if _layout(dims) & GQA_TILED:
        qq, kk = _repeat_tiled(qq, kk, len(v_heads))
    o, S = recurrence(qq, kk, fr["v"], fr["g"], fr["beta"], S0, cu, threads=threads)
    return dict(o=o, S=S, conv_state=fr["conv_state"], q=fr["q"], k=fr["k"], v=fr["v"],
                g=fr["g"], beta=fr["beta"], v_heads=v_heads, channels=ch)


def decode_steps(inputs: dict, steps: int, threads=None, k_heads=None, S0=None,
                 conv_state0=None):
    """``steps`` single-token steps of the decode workload (x [steps, B, conv_dim]).

    Starts from the pools gathered at the workload's slots (or from S0 [B, H_v', d_k, d_v]
    and conv_state0 [B, rows, C'] for the selected heads/channels), carries the states from
    step to step and returns dict(o [steps, B, H_v', d_v], S, conv_state, v_heads, channels).
    """
    dims = inputs["dims"]
    H_k, d_k, d_v, d_conv = (dims[n] for n in ("H_k", "d_k", "d_v", "d_conv"))
    k_heads = list(range(H_k)) if k_heads is None else sorted(k_heads)
    ch, v_heads = _channels(dims, k_heads)
    slots = inputs["slot_ids"]
    B = len(slots)
    cu = np.arange(B + 1, dtype=np.int32)
    S = (_f64(inputs["state"])[slots][:, v_heads] if S0 is None else _f64(S0).copy())
    cst = (_decode_x(inputs["conv_state"][slots], inputs["conv_state_dtype"], ch)
           if conv_state0 is None else _f64(conv_state0).copy())
    conv_w = _f64(inputs["conv_w"])[ch]
    A_log = np.asarray(inputs["A_log"])[v_heads]
    dt_bias = np.asarray(inputs["dt_bias"])[v_heads]
    outs = []
    ga, gb = _gates(inputs)
    for s in range(steps):
        x = _decode_x(inputs["x"][s], inputs["x_dtype"], ch)
        fr = front(x, conv_w, cst, cu, ga[s][:, v_heads], gb[s][:, v_heads], A_log, dt_bias,
                   H_k=len(k_heads), H_v=len(v_heads), d_k=d_k, d_v=d_v, d_conv=d_conv,
                   eps=inputs["eps"], q_scale=inputs["q_scale"], threads=threads)
        cst = fr["conv_state"]
        qq, kk = fr["q"], fr["k"]
        if _layout(dims) & GQA_TILED:
            qq, kk = _repeat_tiled(qq, kk, len(v_heads))
        o, S = recurrence(qq, kk, fr["v"], fr["g"], fr["beta"], S, cu, threads=threads)
        outs.append(o)
    return dict(o=np.stack(outs), S=S, conv_state=cst, v_heads=v_heads, channels=ch)


def gated_norm(o, z, norm_w, eps):
    """out[t, h, :] = o[t, h, :] / sqrt(mean_j o[t, h, j]^2 + eps) * norm_w * z * sigmoid(z)
    over the value-head dimension, in fp64 (ik_llama.cpp src/llama-delta-net.cpp,
    build_layer_attn_linear_core: the RMS norm with the ssm_norm weight, shared by all value
    heads, then the product with SiLU(z)). Reading: eps is added to the mean of squares, as in
    an RMS norm; its value is the model's norm epsilon (1e-6 here)."""
    o = np.asarray(o, dtype=np.float64)
    z = np.asarray(z, dtype=np.float64)
    w = np.asarray(norm_w, dtype=np.float64)
    rms = np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps)
    silu = z / (1.0 + np.exp(-z))
    return o / rms * w * silu
