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


def layer(inputs: dict, threads=None, heads=None):
    """Front + recurrence over one synthetic workload dict (see ``synthetic``).

    Gathers the conv and recurrent states by slot, runs the oracle, and returns
    dict(o, S (per sequence), conv_state (per sequence), q, k, v, g, beta).
    ``heads``: optional list of v-heads to run the recurrence for (sampled parity on
    large workloads); the returned o and S then hold only those heads, in that order.
    """
    dims = inputs["dims"]
    H_k, H_v, d_k, d_v, d_conv = (dims[n] for n in ("H_k", "H_v", "d_k", "d_v", "d_conv"))
    cu = inputs["cu_seqlens"]
    slots = inputs["slot_ids"]
    reset = inputs.get("reset")
    if inputs["x_dtype"] == "bf16":
        x = bf16_bits_to_f64(inputs["x"])
    else:
        x = _f64(inputs["x"])
    conv_state = None
    if d_conv > 0:
        pool = inputs["conv_state"]
        pool = bf16_bits_to_f64(pool) if inputs["conv_state_dtype"] == "bf16" else _f64(pool)
        conv_state = pool[slots]
    fr = front(x, inputs.get("conv_w"), conv_state, cu, inputs["a"], inputs["b"],
               inputs["A_log"], inputs["dt_bias"], H_k=H_k, H_v=H_v, d_k=d_k, d_v=d_v,
               d_conv=d_conv, eps=inputs["eps"], q_scale=inputs["q_scale"], reset=reset,
               threads=threads)
    S0 = _f64(inputs["state"])[slots]
    if reset is not None:
        S0[np.asarray(reset, dtype=bool)] = 0.0
    q, k, v, g, beta = fr["q"], fr["k"], fr["v"], fr["g"], fr["beta"]
    if heads is not None:
        heads = list(heads)
        ratio = H_v // H_k
        kh = [h // ratio for h in heads]
        # each selected v-head keeps its own k-head: run with H_k' = H_v' = len(heads)
        q = q[:, kh, :]; k = k[:, kh, :]
        v = v[:, heads, :]; g = g[:, heads]; beta = beta[:, heads]
        S0 = S0[:, heads]
    o, S = recurrence(q, k, v, g, beta, S0, cu, threads=threads)
    return dict(o=o, S=S, conv_state=fr["conv_state"], q=fr["q"], k=fr["k"], v=fr["v"],
                g=fr["g"], beta=fr["beta"])
