"""B200 (sm_100a) gated delta-rule linear-attention layer (Gated DeltaNet).

Thin Python binding over the C ABI of libgdn.so (include/gdn.h). Every function marshals
torch CUDA tensors into pointers and calls the library on the current torch stream; all
arithmetic runs in the library's CUDA kernels. Functions raise ``GdnError`` on a non-OK
status. Same names as the C entry points, without the ``gdn_`` prefix.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import (GDN_BF16, GDN_EALIGN, GDN_ECUDA, GDN_EINVAL, GDN_ESLOT, GDN_ETIMEOUT,
                   GDN_EUNSUPPORTED, GDN_EWORKSPACE, GDN_F16, GDN_F32, GDN_GATES_MIXED_BA,
                   GDN_GQA_TILED, GDN_LAYOUT_DEFAULT, GDN_OK,
                   GDN_PREFILL_DEFAULT, GDN_PREFILL_OUT_GATE, GDN_PREFILL_RECURRENT,
                   GDN_PREFILL_SIMT, GDN_PREFILL_TC_HEAD_SCAN, GDN_PREFILL_TC_TILE_SCAN)

__all__ = ["Dims", "GdnError", "conv_step", "decode_step", "layer_decode",
           "layer_decode_plan", "layer_decode_launches", "gated_norm", "DecodePipe",
           "decode_pipe_buffer_size",
           "OutGate",
           "decode_workspace_size", "chunked_prefill", "layer_prefill",
           "chunked_prefill_noalloc", "prefill_workspace_size", "state_slot_copy", "device_status", "status_string",
           "front_outputs", "DTYPE_CODE"]

DTYPE_CODE = {torch.float32: GDN_F32, torch.bfloat16: GDN_BF16, torch.float16: GDN_F16}


class GdnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


@dataclass(frozen=True)
class Dims:
    n_slots: int
    H_k: int
    H_v: int
    d_k: int
    d_v: int
    d_conv: int = 4
    layout: int = GDN_LAYOUT_DEFAULT  # GDN_GQA_TILED | GDN_GATES_MIXED_BA

    @property
    def conv_dim(self) -> int:
        return 2 * self.H_k * self.d_k + self.H_v * self.d_v

    def c(self) -> _lib.GdnDims:
        return _lib.GdnDims(self.n_slots, self.H_k, self.H_v, self.d_k, self.d_v, self.d_conv,
                            self.layout)


def _p(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("gdn: tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("gdn: tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _code(t):
    return DTYPE_CODE[t.dtype]


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


@dataclass(frozen=True)
class OutGate:
    """The layer's output gate: RMSNorm(o) * norm_w * SiLU(z) (z token-major like o)."""
    z: torch.Tensor
    norm_w: torch.Tensor
    eps: float = 1e-6

    def c(self):
        return ctypes.byref(_lib.GdnOutGate(_p(self.z), _code(self.z), _p(self.norm_w),
                                            float(self.eps)))


def _gate(gate):
    return None if gate is None else gate.c()


def _check(rc: int, where: str):
    if rc != GDN_OK:
        raise GdnError(rc, where)


def status_string(status: int) -> str:
    return _lib.load().gdn_status_string(int(status)).decode()


def front_outputs(dims: Dims, T: int, dtype=torch.float32, device="cuda"):
    """Allocate q, k, v (dtype), g, beta (fp32) for T tokens."""
    q = torch.empty((T, dims.H_k, dims.d_k), dtype=dtype, device=device)
    k = torch.empty((T, dims.H_k, dims.d_k), dtype=dtype, device=device)
    v = torch.empty((T, dims.H_v, dims.d_v), dtype=dtype, device=device)
    g = torch.empty((T, dims.H_v), dtype=torch.float32, device=device)
    beta = torch.empty((T, dims.H_v), dtype=torch.float32, device=device)
    return q, k, v, g, beta


def conv_step(dims: Dims, x, conv_w, conv_state, cu_seqlens, slot_ids, a, b, A_log, dt_bias,
              q, k, v, g, beta, *, eps=1e-6, q_scale=None, reset=None, stream=None):
    """gdn_conv_step: conv1d + SiLU + L2 norm + gates for packed sequences (in place).
    cu_seqlens=None: one token per sequence (x has one row per slot id)."""
    lib = _lib.load()
    if q_scale is None:
        q_scale = dims.d_k ** -0.5
    n_seqs = cu_seqlens.numel() - 1 if cu_seqlens is not None else x.shape[0]
    rc = lib.gdn_conv_step(
        ctypes.byref(dims.c()), _p(x), _code(x), _p(conv_w), _p(conv_state),
        _code(conv_state) if conv_state is not None else GDN_F32, _p(cu_seqlens),
        _p(slot_ids), _p(reset), n_seqs, x.shape[0], _p(a), _p(b), _p(A_log), _p(dt_bias),
        float(eps), float(q_scale), _p(q), _p(k), _p(v), _code(q), _p(g), _p(beta),
        _stream(stream))
    _check(rc, "gdn_conv_step")


def decode_step(dims: Dims, q, k, v, g, beta, state, slot_ids, o, *, reset=None, stream=None):
    """gdn_decode_step: one token per sequence, state updated in place, o written."""
    lib = _lib.load()
    rc = lib.gdn_decode_step(ctypes.byref(dims.c()), _p(q), _p(k), _p(v), _code(q), _p(g),
                             _p(beta), _p(state), _p(slot_ids), _p(reset), slot_ids.numel(),
                             _p(o), _code(o), _stream(stream))
    _check(rc, "gdn_decode_step")


def decode_workspace_size(dims: Dims, n_seqs: int) -> int:
    lib = _lib.load()
    return int(lib.gdn_decode_workspace_size(ctypes.byref(dims.c()), int(n_seqs)))


def layer_decode_launches(dims: Dims, n_seqs: int, gated: bool = False) -> int:
    """Kernels one layer_decode call launches for n_seqs sequences (1, 2, or 3 with a gate)."""
    lib = _lib.load()
    return int(lib.gdn_layer_decode_launches(ctypes.byref(dims.c()), int(n_seqs), int(gated)))


def layer_decode(dims: Dims, x, conv_w, conv_state, slot_ids, a, b, A_log, dt_bias, state, o, *,
                 eps=1e-6, q_scale=None, reset=None, workspace=None, gate=None, stream=None):
    """gdn_layer_decode: front + single-token step for B sequences in one call
    (x [B, conv_dim] -> o [B, H_v, d_v]); allocates the workspace if not given. gate: an
    OutGate applied inside the decode kernel (o receives the gated output)."""
    lib = _lib.load()
    if q_scale is None:
        q_scale = dims.d_k ** -0.5
    n = slot_ids.numel()
    if workspace is None:
        workspace = torch.empty(max(decode_workspace_size(dims, n), 1), dtype=torch.uint8,
                                device=x.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib.gdn_layer_decode(ctypes.byref(dims.c()), _p(x), _code(x), _p(conv_w),
                              _p(conv_state),
                              _code(conv_state) if conv_state is not None else GDN_F32,
                              _p(slot_ids), _p(reset), n, _p(a), _p(b), _p(A_log), _p(dt_bias),
                              float(eps), float(q_scale), _p(state), _p(o), _code(o),
                              _p(workspace), ws_bytes, _gate(gate), _stream(stream))
    _check(rc, "gdn_layer_decode")


def layer_decode_plan(dims: Dims, x, conv_w, conv_state, slot_ids, a, b, A_log, dt_bias, state,
                      o, *, eps=1e-6, q_scale=None, reset=None, workspace=None, gate=None,
                      stream=None):
    """layer_decode with every argument marshalled once: returns a callable that issues
    gdn_layer_decode on the same buffers (their contents may change between calls) and the
    given stream (the current one at plan time if None). For a step loop over fixed buffers,
    where the per-call argument checks and conversions would cost more host time than the
    GPU step."""
    lib = _lib.load()
    if q_scale is None:
        q_scale = dims.d_k ** -0.5
    n = slot_ids.numel()
    if workspace is None:
        workspace = torch.empty(max(decode_workspace_size(dims, n), 1), dtype=torch.uint8,
                                device=x.device)
    cdims = dims.c()
    cgate = _gate(gate)  # keeps its struct alive
    keep = (cdims, cgate, gate, workspace, x, conv_w, conv_state, slot_ids, reset, a, b, A_log,
            dt_bias, state, o)
    args = (ctypes.byref(cdims), _p(x), _code(x), _p(conv_w), _p(conv_state),
            _code(conv_state) if conv_state is not None else GDN_F32, _p(slot_ids), _p(reset), n,
            _p(a), _p(b), _p(A_log), _p(dt_bias), ctypes.c_float(eps), ctypes.c_float(q_scale),
            _p(state), _p(o), _code(o), _p(workspace),
            ctypes.c_size_t(workspace.numel() * workspace.element_size()), cgate,
            _stream(stream))
    fn = lib.gdn_layer_decode

    def run():
        rc = fn(*args)
        if rc != GDN_OK:
            raise GdnError(rc, "gdn_layer_decode")
        return keep  # the buffers stay referenced as long as the plan is

    return run


def decode_pipe_buffer_size(dims: Dims, n_seqs: int, x_dtype=torch.bfloat16,
                            o_dtype=torch.bfloat16) -> int:
    return int(_lib.load().gdn_decode_pipe_buffer_size(ctypes.byref(dims.c()), int(n_seqs),
                                                       DTYPE_CODE[x_dtype],
                                                       DTYPE_CODE[o_dtype]))


def _host_ptr(t):
    if t is None:
        return None
    if t.is_cuda:
        raise ValueError("gdn: the decode pipeline takes host tensors")
    if not t.is_contiguous():
        raise ValueError("gdn: tensors must be contiguous")
    return t.data_ptr()


class DecodePipe:
    """gdn_decode_pipe_*: the layer decode step fed from and returned to host memory, the
    copies on the pipeline's own streams, overlapped with the neighbouring steps (two staging
    sets in one device buffer). step() takes HOST tensors (pinned for asynchronous copies)
    that must stay unchanged until the step's copies have run; flush() makes the compute
    stream wait for every copy issued so far."""

    def __init__(self, dims: Dims, n_seqs: int, conv_w, conv_state, A_log, dt_bias, state, *,
                 x_dtype=torch.bfloat16, o_dtype=torch.bfloat16, eps=1e-6, q_scale=None,
                 stream=None):
        lib = _lib.load()
        if q_scale is None:
            q_scale = dims.d_k ** -0.5
        size = decode_pipe_buffer_size(dims, n_seqs, x_dtype, o_dtype)
        if size == 0:
            raise GdnError(GDN_EINVAL, "gdn_decode_pipe_buffer_size")
        # allocated on the compute stream, so that the caching allocator reuses it only after
        # the steps enqueued there
        s_obj = stream if stream is not None else torch.cuda.current_stream(state.device)
        with torch.cuda.stream(s_obj):
            self.buffer = torch.empty(size, dtype=torch.uint8, device=state.device)
        self._keep = (conv_w, conv_state, A_log, dt_bias, state)
        self.packed_bytes = int(lib.gdn_decode_pipe_packed_bytes(ctypes.byref(dims.c()),
                                                                 int(n_seqs),
                                                                 DTYPE_CODE[x_dtype]))
        up = lambda v: (v + 255) // 256 * 256  # noqa: E731
        xb = n_seqs * dims.conv_dim * torch.empty((), dtype=x_dtype).element_size()
        mixed = (dims.layout & GDN_GATES_MIXED_BA) != 0
        ab = n_seqs * dims.H_v * 4
        oa = up(xb)
        ob = oa + up(ab * (2 if mixed else 1))
        osl = ob + (0 if mixed else up(ab))
        # byte offsets of x, a, b (None with the fused beta/alpha layout) and the slot ids
        self.packed_offsets = (0, oa, None if mixed else ob, osl)
        assert self.packed_bytes == osl + n_seqs * 4, "packed row layout out of step"
        self._lib = lib
        self.n_seqs = n_seqs
        h = ctypes.c_void_p()
        rc = lib.gdn_decode_pipe_create(
            ctypes.byref(dims.c()), int(n_seqs), DTYPE_CODE[x_dtype], _p(conv_w), _p(conv_state),
            _code(conv_state) if conv_state is not None else GDN_F32, _p(A_log), _p(dt_bias),
            ctypes.c_float(eps), ctypes.c_float(q_scale), _p(state), DTYPE_CODE[o_dtype],
            _p(self.buffer), ctypes.c_size_t(size), ctypes.c_void_p(s_obj.cuda_stream),
            ctypes.byref(h))
        _check(rc, "gdn_decode_pipe_create")
        self._h = h

    def step_ptrs(self, x, a, b, slot_ids, reset, o):
        """step() on raw host addresses (ints; b, reset may be None)."""
        rc = self._lib.gdn_decode_pipe_step(self._h, x, a, b, slot_ids, reset, o)
        if rc != GDN_OK:
            raise GdnError(rc, "gdn_decode_pipe_step")

    def step_packed_ptr(self, row, reset, o):
        """gdn_decode_pipe_step_packed on raw host addresses (ints; reset may be None): x, a,
        b and the slot ids in one host row laid out as packed_offsets() gives."""
        rc = self._lib.gdn_decode_pipe_step_packed(self._h, row, reset, o)
        if rc != GDN_OK:
            raise GdnError(rc, "gdn_decode_pipe_step_packed")

    def step(self, x, a, b, slot_ids, o, reset=None):
        self.step_ptrs(_host_ptr(x), _host_ptr(a), _host_ptr(b), _host_ptr(slot_ids),
                       _host_ptr(reset), _host_ptr(o))

    def flush(self):
        _check(self._lib.gdn_decode_pipe_flush(self._h), "gdn_decode_pipe_flush")

    def close(self):
        """Release the pipeline; its buffer is freed by torch's caching allocator in stream
        order, after the last step on the compute stream."""
        h, self._h = getattr(self, "_h", None), None
        if h:
            _check(self._lib.gdn_decode_pipe_destroy(h), "gdn_decode_pipe_destroy")

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def gated_norm(dims: Dims, o, gate: OutGate, out=None, *, stream=None):
    """gdn_gated_norm: out = RMSNorm(o) * norm_w * SiLU(z) per (token, value head); in place
    when out is None or o."""
    lib = _lib.load()
    out = o if out is None else out
    rc = lib.gdn_gated_norm(ctypes.byref(dims.c()), _p(o), _code(o), gate.c(), _p(out),
                            _code(out), o.shape[0], _stream(stream))
    _check(rc, "gdn_gated_norm")
    return out


def prefill_workspace_size(dims: Dims, T_total: int, n_seqs: int, chunk: int = 64,
                           qkv_dtype=torch.float16, flags: int = 0) -> int:
    lib = _lib.load()
    return int(lib.gdn_prefill_workspace_size(ctypes.byref(dims.c()), int(T_total), int(n_seqs),
                                              int(chunk), DTYPE_CODE[qkv_dtype], int(flags)))


def chunked_prefill(dims: Dims, q, k, v, g, beta, state, slot_ids, cu_seqlens, o, *,
                    chunk=64, reset=None, workspace=None, flags=0, stream=None):
    """gdn_chunked_prefill over packed sequences; allocates the workspace if not given."""
    lib = _lib.load()
    n_seqs = cu_seqlens.numel() - 1
    T = q.shape[0]
    if workspace is None:
        need = prefill_workspace_size(dims, T, n_seqs, chunk, q.dtype, flags)
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device) \
            if need > 0 else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    rc = lib.gdn_chunked_prefill(ctypes.byref(dims.c()), _p(q), _p(k), _p(v), _code(q), _p(g),
                                 _p(beta), _p(state), _p(slot_ids), _p(cu_seqlens), _p(reset),
                                 n_seqs, T, int(chunk), _p(o), _code(o), _p(workspace),
                                 ws_bytes, int(flags), _stream(stream))
    _check(rc, "gdn_chunked_prefill")


def layer_prefill(dims: Dims, x, conv_w, conv_state, cu_seqlens, slot_ids, a, b, A_log, dt_bias,
                  state, o, *, eps=1e-6, q_scale=None, chunk=64, reset=None, workspace=None,
                  flags=0, gate=None, stream=None):
    """gdn_layer_prefill: the front applied inside the chunked prefill, x -> o in one call
    (q, k, v, g, beta are never written); allocates the workspace if not given."""
    lib = _lib.load()
    if q_scale is None:
        q_scale = dims.d_k ** -0.5
    n_seqs = cu_seqlens.numel() - 1
    T = x.shape[0]
    if workspace is None:
        need = prefill_workspace_size(dims, T, n_seqs, chunk, torch.float16,
                                      GDN_PREFILL_OUT_GATE if gate is not None else 0)
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device) \
            if need > 0 else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    rc = lib.gdn_layer_prefill(ctypes.byref(dims.c()), _p(x), _code(x), _p(conv_w),
                               _p(conv_state), _code(conv_state), _p(cu_seqlens), _p(slot_ids),
                               _p(reset), n_seqs, T, _p(a), _p(b), _p(A_log), _p(dt_bias),
                               float(eps), float(q_scale), _p(state), int(chunk), _p(o), _code(o),
                               _p(workspace), ws_bytes, int(flags), _gate(gate), _stream(stream))
    _check(rc, "gdn_layer_prefill")


def chunked_prefill_noalloc(dims: Dims, q, k, v, g, beta, state, slot_ids, cu_seqlens, o, *,
                            chunk=64, reset=None, stream=None):
    """gdn_chunked_prefill_noalloc: the tensor-core prefill using the library's fixed device
    scratch instead of a workspace, for callers that cannot allocate device memory."""
    lib = _lib.load()
    n_seqs = cu_seqlens.numel() - 1
    rc = lib.gdn_chunked_prefill_noalloc(ctypes.byref(dims.c()), _p(q), _p(k), _p(v), _code(q),
                                         _p(g), _p(beta), _p(state), _p(slot_ids),
                                         _p(cu_seqlens), _p(reset), n_seqs, q.shape[0],
                                         int(chunk), _p(o), _code(o), _stream(stream))
    _check(rc, "gdn_chunked_prefill_noalloc")


def state_slot_copy(dims: Dims, state, conv_state, src, dst, *, stream=None):
    """gdn_state_slot_copy: state[dst[i]] = state[src[i]] (and conv state), bit-exact."""
    lib = _lib.load()
    rc = lib.gdn_state_slot_copy(ctypes.byref(dims.c()), _p(state), _p(conv_state),
                                 _code(conv_state) if conv_state is not None else GDN_F32,
                                 _p(src), _p(dst), src.numel(), _stream(stream))
    _check(rc, "gdn_state_slot_copy")


def device_status(clear: bool = True, stream=None) -> int:
    """Synchronise the stream and return (optionally clearing) the device status word."""
    lib = _lib.load()
    out = ctypes.c_int32(0)
    rc = lib.gdn_device_status(ctypes.byref(out), 1 if clear else 0, _stream(stream))
    _check(rc, "gdn_device_status")
    return int(out.value)
