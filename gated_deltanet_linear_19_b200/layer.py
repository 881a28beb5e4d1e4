"""GatedDeltaNet layer object: per-slot state pools plus the front -> core call sequence.

Holds the recurrent-state pool [n_slots, H_v, d_k, d_v] (fp32) and the conv-state pool
[n_slots, d_conv-1, conv_dim] (bf16 by default), and runs, on the current torch stream,
  decode : gdn_layer_decode (the front with fp32 q/k/v, then the single-token step, in one
           call)
  prefill: gdn_layer_prefill (front inside the chunked prefill) where it applies (d = 128,
           d_conv = 4, bf16 x and conv state, fp16 operands), else gdn_conv_step (fp16
           q/k/v, fp32 for the precise path) -> gdn_chunked_prefill
Intermediate buffers are allocated through torch (cached per token count) and reused, so a
steady-state step allocates nothing. All arithmetic runs in libgdn.so.
"""
from __future__ import annotations

import torch

from . import (DecodePipe, GDN_PREFILL_OUT_GATE, GDN_PREFILL_RECURRENT, GDN_PREFILL_SIMT, Dims,
               chunked_prefill, conv_step, decode_workspace_size, front_outputs, gated_norm,
               layer_decode, layer_decode_plan, layer_prefill, prefill_workspace_size)


class GDNLayer:
    def __init__(self, dims: Dims, conv_w, A_log, dt_bias, *, eps=1e-6, q_scale=None,
                 device="cuda", conv_dtype=torch.bfloat16, prefill_qkv_dtype=torch.float16,
                 o_dtype=torch.bfloat16):
        self.dims = dims
        self.device = torch.device(device)
        self.eps = float(eps)
        self.q_scale = float(q_scale if q_scale is not None else dims.d_k ** -0.5)
        self.conv_w = None if conv_w is None else conv_w.to(self.device, torch.float32).contiguous()
        self.A_log = A_log.to(self.device, torch.float32).contiguous()
        self.dt_bias = dt_bias.to(self.device, torch.float32).contiguous()
        self.state = torch.zeros((dims.n_slots, dims.H_v, dims.d_k, dims.d_v),
                                 dtype=torch.float32, device=self.device)
        rows = max(dims.d_conv - 1, 0)
        self.conv_state = (torch.zeros((dims.n_slots, rows, dims.conv_dim), dtype=conv_dtype,
                                       device=self.device) if rows > 0 else None)
        self.prefill_qkv_dtype = prefill_qkv_dtype
        self.o_dtype = o_dtype
        self._bufs = {}

    # ------------------------------------------------------------------ buffers
    def _front_bufs(self, T: int, dtype):
        key = ("front", T, dtype)
        if key not in self._bufs:
            self._bufs[key] = front_outputs(self.dims, T, dtype, self.device)
        return self._bufs[key]

    def _out(self, T: int):
        key = ("o", T)
        if key not in self._bufs:
            self._bufs[key] = torch.empty((T, self.dims.H_v, self.dims.d_v), dtype=self.o_dtype,
                                          device=self.device)
        return self._bufs[key]

    def _workspace(self, T: int, n_seqs: int, chunk: int, dtype, flags: int):
        need = prefill_workspace_size(self.dims, T, n_seqs, chunk, dtype, flags)
        if need == 0:
            return None
        ws = self._bufs.get("ws")
        if ws is None or ws.numel() < need:
            ws = torch.empty(need, dtype=torch.uint8, device=self.device)
            self._bufs["ws"] = ws
        return ws

    # ------------------------------------------------------------------ steps
    def _decode_ws(self, B: int):
        key = ("dec_ws", B)
        if key not in self._bufs:
            self._bufs[key] = torch.empty(max(decode_workspace_size(self.dims, B), 1),
                                          dtype=torch.uint8, device=self.device)
        return self._bufs[key]

    def decode(self, x, a, b, slot_ids, *, reset=None, out=None, gate=None):
        """One token for each of B sequences: x [B, conv_dim], a/b [B, H_v] -> o [B, H_v, d_v].
        gate: an OutGate (z [B, H_v, d_v]) fused into the decode kernel."""
        B = x.shape[0]
        o = out if out is not None else self._out(B)
        layer_decode(self.dims, x, self.conv_w, self.conv_state, slot_ids, a, b, self.A_log,
                     self.dt_bias, self.state, o, eps=self.eps, q_scale=self.q_scale,
                     reset=reset, workspace=self._decode_ws(B), gate=gate)
        return o

    def decode_plan(self, x, a, b, slot_ids, *, reset=None, out=None, gate=None, stream=None):
        """decode on fixed buffers, marshalled once: returns (run, o) where run() issues the
        step (reading whatever x, a, b, slot_ids hold at that moment) and o receives it."""
        B = x.shape[0]
        o = out if out is not None else torch.empty((B, self.dims.H_v, self.dims.d_v),
                                                    dtype=self.o_dtype, device=self.device)
        run = layer_decode_plan(self.dims, x, self.conv_w, self.conv_state, slot_ids, a, b,
                                self.A_log, self.dt_bias, self.state, o, eps=self.eps,
                                q_scale=self.q_scale, reset=reset,
                                workspace=self._decode_ws(B), gate=gate, stream=stream)
        return run, o

    def decode_pipe(self, n_seqs, *, x_dtype=torch.bfloat16, stream=None):
        """A DecodePipe over this layer's pools: decode steps fed from and returned to host
        memory, the copies overlapped with the neighbouring steps."""
        return DecodePipe(self.dims, n_seqs, self.conv_w, self.conv_state, self.A_log,
                          self.dt_bias, self.state, x_dtype=x_dtype, o_dtype=self.o_dtype,
                          eps=self.eps, q_scale=self.q_scale, stream=stream)

    def fused_prefill_applies(self, x, chunk=64, flags=0, qkv_dtype=None) -> bool:
        d = self.dims
        dt = qkv_dtype or self.prefill_qkv_dtype
        return (d.d_k == 128 and d.d_v == 128 and d.d_conv == 4 and chunk == 64
                and dt == torch.float16 and x.dtype == torch.bfloat16
                and self.conv_state is not None and self.conv_state.dtype == torch.bfloat16
                and not (flags & (GDN_PREFILL_SIMT | GDN_PREFILL_RECURRENT)))

    def prefill(self, x, a, b, cu_seqlens, slot_ids, *, reset=None, chunk=64, out=None,
                flags=0, qkv_dtype=None, fused=None, gate=None):
        """Packed sequences: x [T, conv_dim], a/b [T, H_v], cu_seqlens [n+1] -> o [T, H_v, d_v].
        fused=None uses gdn_layer_prefill where it applies, False forces the two calls.
        gate: an OutGate (z [T, H_v, d_v]) applied to o in place after the prefill."""
        T = x.shape[0]
        if fused is None:
            fused = self.fused_prefill_applies(x, chunk, flags, qkv_dtype)
        if fused:
            o = out if out is not None else self._out(T)
            ws = self._workspace(T, cu_seqlens.numel() - 1, chunk, torch.float16,
                                 GDN_PREFILL_OUT_GATE if gate is not None else 0)
            layer_prefill(self.dims, x, self.conv_w, self.conv_state, cu_seqlens, slot_ids, a, b,
                          self.A_log, self.dt_bias, self.state, o, eps=self.eps,
                          q_scale=self.q_scale, chunk=chunk, reset=reset, workspace=ws,
                          flags=flags, gate=gate)
            return o
        dt = qkv_dtype or self.prefill_qkv_dtype
        q, k, v, g, beta = self._front_bufs(T, dt)
        conv_step(self.dims, x, self.conv_w, self.conv_state, cu_seqlens, slot_ids, a, b,
                  self.A_log, self.dt_bias, q, k, v, g, beta, eps=self.eps,
                  q_scale=self.q_scale, reset=reset)
        o = out if out is not None else self._out(T)
        ws = self._workspace(T, cu_seqlens.numel() - 1, chunk, dt, flags)
        # with an output gate the core writes fp32 first, so that o is rounded only once
        core_o = o if gate is None else torch.empty(o.shape, dtype=torch.float32,
                                                    device=self.device)
        chunked_prefill(self.dims, q, k, v, g, beta, self.state, slot_ids, cu_seqlens, core_o,
                        chunk=chunk, reset=reset, workspace=ws, flags=flags)
        if gate is not None:
            gated_norm(self.dims, core_o, gate, o)
        return o
