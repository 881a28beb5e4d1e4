"""Helpers shared by the GPU parity tests: workload upload and error metrics."""
from __future__ import annotations

import numpy as np
import torch

from gated_deltanet_linear_19_b200 import Dims
from gated_deltanet_linear_19_b200.layer import GDNLayer


def rel_l2(x, ref) -> float:
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref.ravel())
    return float(np.linalg.norm((x - ref).ravel()) / (den if den > 0 else 1.0))


def bf16_floor(ref) -> float:
    """Relative L2 error of rounding the reference itself to bf16 (the output-format floor)."""
    r = torch.from_numpy(np.asarray(ref, dtype=np.float32)).to(torch.bfloat16).double().numpy()
    return rel_l2(r, ref)


def t_bits(a: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bit patterns -> torch.bfloat16 tensor (same bits)."""
    return torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).to(device)


def t_f32(a, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def t_i32(a, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


def dims_of(w) -> Dims:
    d = w["dims"]
    return Dims(n_slots=d["n_slots"], H_k=d["H_k"], H_v=d["H_v"], d_k=d["d_k"], d_v=d["d_v"],
                d_conv=d["d_conv"])


def make_layer(w, **kw) -> GDNLayer:
    """A layer holding the workload's weights and state pools (copied to the device)."""
    dims = dims_of(w)
    conv_w = None if w.get("conv_w") is None else t_f32(w["conv_w"])
    layer = GDNLayer(dims, conv_w, t_f32(w["A_log"]), t_f32(w["dt_bias"]), eps=w["eps"],
                     q_scale=w["q_scale"], **kw)
    layer.state.copy_(t_f32(w["state"]))
    if layer.conv_state is not None and w.get("conv_state") is not None:
        if layer.conv_state.dtype == torch.bfloat16:
            layer.conv_state.copy_(t_bits(w["conv_state"]))
        else:
            layer.conv_state.copy_(t_f32(w["conv_state"]))
    return layer


def x_tensor(w, x=None):
    x = w["x"] if x is None else x
    return t_bits(x) if w["x_dtype"] == "bf16" else t_f32(x)


def run_prefill(w, layer=None, **kw):
    """Front + chunked prefill of a packed workload; returns (o, state pool, conv pool, layer)."""
    layer = layer or make_layer(w)
    reset = None if w.get("reset") is None else \
        torch.from_numpy(np.asarray(w["reset"], np.uint8)).cuda()
    o = layer.prefill(x_tensor(w), t_f32(w["a"]), t_f32(w["b"]), t_i32(w["cu_seqlens"]),
                      t_i32(w["slot_ids"]), reset=reset, chunk=kw.pop("chunk", w.get("chunk", 64)),
                      **kw)
    torch.cuda.synchronize()
    conv = None
    if layer.conv_state is not None:
        conv = layer.conv_state.cpu()
        conv = conv.view(torch.int16).numpy().view(np.uint16) \
            if conv.dtype == torch.bfloat16 else conv.numpy()
    return o.float().cpu().numpy(), layer.state.cpu().numpy(), conv, layer
