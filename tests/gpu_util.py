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


def head_errors(x, ref, cu=None):
    """Per (sequence, head) errors of x against ref.

    x, ref: [T, H, ...] token-major with sequence bounds cu (rows cu[n]:cu[n+1] are sequence
    n), or [n_seqs, H, ...] per sequence when cu is None. Returns three arrays [n_seqs, H]:
    the relative L2 error, the max absolute error divided by the RMS of ref over that
    (sequence, head), and the relative L2 error of ref itself rounded to bf16 (the floor a
    bf16 output cannot go below). Empty sequences give 0."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if cu is None:
        bounds = [(n, n + 1) for n in range(ref.shape[0])]
    else:
        cu = np.asarray(cu, dtype=np.int64)
        bounds = [(int(cu[n]), int(cu[n + 1])) for n in range(len(cu) - 1)]
    H = ref.shape[1]
    ref_bf16 = torch.from_numpy(ref.astype(np.float32)).to(torch.bfloat16).double().numpy()
    rel = np.zeros((len(bounds), H))
    mx = np.zeros((len(bounds), H))
    floor = np.zeros((len(bounds), H))
    for n, (a, b) in enumerate(bounds):
        if b <= a:
            continue
        for h in range(H):
            r = ref[a:b, h].ravel()
            d = x[a:b, h].ravel() - r
            nr = np.linalg.norm(r)
            den = nr if nr > 0 else 1.0
            rms = nr / np.sqrt(r.size)
            rel[n, h] = np.linalg.norm(d) / den
            mx[n, h] = np.abs(d).max() / (rms if rms > 0 else 1.0)
            floor[n, h] = np.linalg.norm(ref_bf16[a:b, h].ravel() - r) / den
    return rel, mx, floor


def assert_heads(x, ref, tol, cu=None, max_abs=None, label="", bf16_out=False):
    """Every (sequence, head) within relative L2 `tol` and (if given) every element within
    `max_abs` times the RMS of ref over its (sequence, head). With bf16_out, a (sequence,
    head) whose own bf16 rounding floor is close to or above tol (a few tokens only) may
    exceed tol by at most 5e-4 beyond that floor: the rounding of the output format itself
    cannot be undone. Returns the worst values."""
    rel, mx, floor = head_errors(x, ref, cu)
    bound = np.full_like(rel, tol)
    if bf16_out:
        bound = np.maximum(bound, floor + 5e-4)
    excess = rel - bound
    worst_rel, worst_mx = float(rel.max()), float(mx.max())
    print(f"{label} per (seq, head): worst rel_l2 {worst_rel:.3e} (its floor "
          f"{float(floor.ravel()[rel.argmax()]):.3e}), worst max|err|/rms {worst_mx:.3e}")
    assert excess.max() < 0, (label, np.unravel_index(excess.argmax(), rel.shape),
                              float(rel.ravel()[excess.argmax()]),
                              float(bound.ravel()[excess.argmax()]))
    if max_abs is not None:
        assert worst_mx < max_abs, (label, np.unravel_index(mx.argmax(), mx.shape), worst_mx)
    return worst_rel, worst_mx


def by_sequence(o_steps):
    """Decode outputs [steps, B, H, d] -> ([B * steps, H, d], cu) grouped per sequence."""
    st, B = o_steps.shape[:2]
    o = np.ascontiguousarray(np.swapaxes(np.asarray(o_steps), 0, 1)).reshape(B * st,
                                                                              *o_steps.shape[2:])
    return o, np.arange(0, B * st + 1, st)


def subset_packed(w, keep):
    """The packed workload restricted to the sequences in `keep` (same pools and weights):
    the expected result of a call in which only those sequences run."""
    cu = np.asarray(w["cu_seqlens"], dtype=np.int64)
    rows = np.concatenate([np.arange(cu[n], cu[n + 1]) for n in keep]).astype(np.int64)
    lens = [int(cu[n + 1] - cu[n]) for n in keep]
    sub = dict(w)
    sub["x"] = np.asarray(w["x"])[rows]
    sub["a"] = np.asarray(w["a"])[rows]
    sub["b"] = np.asarray(w["b"])[rows]
    sub["cu_seqlens"] = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    sub["slot_ids"] = np.asarray(w["slot_ids"])[list(keep)].astype(np.int32)
    if w.get("reset") is not None:
        sub["reset"] = np.asarray(w["reset"])[list(keep)]
    return sub, rows
