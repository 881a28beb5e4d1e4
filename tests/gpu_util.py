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


def t_f32_or_none(a, device="cuda"):
    return None if a is None else t_f32(a, device)


def t_i32(a, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


def dims_of(w) -> Dims:
    d = w["dims"]
    return Dims(n_slots=d["n_slots"], H_k=d["H_k"], H_v=d["H_v"], d_k=d["d_k"], d_v=d["d_v"],
                d_conv=d["d_conv"], layout=d.get("layout", 0))


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
    o = layer.prefill(x_tensor(w), t_f32(w["a"]), t_f32_or_none(w["b"]), t_i32(w["cu_seqlens"]),
                      t_i32(w["slot_ids"]), reset=reset, chunk=kw.pop("chunk", w.get("chunk", 64)),
                      **kw)
    torch.cuda.synchronize()
    conv = None
    if layer.conv_state is not None:
        conv = layer.conv_state.cpu()
        conv = conv.view(torch.int16).numpy().view(np.uint16) \
            if conv.dtype == torch.bfloat16 else conv.numpy()
    return o.float().cpu().numpy(), layer.state.cpu().numpy(), conv, layer


def _bounds(ref, cu, chunk=None):
    """Row ranges of the groups: the sequences (cu), or with `chunk` the chunk-sized pieces
    of every sequence (the unit of the chunked algorithm)."""
    if cu is None:
        seqs = [(n, n + 1) for n in range(ref.shape[0])]
    else:
        cu = np.asarray(cu, dtype=np.int64)
        seqs = [(int(cu[n]), int(cu[n + 1])) for n in range(len(cu) - 1)]
    if chunk is None:
        return seqs
    return [(a + c, min(a + c + chunk, b)) for a, b in seqs for c in range(0, b - a, chunk)]


def group_norms(ref, cu=None, chunk=None):
    """L2 norm of ref per (group, head): [groups, H] (0 if empty)."""
    ref = np.asarray(ref, dtype=np.float64)
    bounds = _bounds(ref, cu, chunk)
    nrm = np.zeros((len(bounds), ref.shape[1]))
    for n, (a, b) in enumerate(bounds):
        if b > a:
            for h in range(ref.shape[1]):
                nrm[n, h] = np.linalg.norm(ref[a:b, h].ravel())
    return nrm


def head_rel(x, ref, cu=None, chunk=None, norm_floor=0.0):
    """Relative L2 error of x against ref per (group, head): [groups, H] (0 if empty).
    x, ref: [T, H, ...] token-major with sequence bounds cu, or [n_seqs, H, ...] (cu None);
    groups are sequences, or chunk-sized pieces of them. The denominator is at least
    norm_floor (a group whose reference nearly vanishes is judged against that scale)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    bounds = _bounds(ref, cu, chunk)
    rel = np.zeros((len(bounds), ref.shape[1]))
    for n, (a, b) in enumerate(bounds):
        if b <= a:
            continue
        for h in range(ref.shape[1]):
            r = ref[a:b, h].ravel()
            nr = max(np.linalg.norm(r), norm_floor)
            rel[n, h] = np.linalg.norm(x[a:b, h].ravel() - r) / (nr if nr > 0 else 1.0)
    return rel


def bf16_round(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def operand_ref(ref, w, vh=None):
    """The oracle's recurrence run on the fp16-rounded q, k, v of ref (oracle.layer output):
    what the tensor-core path, which takes its q, k, v operands in fp16, would give if
    everything after that rounding were exact."""
    import oracle
    r16 = lambda a: np.asarray(a).astype(np.float16).astype(np.float64)
    S0 = np.asarray(w["state"], dtype=np.float64)[w["slot_ids"]]
    if vh is not None:
        S0 = S0[:, vh]
    if w.get("reset") is not None:
        S0 = S0.copy()
        S0[np.asarray(w["reset"], dtype=bool)] = 0.0
    q, k = r16(ref["q"]), r16(ref["k"])
    if w["dims"].get("layout", 0) & 1:  # tiled GQA: key head h % H_k for value head h
        idx = [h % q.shape[1] for h in range(ref["v"].shape[1])]
        q, k = q[:, idx], k[:, idx]
    o16, _ = oracle.recurrence(q, k, r16(ref["v"]), ref["g"], ref["beta"], S0, w["cu_seqlens"])
    return o16


def _check_groups(x, ref, tol, cu, chunk, bf16_out, ref16, slack, label):
    # groups whose reference is below 1e-3 of the median group's norm (a state or output
    # that a degenerate gate has all but erased) are judged against that scale: relative to
    # itself, a nearly vanishing group only measures the rounding of the formats
    nrm = group_norms(ref, cu, chunk)
    nz = nrm[nrm > 0]
    floor = 1e-3 * float(np.median(nz)) if nz.size else 0.0
    rel = head_rel(x, ref, cu, chunk, floor)
    extra = np.zeros_like(rel)
    if bf16_out:
        extra += head_rel(bf16_round(ref), ref, cu, chunk, floor)
    if ref16 is not None:
        extra += head_rel(ref16, ref, cu, chunk, floor)
    bound = np.where(extra > 0, np.maximum(tol, extra + 5e-4), tol) * slack
    k = int((rel / bound).argmax())
    what = "chunk" if chunk else "seq"
    print(f"{label} per ({what}, head): worst rel_l2 {rel.max():.3e}; largest rel_l2/bound "
          f"{float((rel / bound).max()):.3f} at {np.unravel_index(k, rel.shape)} "
          f"(rel {rel.ravel()[k]:.3e}, bound {bound.ravel()[k]:.3e})")
    assert (rel - bound).max() < 0, (label, what, np.unravel_index(k, rel.shape),
                                     float(rel.ravel()[k]), float(bound.ravel()[k]))


def assert_heads(x, ref, tol, cu=None, label="", bf16_out=False, ref16=None, chunk=None):
    """Per (sequence, head) parity: relative L2 within a bound that is tol, raised where the
    unavoidable rounding of the formats alone comes close to it (bf16_out: the bf16 rounding
    of that group's own reference; ref16: the oracle run on fp16-rounded operands), plus 5e-4.
    With `chunk`, also every chunk-sized piece of every sequence, per head, within 1.5 times
    its own such bound: an error confined to one chunk cannot hide in a sequence's average."""
    _check_groups(x, ref, tol, cu, None, bf16_out, ref16, 1.0, label)
    if chunk is not None and cu is not None:
        _check_groups(x, ref, tol, cu, chunk, bf16_out, ref16, 1.5, label)
    return float(head_rel(x, ref, cu).max())


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
