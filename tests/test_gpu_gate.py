"""The layer's output gate RMSNorm(o) * norm_w * SiLU(z) (ik_llama.cpp
build_layer_attn_linear_core): fused into the decode kernel (the column tiles of a head
exchange their sums of squares within a thread-block cluster), after the layer prefill, and on
its own, against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from gated_deltanet_linear_19_b200 import OutGate, device_status, gated_norm
from tests.gpu_util import (assert_heads, by_sequence, dims_of, make_layer, operand_ref,
                            rel_l2, run_prefill, t_bits, t_f32, t_i32)

pytestmark = pytest.mark.gpu


def _gate(shape, d_v, seed, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    z = torch.randn(shape, generator=g).to(dtype)
    w = (1.0 + 0.1 * torch.randn(d_v, generator=g)).float()
    return z, w


@pytest.mark.parametrize("n_seqs", [4, 16])  # one-kernel layer decode / front + decode
@pytest.mark.parametrize("odt,tol", [(torch.float32, 1e-5), (torch.bfloat16, 2e-3)])
def test_decode_with_fused_gate(odt, tol, n_seqs):
    w = synthetic.decode(steps=3, n_seqs=n_seqs, n_slots=n_seqs)
    layer = make_layer(w, o_dtype=odt)
    dims = layer.dims
    slots = t_i32(w["slot_ids"])
    _, nw = _gate((1, dims.H_v, dims.d_v), dims.d_v, 99)
    zs, outs = [], []
    for s in range(3):
        z, _ = _gate((n_seqs, dims.H_v, dims.d_v), dims.d_v, 100 + s)
        zs.append(z.double().numpy())
        gate = OutGate(z.cuda(), nw.cuda(), 1e-6)
        outs.append(layer.decode(t_bits(w["x"][s]), t_f32(w["a"][s]), t_f32(w["b"][s]), slots,
                                 gate=gate).float().cpu().numpy())
    assert device_status() == 0
    ref = oracle.decode_steps(w, 3)
    exp = np.stack([oracle.gated_norm(ref["o"][s], zs[s], nw.double().numpy(), 1e-6)
                    for s in range(3)])
    o = np.stack(outs)
    e = rel_l2(o, exp)
    print(f"decode + gate ({odt}): {e:.3e}")
    assert e < tol
    og, cu = by_sequence(o)
    eg, _ = by_sequence(exp)
    assert_heads(og, eg, tol, cu=cu, label="decode gate", bf16_out=odt == torch.bfloat16)
    assert rel_l2(layer.state.cpu().numpy(), ref["S"]) < 1e-5


def test_layer_prefill_with_gate():
    lengths = [300, 77]
    w = synthetic.packed(lengths, seed=740, slots=[1, 0], state_std=0.02, conv_std=1.0,
                         n_slots=2)
    layer = make_layer(w)
    T = int(w["cu_seqlens"][-1])
    z, nw = _gate((T, layer.dims.H_v, layer.dims.d_v), layer.dims.d_v, 7)
    gate = OutGate(z.cuda(), nw.cuda(), 1e-6)
    o, S, _, _ = run_prefill(w, layer=layer, gate=gate)
    assert device_status() == 0
    ref = oracle.layer(w)
    exp = oracle.gated_norm(ref["o"], z.double().numpy(), nw.double().numpy(), 1e-6)
    e = rel_l2(o, exp)
    print(f"layer prefill + gate: {e:.3e}")
    assert e < 2e-3
    r16 = oracle.gated_norm(operand_ref(ref, w), z.double().numpy(), nw.double().numpy(), 1e-6)
    assert_heads(o, exp, 2e-3, cu=w["cu_seqlens"], label="prefill gate", bf16_out=True,
                 ref16=r16, chunk=64)


@pytest.mark.parametrize("d_v", [32, 64, 128])
@pytest.mark.parametrize("io", [(torch.float32, torch.float32), (torch.bfloat16, torch.bfloat16),
                                (torch.float32, torch.bfloat16)])
def test_gated_norm_kernel(d_v, io):
    from gated_deltanet_linear_19_b200 import Dims
    odt, zdt = io
    dims = Dims(n_slots=1, H_k=2, H_v=4, d_k=d_v, d_v=d_v)
    g = torch.Generator().manual_seed(d_v)
    T = 37
    o = (torch.randn((T, 4, d_v), generator=g) * 3.0).to(odt)
    z, nw = _gate((T, 4, d_v), d_v, d_v + 1, zdt)
    out = torch.empty_like(o, device="cuda")
    gated_norm(dims, o.cuda(), OutGate(z.cuda(), nw.cuda(), 1e-6), out)
    assert device_status() == 0
    exp = oracle.gated_norm(o.double().numpy(), z.double().numpy(), nw.double().numpy(), 1e-6)
    tol = 1e-5 if odt == torch.float32 else 2e-3
    assert_heads(out.float().cpu().numpy(), exp, tol, cu=np.arange(T + 1), label="gated_norm",
                 bf16_out=odt == torch.bfloat16)
    # in place
    oc = o.cuda()
    gated_norm(dims, oc, OutGate(z.cuda(), nw.cuda(), 1e-6))
    assert torch.equal(oc, out)
