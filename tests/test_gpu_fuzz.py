"""Seeded random mixed batches against the fp64 oracle: sequence counts on both sides of the
short-path grid limits, lengths from empty through the 16-token routing edge to several
chunks, random slots, resets, weight layouts and output gates, through both prefill paths
(gdn_layer_prefill and gdn_conv_step + gdn_chunked_prefill). Each case checks every
(sequence, head) and every chunk against the oracle, the conv state bit for bit and the pool
rows no sequence owns."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from gated_deltanet_linear_19_b200 import OutGate, device_status
from tests.gpu_util import assert_heads, make_layer, operand_ref, run_prefill

pytestmark = pytest.mark.gpu

LAYOUTS = [0, synthetic.GQA_TILED, synthetic.GATES_MIXED_BA,
           synthetic.GQA_TILED | synthetic.GATES_MIXED_BA]


def _case(seed):
    r = np.random.default_rng(9000 + seed)
    n = int(r.choice([1, 2, 5, 9, 10, 14]))
    pick = r.random(n)
    lengths = [0 if p < 0.1 else int(r.integers(1, 17)) if p < 0.55 else
               int(r.choice([17, 63, 64, 65, 129, 200])) for p in pick]
    n_slots = n + int(r.integers(0, 4))
    slots = r.permutation(n_slots)[:n].tolist()
    reset = (r.random(n) < 0.3).astype(np.uint8).tolist()
    layout = LAYOUTS[int(r.integers(0, len(LAYOUTS)))]
    fused = None if r.random() < 0.6 else False
    gated = bool(r.random() < 0.3)
    return lengths, slots, n_slots, reset, layout, fused, gated


@pytest.mark.parametrize("seed", range(12))
def test_random_mixed_batch(seed):
    lengths, slots, n_slots, reset, layout, fused, gated = _case(seed)
    w = synthetic.packed(lengths, seed=800 + seed, slots=slots, state_std=0.02, conv_std=1.0,
                         n_slots=n_slots, layout=layout)
    w["reset"] = np.array(reset, np.uint8)
    T = int(w["cu_seqlens"][-1])
    dims = w["dims"]
    gated = gated and T > 0
    gate, z, nw = None, None, None
    if gated:
        g = torch.Generator().manual_seed(seed)
        z = torch.randn((max(T, 1), dims["H_v"], dims["d_v"]), generator=g)[:T]
        nw = 1.0 + 0.1 * torch.randn(dims["d_v"], generator=g)
        gate = OutGate(z.cuda().contiguous(), nw.cuda(), 1e-6)
    layer = make_layer(w)
    o, S, conv, _ = run_prefill(w, layer=layer, fused=fused, gate=gate)
    assert device_status() == 0, (lengths, slots)
    ref = oracle.layer(w)
    exp = ref["o"]
    if gated:
        exp = oracle.gated_norm(ref["o"], z.double().numpy(), nw.double().numpy(), 1e-6)
    label = f"fuzz {seed} n={len(lengths)} lengths={lengths} fused={fused} gated={gated}"
    if T > 0:
        # the floor of the fp16 q, k, v operands, through the gate when there is one (the
        # gate normalises each (token, head) row, so a row's relative error carries over)
        r16 = operand_ref(ref, w)
        if gated:
            r16 = oracle.gated_norm(r16, z.double().numpy(), nw.double().numpy(), 1e-6)
        assert_heads(o, exp, 2e-3, cu=w["cu_seqlens"], label=label, bf16_out=True, ref16=r16,
                     chunk=64)
    assert_heads(S[w["slot_ids"]], ref["S"], 2e-3, label=label + " S")
    np.testing.assert_array_equal(conv[w["slot_ids"]],
                                  synthetic.f32_to_bf16_bits(ref["conv_state"].astype(np.float32)))
    others = [s for s in range(n_slots) if s not in set(slots)]
    np.testing.assert_array_equal(S[others], w["state"][others])


@pytest.mark.parametrize("seed", range(8))
def test_random_decode_steps(seed):
    """Random batch sizes on both sides of the one-kernel layer decode's limit (9 sequences at
    H_v = 32: one kernel; 10 and more: front + decode), layouts, resets and gates, over 3
    steps against the oracle."""
    from tests.gpu_util import by_sequence, t_bits, t_f32, t_f32_or_none, t_i32
    r = np.random.default_rng(9500 + seed)
    B = int(r.choice([1, 3, 8, 9, 10, 17, 40]))
    layout = LAYOUTS[int(r.integers(0, len(LAYOUTS)))]
    gated = bool(r.random() < 0.4)
    n_slots = B + int(r.integers(0, 5))
    w = synthetic.decode(seed=700 + seed, steps=3, n_seqs=B, n_slots=n_slots, layout=layout)
    w["slot_ids"] = r.permutation(n_slots)[:B].astype(np.int32)
    rst = (r.random(B) < 0.3).astype(np.uint8)
    layer = make_layer(w, o_dtype=torch.float32)
    dims = layer.dims
    slots = t_i32(w["slot_ids"])
    g = torch.Generator().manual_seed(seed)
    nw = (1.0 + 0.1 * torch.randn(dims.d_v, generator=g)).float()
    outs, zs = [], []
    for s in range(3):
        gate = None
        if gated:
            z = torch.randn((B, dims.H_v, dims.d_v), generator=g)
            zs.append(z.double().numpy())
            gate = OutGate(z.cuda(), nw.cuda(), 1e-6)
        reset = torch.from_numpy(rst).cuda() if s == 0 else None
        outs.append(layer.decode(t_bits(w["x"][s]), t_f32(w["a"][s]), t_f32_or_none(
            None if w["b"] is None else w["b"][s]), slots, reset=reset, gate=gate)
            .float().cpu().numpy())
    assert device_status() == 0
    # the oracle from the first step's effective states: rows of reset sequences zeroed
    keep = (rst == 0)[:, None, None, None]
    S0 = np.asarray(w["state"], np.float64)[w["slot_ids"]] * keep
    c0 = oracle.bf16_bits_to_f64(np.asarray(w["conv_state"])[w["slot_ids"]]) * keep[..., 0]
    ref = oracle.decode_steps(w, 3, S0=S0, conv_state0=c0)
    exp = ref["o"]
    if gated:
        exp = np.stack([oracle.gated_norm(ref["o"][s], zs[s], nw.double().numpy(), 1e-6)
                        for s in range(3)])
    o = np.stack(outs)
    og, cu = by_sequence(o)
    eg, _ = by_sequence(exp)
    label = f"fuzz decode {seed} B={B} layout={layout} gated={gated}"
    assert_heads(og, eg, 1e-5 if not gated else 2e-5, cu=cu, label=label)
    assert_heads(layer.state.cpu().numpy()[w["slot_ids"]], ref["S"], 1e-5, label=label + " S")
    conv = layer.conv_state.cpu().view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(conv[w["slot_ids"]],
                                  synthetic.f32_to_bf16_bits(ref["conv_state"].astype(np.float32)))
