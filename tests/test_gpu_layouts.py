"""The other weight family's layouts (ik_llama.cpp build_layer_attn_linear_core /
build_layer_attn_linear): key heads repeated to the value heads tiled (value head h reads
key head h % H_k) instead of grouped, and the gate inputs as the fused beta/alpha projection
[T, H_k, 2 r] instead of separate a, b. Decode, both prefill paths and the front, against the
oracle run with the same layout."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from gated_deltanet_linear_19_b200 import device_status
from tests.gpu_util import (assert_heads, by_sequence, make_layer, operand_ref, rel_l2,
                            run_prefill, t_bits, t_f32, t_f32_or_none, t_i32)

pytestmark = pytest.mark.gpu

LAYOUTS = [synthetic.GQA_TILED, synthetic.GATES_MIXED_BA,
           synthetic.GQA_TILED | synthetic.GATES_MIXED_BA]


@pytest.mark.parametrize("layout", LAYOUTS)
def test_layer_decode_layouts(layout):
    w = synthetic.decode(steps=3, n_seqs=8, n_slots=8, H_k=4, H_v=8, layout=layout)
    layer = make_layer(w, o_dtype=torch.float32)
    slots = t_i32(w["slot_ids"])
    outs = []
    for s in range(3):
        b = None if w["b"] is None else t_f32(w["b"][s])
        outs.append(layer.decode(t_bits(w["x"][s]), t_f32(w["a"][s]), b, slots).cpu().numpy())
    assert device_status() == 0
    ref = oracle.decode_steps(w, 3)
    o = np.stack(outs)
    assert rel_l2(o, ref["o"]) < 1e-5
    assert rel_l2(layer.state.cpu().numpy(), ref["S"]) < 1e-5
    og, cu = by_sequence(o)
    rg, _ = by_sequence(ref["o"])
    assert_heads(og, rg, 1e-5, cu=cu, label=f"decode layout {layout}")


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("fused", [None, False])
def test_prefill_layouts(layout, fused):
    """fused=None: gdn_layer_prefill (front inside the prep); False: gdn_conv_step +
    gdn_chunked_prefill (the short sequence takes the token-by-token kernel)."""
    lengths = [300, 5, 129]
    w = synthetic.packed(lengths, seed=720 + layout, slots=[2, 0, 1], state_std=0.02,
                         conv_std=1.0, n_slots=3, H_k=4, H_v=8, layout=layout)
    o, S, conv, _ = run_prefill(w, fused=fused)
    assert device_status() == 0
    ref = oracle.layer(w)
    e_o, e_s = rel_l2(o, ref["o"]), rel_l2(S[w["slot_ids"]], ref["S"])
    print(f"prefill layout {layout} fused={fused}: o {e_o:.3e} S {e_s:.3e}")
    assert e_o < 2e-3 and e_s < 2e-3
    cu = w["cu_seqlens"]
    assert_heads(o, ref["o"], 2e-3, cu=cu, label=f"prefill layout {layout}", bf16_out=True,
                 ref16=operand_ref(ref, w), chunk=64)
    assert_heads(S[w["slot_ids"]], ref["S"], 2e-3, label=f"prefill layout {layout} S")
    np.testing.assert_array_equal(conv[w["slot_ids"]],
                                  synthetic.f32_to_bf16_bits(ref["conv_state"].astype(np.float32)))


def test_front_mixed_gates():
    from gated_deltanet_linear_19_b200 import conv_step
    from tests.gpu_util import dims_of
    w = synthetic.packed([3, 40], seed=730, slots=[1, 0], conv_std=1.0, n_slots=2, H_k=4,
                         H_v=8, layout=synthetic.GATES_MIXED_BA)
    layer = make_layer(w)
    T = int(w["cu_seqlens"][-1])
    q, k, v, g, beta = layer._front_bufs(T, torch.float32)
    conv_step(layer.dims, t_bits(w["x"]), layer.conv_w, layer.conv_state, t_i32(w["cu_seqlens"]),
              t_i32(w["slot_ids"]), t_f32(w["a"]), None, layer.A_log, layer.dt_bias,
              q, k, v, g, beta, eps=w["eps"], q_scale=w["q_scale"])
    assert device_status() == 0
    ref = oracle.layer(w)
    assert rel_l2(g.cpu().numpy(), ref["g"]) < 2e-6
    assert rel_l2(beta.cpu().numpy(), ref["beta"]) < 2e-6
    assert rel_l2(v.cpu().numpy(), ref["v"]) < 2e-6
