"""GPU parity of the decode step (gdn_conv_step + gdn_decode_step) against the fp64 oracle
at the Qwen3-Next layer shape (64 sequences, H_k=16 -> H_v=32, d=128)."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from gated_deltanet_linear_19_b200 import Dims, decode_step, device_status, front_outputs
from tests.gpu_util import bf16_floor, make_layer, rel_l2, t_bits, t_f32, t_i32

pytestmark = pytest.mark.gpu

TOL = 2e-3


def _run_steps(w, steps, o_dtype=torch.bfloat16, reset_first=None):
    layer = make_layer(w, o_dtype=o_dtype)
    slots = t_i32(w["slot_ids"])
    outs = []
    for s in range(steps):
        rs = None
        if reset_first is not None and s == 0:
            rs = torch.from_numpy(reset_first).cuda()
        o = layer.decode(t_bits(w["x"][s]), t_f32(w["a"][s]), t_f32(w["b"][s]), slots, reset=rs)
        outs.append(o.float().cpu().numpy())
    torch.cuda.synchronize()
    assert device_status() == 0
    return np.stack(outs), layer


def test_decode_8_steps_all_heads():
    w = synthetic.decode(steps=8)
    o, layer = _run_steps(w, 8)
    ref = oracle.decode_steps(w, 8)
    e_o, e_s = rel_l2(o, ref["o"]), rel_l2(layer.state.cpu().numpy(), ref["S"])
    floor = bf16_floor(ref["o"])
    print(f"decode 8 steps: rel_l2 o={e_o:.3e} (bf16 floor {floor:.3e}) S={e_s:.3e}")
    assert e_o < TOL and e_s < 1e-5
    conv = layer.conv_state.cpu().view(torch.int16).numpy().view(np.uint16)
    exp = synthetic.f32_to_bf16_bits(ref["conv_state"].astype(np.float32))
    np.testing.assert_array_equal(conv, exp)


def test_decode_256_steps_sampled_heads():
    w = synthetic.decode(steps=256)
    o, layer = _run_steps(w, 256)
    k_heads = [0, 9, 15]
    ref = oracle.decode_steps(w, 256, k_heads=k_heads)
    vh = ref["v_heads"]
    e_o = rel_l2(o[:, :, vh], ref["o"])
    e_s = rel_l2(layer.state.cpu().numpy()[:, vh], ref["S"])
    print(f"decode 256 steps (v-heads {vh}): rel_l2 o={e_o:.3e} S={e_s:.3e}")
    assert e_o < TOL and e_s < 1e-5


def test_decode_fp32_output_and_reset():
    w = synthetic.decode(steps=3, n_seqs=8, n_slots=8)
    rs = np.array([1, 0, 0, 1, 0, 0, 0, 1], np.uint8)
    o, layer = _run_steps(w, 3, o_dtype=torch.float32, reset_first=rs)
    w2 = dict(w)
    w2["state"] = w["state"].copy()
    w2["conv_state"] = w["conv_state"].copy()
    w2["state"][rs.astype(bool)] = 0
    w2["conv_state"][rs.astype(bool)] = 0
    ref = oracle.decode_steps(w2, 3)
    assert rel_l2(o, ref["o"]) < 1e-5
    assert rel_l2(layer.state.cpu().numpy(), ref["S"]) < 1e-5


def test_decode_noncontiguous_slots_touch_only_their_rows():
    w = synthetic.decode(steps=2, n_seqs=5, n_slots=12)
    w["slot_ids"] = np.array([11, 3, 7, 0, 5], np.int32)
    o, layer = _run_steps(w, 2, o_dtype=torch.float32)
    ref = oracle.decode_steps(w, 2)
    pool = layer.state.cpu().numpy()
    assert rel_l2(pool[w["slot_ids"]], ref["S"]) < 1e-5
    untouched = [s for s in range(12) if s not in set(w["slot_ids"].tolist())]
    np.testing.assert_array_equal(pool[untouched], w["state"][untouched])


def test_decode_is_deterministic():
    w = synthetic.decode(steps=2, n_seqs=16, n_slots=16)
    o1, l1 = _run_steps(w, 2)
    o2, l2 = _run_steps(w, 2)
    np.testing.assert_array_equal(o1, o2)
    assert torch.equal(l1.state, l2.state)


def test_decode_bad_and_duplicate_slots_set_status():
    dims = Dims(n_slots=4, H_k=2, H_v=4, d_k=128, d_v=128)
    q, k, v, g, beta = front_outputs(dims, 2)
    for t in (q, k, v, g, beta):
        t.zero_()
    state = torch.zeros((4, 4, 128, 128), device="cuda")
    o = torch.empty((2, 4, 128), device="cuda")
    decode_step(dims, q, k, v, g, beta, state, t_i32([0, 9]), o)
    assert device_status() == -2
    decode_step(dims, q, k, v, g, beta, state, t_i32([2, 2]), o)
    assert device_status() == -2
    decode_step(dims, q, k, v, g, beta, state, t_i32([2, 1]), o)
    assert device_status() == 0
