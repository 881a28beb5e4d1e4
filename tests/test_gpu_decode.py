"""GPU parity of the decode step (gdn_conv_step + gdn_decode_step) against the fp64 oracle
at the Qwen3-Next layer shape (64 sequences, H_k=16 -> H_v=32, d=128)."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from gated_deltanet_linear_19_b200 import (Dims, conv_step, decode_step, device_status,
                                           front_outputs, state_slot_copy)
from tests.gpu_util import (assert_heads, bf16_floor, by_sequence, dims_of, make_layer, rel_l2,
                            t_bits, t_f32, t_i32)

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
    # every (sequence, value head) on its own, over its 8 tokens
    og, cu = by_sequence(o)
    rg, _ = by_sequence(ref["o"])
    assert_heads(og, rg, TOL, cu=cu, label="decode 8 steps o", bf16_out=True)
    assert_heads(layer.state.cpu().numpy(), ref["S"], 1e-5, label="decode 8 steps S")
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
    og, cu = by_sequence(o[:, :, vh])
    rg, _ = by_sequence(ref["o"])
    assert_heads(og, rg, TOL, cu=cu, label="decode 256 steps o", bf16_out=True)


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


def _kept_decode(w, keep):
    sub = dict(w)
    sub["x"] = w["x"][:, keep]
    sub["a"] = w["a"][:, keep]
    sub["b"] = w["b"][:, keep]
    sub["slot_ids"] = w["slot_ids"][keep]
    return sub


def test_decode_repeated_slot_first_occurrence_wins():
    """Sequences 2 and 4 repeat the slots of sequences 0 and 1: they are skipped entirely
    (no pool row, conv row or output written), the others run as if they were alone."""
    w = synthetic.decode(steps=1, n_seqs=5, n_slots=6)
    w["slot_ids"] = np.array([2, 4, 2, 0, 4], np.int32)
    layer = make_layer(w, o_dtype=torch.float32)
    dims = layer.dims
    o = torch.full((5, dims.H_v, dims.d_v), float("nan"), device="cuda")
    layer.decode(t_bits(w["x"][0]), t_f32(w["a"][0]), t_f32(w["b"][0]), t_i32(w["slot_ids"]),
                 out=o)
    assert device_status() == -2
    keep = [0, 1, 3]
    ref = oracle.decode_steps(_kept_decode(w, keep), 1)
    oc = o.cpu().numpy()
    assert rel_l2(oc[keep], ref["o"][0]) < 1e-5
    assert np.isnan(oc[[2, 4]]).all()
    pool = layer.state.cpu().numpy()
    assert rel_l2(pool[[2, 4, 0]], ref["S"]) < 1e-5
    np.testing.assert_array_equal(pool[[1, 3, 5]], w["state"][[1, 3, 5]])
    conv = layer.conv_state.cpu().view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(conv[[2, 4, 0]],
                                  synthetic.f32_to_bf16_bits(ref["conv_state"].astype(np.float32)))
    np.testing.assert_array_equal(conv[[1, 3, 5]], w["conv_state"][[1, 3, 5]])


def test_decode_step_right_after_slot_copy_and_back_to_back():
    """gdn_decode_step directly after gdn_state_slot_copy (which writes the rows it reads), and
    twice back to back on the same rows, against the oracle: every state read of a decode
    launch must see the writes of the kernel before it."""
    w = synthetic.decode(steps=2, n_seqs=4, n_slots=8)
    layer = make_layer(w, o_dtype=torch.float32)
    dims = layer.dims
    bufs = []
    for s in range(2):  # the front of both steps first, on the original slots 0..3
        q, k, v, g, beta = front_outputs(dims, 4)
        conv_step(dims, t_bits(w["x"][s]), layer.conv_w, layer.conv_state, None,
                  t_i32([0, 1, 2, 3]), t_f32(w["a"][s]), t_f32(w["b"][s]), layer.A_log,
                  layer.dt_bias, q, k, v, g, beta, eps=w["eps"], q_scale=w["q_scale"])
        bufs.append((q, k, v, g, beta))
    dst = t_i32([4, 5, 6, 7])
    state_slot_copy(dims, layer.state, None, t_i32([0, 1, 2, 3]), dst)
    outs = []
    for s in range(2):
        o = torch.empty((4, dims.H_v, dims.d_v), device="cuda")
        decode_step(dims, *bufs[s], layer.state, dst, o)
        outs.append(o)
    torch.cuda.synchronize()
    assert device_status() == 0
    ref = oracle.decode_steps(dict(w, slot_ids=np.arange(4, dtype=np.int32)), 2)
    for s in range(2):
        assert rel_l2(outs[s].cpu().numpy(), ref["o"][s]) < 1e-5
    pool = layer.state.cpu().numpy()
    assert rel_l2(pool[4:8], ref["S"]) < 1e-5
    np.testing.assert_array_equal(pool[0:4], w["state"][0:4])


@pytest.mark.parametrize("n_seqs,H_k,H_v", [(4, 16, 32), (16, 16, 32), (4, 8, 8)])
def test_layer_decode_equals_front_then_decode_step(n_seqs, H_k, H_v):
    """gdn_layer_decode against gdn_conv_step followed by gdn_decode_step: the same
    arithmetic, so bit-identical outputs and pools. 4 sequences take the one-kernel path
    (clusters of 4 x 2 and, with H_v = H_k, 4 x 1 CTAs), 16 the front + decode kernels."""
    w = synthetic.decode(steps=3, n_seqs=n_seqs, n_slots=n_seqs, H_k=H_k, H_v=H_v)
    l1 = make_layer(w)
    l2 = make_layer(w)
    dims = l1.dims
    slots = t_i32(w["slot_ids"])
    for s in range(3):
        o1 = l1.decode(t_bits(w["x"][s]), t_f32(w["a"][s]), t_f32(w["b"][s]), slots).clone()
        q, k, v, g, beta = front_outputs(dims, n_seqs)
        conv_step(dims, t_bits(w["x"][s]), l2.conv_w, l2.conv_state, t_i32(np.arange(n_seqs + 1)), slots,
                  t_f32(w["a"][s]), t_f32(w["b"][s]), l2.A_log, l2.dt_bias, q, k, v, g, beta,
                  eps=w["eps"], q_scale=w["q_scale"])
        o2 = torch.empty_like(o1)
        decode_step(dims, q, k, v, g, beta, l2.state, slots, o2)
        assert torch.equal(o1, o2)
    assert torch.equal(l1.state, l2.state)
    assert torch.equal(l1.conv_state, l2.conv_state)
    assert device_status() == 0


def test_layer_decode_plan_equals_layer_decode():
    """A decode plan (arguments marshalled once, fixed buffers refilled between steps) gives
    bit for bit what layer.decode gives, step after step, with and without a gate."""
    from gated_deltanet_linear_19_b200 import OutGate
    for n_seqs in (4, 16):
        w = synthetic.decode(steps=3, n_seqs=n_seqs, n_slots=n_seqs)
        l1, l2 = make_layer(w), make_layer(w)
        dims = l1.dims
        slots = t_i32(w["slot_ids"])
        xb = torch.empty((n_seqs, dims.conv_dim), dtype=torch.bfloat16, device="cuda")
        ab = torch.empty((n_seqs, dims.H_v), device="cuda")
        bb = torch.empty((n_seqs, dims.H_v), device="cuda")
        z = torch.randn((n_seqs, dims.H_v, dims.d_v), device="cuda").to(torch.bfloat16)
        nw = torch.ones(dims.d_v, device="cuda")
        gate = OutGate(z, nw, 1e-6)
        run, o2 = l2.decode_plan(xb, ab, bb, slots, gate=gate)
        for s in range(3):
            o1 = l1.decode(t_bits(w["x"][s]), t_f32(w["a"][s]), t_f32(w["b"][s]), slots,
                           gate=gate).clone()
            xb.copy_(t_bits(w["x"][s]))
            ab.copy_(t_f32(w["a"][s]))
            bb.copy_(t_f32(w["b"][s]))
            run()
            torch.cuda.synchronize()
            assert torch.equal(o1, o2), (n_seqs, s)
        assert torch.equal(l1.state, l2.state)
        assert torch.equal(l1.conv_state, l2.conv_state)
        assert device_status() == 0
