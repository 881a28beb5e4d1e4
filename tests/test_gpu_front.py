"""GPU parity of gdn_conv_step (conv1d + SiLU + L2 norm + gates, rolling conv state) against
the fp64 oracle, element by element; the conv state must roll bit-exactly."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from gated_deltanet_linear_19_b200 import conv_step, front_outputs, device_status
from tests.gpu_util import dims_of, rel_l2, t_bits, t_f32, t_i32

pytestmark = pytest.mark.gpu


def _run_front(w, qkv_dtype=torch.float32):
    dims = dims_of(w)
    T = int(w["cu_seqlens"][-1])
    x = t_bits(w["x"]) if w["x_dtype"] == "bf16" else t_f32(w["x"])
    conv = None
    if w.get("conv_state") is not None:
        conv = t_bits(w["conv_state"]) if w["conv_state_dtype"] == "bf16" else t_f32(w["conv_state"])
    q, k, v, g, beta = front_outputs(dims, T, qkv_dtype)
    reset = None if w.get("reset") is None else torch.from_numpy(w["reset"]).cuda()
    conv_step(dims, x, None if w["conv_w"] is None else t_f32(w["conv_w"]), conv,
              t_i32(w["cu_seqlens"]), t_i32(w["slot_ids"]), t_f32(w["a"]), t_f32(w["b"]),
              t_f32(w["A_log"]), t_f32(w["dt_bias"]), q, k, v, g, beta, eps=w["eps"],
              q_scale=w["q_scale"], reset=reset)
    assert device_status() == 0
    out = dict(q=q, k=k, v=v, g=g, beta=beta)
    out = {n: t.float().cpu().numpy() for n, t in out.items()}
    if conv is not None:
        c = conv.cpu()
        out["conv"] = c.view(torch.int16).numpy().view(np.uint16) if c.dtype == torch.bfloat16 \
            else c.numpy()
    return out


def _expected_conv_pool(w, ref):
    """Pool after the call: the oracle's rolled rows at the used slots, untouched elsewhere."""
    pool = w["conv_state"].copy()
    rolled = ref["conv_state"]  # float64 of exactly representable bf16 values
    bits = synthetic.f32_to_bf16_bits(rolled.astype(np.float32))
    pool[w["slot_ids"]] = bits
    return pool


@pytest.mark.parametrize("qkv_dtype,tol", [(torch.float32, 2e-6), (torch.float16, 6e-4),
                                           (torch.bfloat16, 4e-3)])
def test_front_varlen_ragged(qkv_dtype, tol):
    lengths = [1, 2, 3, 5, 17, 40, 16, 33]
    w = synthetic.packed(lengths, seed=501, slots=[7, 0, 3, 12, 9, 1, 5, 2], conv_std=1.0,
                         state_std=0.0, n_slots=16)
    w["reset"] = np.array([0, 1, 0, 0, 1, 0, 0, 0], np.uint8)
    out = _run_front(w, qkv_dtype)
    ref = oracle.layer(w)
    for n in ("q", "k", "v"):
        assert rel_l2(out[n], ref[n]) < tol, n
    assert rel_l2(out["g"], ref["g"]) < 2e-6
    assert rel_l2(out["beta"], ref["beta"]) < 2e-6
    np.testing.assert_array_equal(out["conv"], _expected_conv_pool(w, ref))


def test_front_decode_shape():
    d = synthetic.decode(steps=1)
    w = dict(d, x=d["x"][0], a=d["a"][0], b=d["b"][0])
    out = _run_front(w)
    ref = oracle.layer(w)
    for n in ("q", "k", "v", "g", "beta"):
        assert rel_l2(out[n], ref[n]) < 2e-6, n
    np.testing.assert_array_equal(out["conv"], _expected_conv_pool(w, ref))


def test_front_without_conv_fp32():
    w = synthetic.tiny()
    out = _run_front(w)
    ref = oracle.layer(w)
    for n in ("q", "k", "v", "g", "beta"):
        assert rel_l2(out[n], ref[n]) < 2e-6, n


def test_front_bad_slot_sets_status():
    w = synthetic.packed([4, 4], seed=502, slots=[0, 1], n_slots=2, conv_std=1.0)
    w["slot_ids"] = np.array([0, 5], np.int32)  # 5 >= n_slots
    dims = dims_of(w)
    q, k, v, g, beta = front_outputs(dims, 8)
    conv_step(dims, t_bits(w["x"]), t_f32(w["conv_w"]), t_bits(w["conv_state"]),
              t_i32(w["cu_seqlens"]), t_i32(w["slot_ids"]), t_f32(w["a"]), t_f32(w["b"]),
              t_f32(w["A_log"]), t_f32(w["dt_bias"]), q, k, v, g, beta)
    assert device_status() == -2
    assert device_status() == 0  # cleared
