"""GPU parity of the chunked prefill (gdn_conv_step + gdn_chunked_prefill) against the fp64
per-token oracle: tiny fp32 workload (1e-5), ragged multi-tile cases, and the full-size
prefill / varlen / long-context workloads (sampled heads where the oracle is slow)."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from gated_deltanet_linear_19_b200 import (GDN_PREFILL_SIMT, GDN_PREFILL_TC_HEAD_SCAN,
                                           GDN_PREFILL_TC_TILE_SCAN,
                                           device_status)
from tests.gpu_util import (assert_heads, bf16_floor, by_sequence, make_layer, operand_ref,
                            rel_l2, run_prefill, subset_packed, t_bits, t_f32, t_i32)

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-3
TOL_F32 = 1e-5


def check_heads(o, S, ref, cu, tol, label, vh=None, w=None):
    """Per (sequence, v-head) and per (chunk, v-head) parity of the output, per (sequence,
    v-head) parity of the final state (see assert_heads). With w (the workload) the bound also
    allows for the fp16 rounding of the q, k, v operands (operand_ref), for the paths that take
    them in fp16."""
    oo = o if vh is None else o[:, vh]
    SS = S if vh is None else S[:, vh]
    low = tol >= TOL_BF16
    r16 = operand_ref(ref, w, vh) if (w is not None and low) else None
    assert_heads(oo, ref["o"], tol, cu=cu, label=label + " o", bf16_out=low, ref16=r16,
                 chunk=64)
    assert_heads(SS, ref["S"], tol, label=label + " S")


def test_tiny_fp32_simt():
    w = synthetic.tiny()
    layer = make_layer(w, prefill_qkv_dtype=torch.float32, o_dtype=torch.float32)
    o, S, _, _ = run_prefill(w, layer=layer, chunk=16)
    ref = oracle.layer(w)
    e_o, e_s = rel_l2(o, ref["o"]), rel_l2(S[w["slot_ids"]], ref["S"])
    print(f"tiny fp32: o {e_o:.2e} S {e_s:.2e}")
    assert e_o < TOL_F32 and e_s < TOL_F32
    check_heads(o, S[w["slot_ids"]], ref, w["cu_seqlens"], TOL_F32, "tiny fp32")
    assert device_status() == 0


@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_ragged_varlen_fp32_all_chunks(chunk):
    lengths = [1, 5, 64, 65, 130, 17]
    w = synthetic.packed(lengths, seed=601, slots=[3, 9, 0, 4, 11, 6], state_std=0.02,
                         conv_std=1.0, n_slots=12)
    layer = make_layer(w, prefill_qkv_dtype=torch.float32, o_dtype=torch.float32)
    o, S, conv, _ = run_prefill(w, layer=layer, chunk=chunk)
    ref = oracle.layer(w)
    assert rel_l2(o, ref["o"]) < TOL_F32
    assert rel_l2(S[w["slot_ids"]], ref["S"]) < TOL_F32
    check_heads(o, S[w["slot_ids"]], ref, w["cu_seqlens"], TOL_F32, f"ragged fp32 C={chunk}")
    untouched = [s for s in range(12) if s not in set(w["slot_ids"].tolist())]
    np.testing.assert_array_equal(S[untouched], w["state"][untouched])
    np.testing.assert_array_equal(conv[w["slot_ids"]],
                                  synthetic.f32_to_bf16_bits(ref["conv_state"].astype(np.float32)))
    assert device_status() == 0


@pytest.mark.parametrize("flags,fused", [(0, None), (0, False),
                                         (GDN_PREFILL_SIMT, None),
                                         (GDN_PREFILL_TC_HEAD_SCAN, None),
                                         (GDN_PREFILL_TC_HEAD_SCAN, False),
                                         (GDN_PREFILL_TC_TILE_SCAN, None),
                                         (GDN_PREFILL_TC_TILE_SCAN, False)])
def test_ragged_fp16_front_bf16_out(flags, fused):
    """fused=None: gdn_layer_prefill (front inside the prep) where it applies; False: the
    two calls gdn_conv_step + gdn_chunked_prefill. The conv state must match bit for bit."""
    lengths = [300, 1, 77, 129, 2]
    w = synthetic.packed(lengths, seed=602, slots=[1, 0, 3, 2, 4], state_std=0.02, conv_std=1.0,
                         n_slots=5)
    w["reset"] = np.array([0, 0, 1, 0, 0], np.uint8)
    o, S, conv, _ = run_prefill(w, flags=flags, fused=fused)
    ref = oracle.layer(w)
    e_o, e_s = rel_l2(o, ref["o"]), rel_l2(S[w["slot_ids"]], ref["S"])
    print(f"ragged fp16/bf16 flags={flags} fused={fused}: o {e_o:.3e} "
          f"(floor {bf16_floor(ref['o']):.3e}) S {e_s:.3e}")
    assert e_o < TOL_BF16 and e_s < TOL_BF16
    check_heads(o, S[w["slot_ids"]], ref, w["cu_seqlens"], TOL_BF16, "ragged fp16", w=w)
    np.testing.assert_array_equal(conv[w["slot_ids"]],
                                  synthetic.f32_to_bf16_bits(ref["conv_state"].astype(np.float32)))
    assert device_status() == 0


@pytest.mark.parametrize("flags,fused", [(0, None), (0, False),
                                         (GDN_PREFILL_TC_HEAD_SCAN, None)])
def test_prefill_4096_all_heads(flags, fused):
    w = synthetic.prefill()
    o, S, _, _ = run_prefill(w, flags=flags, fused=fused)
    ref = oracle.layer(w)
    e_o, e_s = rel_l2(o, ref["o"]), rel_l2(S[w["slot_ids"]], ref["S"])
    print(f"prefill T=4096 flags={flags} fused={fused}: o {e_o:.3e} "
          f"(floor {bf16_floor(ref['o']):.3e}) S {e_s:.3e}")
    assert e_o < TOL_BF16 and e_s < TOL_BF16
    check_heads(o, S[w["slot_ids"]], ref, w["cu_seqlens"], TOL_BF16, "prefill T=4096", w=w)
    assert device_status() == 0


# flags 0: the whole-head scan here; fused False: the q / k / v path, whose record blocks
# here take one value head each
@pytest.mark.parametrize("flags,fused", [(0, None), (GDN_PREFILL_TC_TILE_SCAN, None), (0, False)])
def test_varlen_16_sequences_sampled_heads(flags, fused):
    w = synthetic.varlen()
    o, S, _, _ = run_prefill(w, flags=flags, fused=fused)
    ref = oracle.layer(w, k_heads=[0, 5, 11, 15])
    vh = ref["v_heads"]
    e_o, e_s = rel_l2(o[:, vh], ref["o"]), rel_l2(S[w["slot_ids"]][:, vh], ref["S"])
    print(f"varlen T={int(w['cu_seqlens'][-1])}: o {e_o:.3e} S {e_s:.3e}")
    assert e_o < TOL_BF16 and e_s < TOL_BF16
    check_heads(o, S[w["slot_ids"]], ref, w["cu_seqlens"], TOL_BF16, "varlen", vh=vh, w=w)
    assert device_status() == 0


def test_long_context_then_decode_sampled_heads():
    w = synthetic.long_context()
    layer = make_layer(w)
    o, S, conv, layer = run_prefill(w, layer=layer)
    k_heads = [0, 5, 10, 15]
    ref = oracle.layer(w, k_heads=k_heads)
    vh = ref["v_heads"]
    e_o, e_s = rel_l2(o[:, vh], ref["o"]), rel_l2(S[w["slot_ids"]][:, vh], ref["S"])
    g = ref["g"]
    print(f"long 4x65536: o {e_o:.3e} S {e_s:.3e}; exp(g) range [{np.exp(g.min()):.2e}, "
          f"{np.exp(g.max()):.2e}]")
    assert e_o < TOL_BF16 and e_s < TOL_BF16
    check_heads(o, S[w["slot_ids"]], ref, w["cu_seqlens"], TOL_BF16, "long", vh=vh, w=w)
    del o
    # 512 decode steps from the prefill's final states
    steps = 512
    d = synthetic.decode(seed=synthetic.SEED_BASE + 40, n_seqs=4, steps=steps,
                         n_slots=w["dims"]["n_slots"])
    d["slot_ids"] = w["slot_ids"]
    d["conv_w"] = w["conv_w"]; d["A_log"] = w["A_log"]; d["dt_bias"] = w["dt_bias"]
    slots = t_i32(w["slot_ids"])
    outs = []
    for s in range(steps):
        outs.append(layer.decode(t_bits(d["x"][s]), t_f32(d["a"][s]), t_f32(d["b"][s]),
                                 slots).float().cpu().numpy())
    refd = oracle.decode_steps(d, steps, k_heads=k_heads, S0=ref["S"],
                               conv_state0=ref["conv_state"])
    e_od = rel_l2(np.stack(outs)[:, :, vh], refd["o"])
    e_sd = rel_l2(layer.state.cpu().numpy()[w["slot_ids"]][:, vh], refd["S"])
    print(f"then 512 decode steps: o {e_od:.3e} S {e_sd:.3e}")
    assert e_od < TOL_BF16 and e_sd < TOL_BF16
    og, cug = by_sequence(np.stack(outs)[:, :, vh])
    rg, _ = by_sequence(refd["o"])
    assert_heads(og, rg, TOL_BF16, cu=cug, label="long then decode o", bf16_out=True)
    assert device_status() == 0


def test_resume_two_calls_equal_one():
    lengths = [200]
    w = synthetic.packed(lengths, seed=603, state_std=0.02, conv_std=1.0, n_slots=1)
    layer1 = make_layer(w, prefill_qkv_dtype=torch.float32, o_dtype=torch.float32)
    o_full, S_full, conv_full, _ = run_prefill(w, layer=layer1)
    layer2 = make_layer(w, prefill_qkv_dtype=torch.float32, o_dtype=torch.float32)
    parts = []
    for a, b in ((0, 77), (77, 200)):
        wp = dict(w, x=w["x"][a:b], a=w["a"][a:b], b=w["b"][a:b],
                  cu_seqlens=np.array([0, b - a], np.int32))
        op, Sp, convp, _ = run_prefill(wp, layer=layer2)
        parts.append(op)
    assert rel_l2(np.concatenate(parts), o_full) < 1e-5
    assert rel_l2(Sp, S_full) < 1e-5
    np.testing.assert_array_equal(convp, conv_full)


def test_prefill_is_deterministic():
    w = synthetic.packed([333, 64], seed=604, state_std=0.02, conv_std=1.0, n_slots=2)
    o1, S1, _, _ = run_prefill(w)
    o2, S2, _, _ = run_prefill(w)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(S1, S2)


def test_empty_sequences_keep_or_reset_state():
    w = synthetic.packed([0, 10, 0], seed=605, slots=[2, 0, 1], state_std=0.02, conv_std=1.0,
                         n_slots=3)
    w["reset"] = np.array([0, 0, 1], np.uint8)
    layer = make_layer(w, prefill_qkv_dtype=torch.float32, o_dtype=torch.float32)
    o, S, _, _ = run_prefill(w, layer=layer)
    ref = oracle.layer(w)
    assert rel_l2(S[w["slot_ids"]], ref["S"]) < TOL_F32
    np.testing.assert_array_equal(S[2], w["state"][2])   # empty, no reset: unchanged
    assert np.all(S[1] == 0)                              # empty with reset: zero
    assert device_status() == 0


@pytest.mark.parametrize("qkv,flags", [("f32", 0), ("f16", 0),
                                       ("f16", GDN_PREFILL_TC_HEAD_SCAN),
                                       ("f16", GDN_PREFILL_TC_TILE_SCAN)])
def test_slow_decay_state_carries_across_chunks(qkv, flags):
    """Gates of about -0.02 per token: the state reaches across many chunks, so the
    inter-chunk terms (W S, Q~ S, the state carry) dominate the output."""
    lengths = [700, 333]
    w = synthetic.packed(lengths, seed=606, slots=[1, 0], state_std=0.02, conv_std=1.0,
                         n_slots=2)
    w["A_log"] = np.zeros_like(w["A_log"])
    w["dt_bias"] = np.full_like(w["dt_bias"], -4.0)
    dt = torch.float32 if qkv == "f32" else torch.float16
    layer = make_layer(w, prefill_qkv_dtype=dt, o_dtype=torch.float32)
    o, S, _, _ = run_prefill(w, layer=layer, flags=flags)
    ref = oracle.layer(w)
    g = ref["g"]
    e_o, e_s = rel_l2(o, ref["o"]), rel_l2(S[w["slot_ids"]], ref["S"])
    print(f"slow decay {qkv} flags={flags}: mean g {g.mean():.3e}; o {e_o:.3e} S {e_s:.3e}")
    tol = TOL_F32 if qkv == "f32" else TOL_BF16
    assert e_o < tol and e_s < tol
    assert device_status() == 0


@pytest.mark.parametrize("fused", [True, False])
def test_layer_prefill_equal_key_and_value_heads(fused):
    """H_k = H_v (one value head per record block: the compact shared-memory layout, three
    blocks per SM, the fused front's x tiles converted in place; in the layer prefill every
    value head also writes its key head's q and k conv-state channels), through
    gdn_layer_prefill and through the two calls, against the oracle per (sequence, head) and
    per chunk, conv state bit-exact."""
    lengths = [130, 3, 64, 200]
    w = synthetic.packed(lengths, seed=607, slots=[2, 0, 1, 3], state_std=0.02, conv_std=1.0,
                         n_slots=4, H_k=4, H_v=4)
    o, S, conv, _ = run_prefill(w, fused=fused)
    ref = oracle.layer(w)
    e_o, e_s = rel_l2(o, ref["o"]), rel_l2(S[w["slot_ids"]], ref["S"])
    print(f"layer prefill H_k=H_v=4 fused={fused}: o {e_o:.3e} S {e_s:.3e}")
    assert e_o < TOL_BF16 and e_s < TOL_BF16
    assert_heads(o, ref["o"], TOL_BF16, cu=w["cu_seqlens"], label=f"H_k=H_v fused={fused}",
                 bf16_out=True, ref16=operand_ref(ref, w), chunk=64)
    assert_heads(S[w["slot_ids"]], ref["S"], TOL_BF16, label=f"H_k=H_v fused={fused} S")
    np.testing.assert_array_equal(conv[w["slot_ids"]],
                                  synthetic.f32_to_bf16_bits(ref["conv_state"].astype(np.float32)))
    assert device_status() == 0


@pytest.mark.parametrize("scale,slow", [(30.0, False), (30.0, True)])
def test_large_magnitude_inputs(scale, slow):
    """x scaled by 30 (SiLU outputs, and so v, U and the state, about 30 times larger), alone
    and with slow decay (the state builds up over hundreds of tokens): the tensor-core path's
    fp16 operands must keep their relative precision at these magnitudes."""
    lengths = [700, 333]
    w = synthetic.packed(lengths, seed=611, slots=[1, 0], state_std=0.02, conv_std=1.0,
                         n_slots=2)
    xf = oracle.bf16_bits_to_f64(w["x"]) * scale
    w["x"] = synthetic.f32_to_bf16_bits(xf.astype(np.float32))
    if slow:
        w["A_log"] = np.zeros_like(w["A_log"])
        w["dt_bias"] = np.full_like(w["dt_bias"], -4.0)
    o, S, _, _ = run_prefill(w)
    ref = oracle.layer(w)
    print(f"x*{scale} slow={slow}: max |v| {np.abs(ref['v']).max():.1f}, max |S| "
          f"{np.abs(ref['S']).max():.1f}")
    assert np.isfinite(o).all() and np.isfinite(S).all()
    e_o, e_s = rel_l2(o, ref["o"]), rel_l2(S[w["slot_ids"]], ref["S"])
    print(f"x*{scale} slow={slow}: o {e_o:.3e} S {e_s:.3e}")
    assert e_o < TOL_BF16 and e_s < TOL_BF16
    check_heads(o, S[w["slot_ids"]], ref, w["cu_seqlens"], TOL_BF16, f"x*{scale}", w=w)
    assert device_status() == 0


@pytest.mark.parametrize("flags,fused", [(0, None), (0, False), (GDN_PREFILL_SIMT, None)])
def test_prefill_repeated_slot_first_occurrence_wins(flags, fused):
    """Sequence 2 repeats the slot of sequence 0: it is skipped entirely (no state or conv
    row, no output written); the others run as if they were alone in the call."""
    lengths = [70, 33, 129, 5]
    w = synthetic.packed(lengths, seed=612, slots=[1, 3, 1, 0], state_std=0.02, conv_std=1.0,
                         n_slots=5)
    layer = make_layer(w)
    T = int(w["cu_seqlens"][-1])
    out = torch.full((T, layer.dims.H_v, layer.dims.d_v), float("nan"), dtype=torch.bfloat16,
                     device="cuda")
    o, S, conv, _ = run_prefill(w, layer=layer, flags=flags, fused=fused, out=out)
    assert device_status() == -2
    keep = [0, 1, 3]
    sub, rows = subset_packed(w, keep)
    ref = oracle.layer(sub)
    assert rel_l2(o[rows], ref["o"]) < TOL_BF16
    cu = np.asarray(w["cu_seqlens"])
    assert np.isnan(o[cu[2]:cu[3]]).all()
    assert rel_l2(S[[1, 3, 0]], ref["S"]) < TOL_BF16
    np.testing.assert_array_equal(S[[2, 4]], w["state"][[2, 4]])
    np.testing.assert_array_equal(conv[[1, 3, 0]],
                                  synthetic.f32_to_bf16_bits(ref["conv_state"].astype(np.float32)))
    np.testing.assert_array_equal(conv[[2, 4]], w["conv_state"][[2, 4]])
