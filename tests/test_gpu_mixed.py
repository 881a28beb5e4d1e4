"""Short sequences and mixed batches: the token-by-token kernel (state in registers across a
sequence's few tokens) on its own (GDN_PREFILL_RECURRENT) and inside gdn_chunked_prefill,
which sends sequences of at most 16 tokens to it and longer ones to the chunked tensor-core
kernels in the same call."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from gated_deltanet_linear_19_b200 import (GDN_PREFILL_RECURRENT, chunked_prefill, conv_step,
                                           decode_step, device_status)
from tests.gpu_util import (assert_heads, dims_of, make_layer, operand_ref, rel_l2,
                            run_prefill, t_bits, t_f32, t_i32)

pytestmark = pytest.mark.gpu


def _front(w, layer, dtype):
    T = int(w["cu_seqlens"][-1])
    q, k, v, g, beta = (t.clone() for t in layer._front_bufs(T, dtype))
    conv_step(layer.dims, t_bits(w["x"]), layer.conv_w, layer.conv_state, t_i32(w["cu_seqlens"]),
              t_i32(w["slot_ids"]), t_f32(w["a"]), t_f32(w["b"]), layer.A_log, layer.dt_bias,
              q, k, v, g, beta, eps=w["eps"], q_scale=w["q_scale"],
              reset=None if w.get("reset") is None else torch.from_numpy(w["reset"]).cuda())
    return q, k, v, g, beta


@pytest.mark.parametrize("qkv,odt,tol", [(torch.float32, torch.float32, 1e-5),
                                         (torch.float16, torch.bfloat16, 2e-3)])
def test_recurrent_kernel_short_sequences(qkv, odt, tol):
    lengths = [1, 2, 5, 16, 16, 3, 0, 9, 40]
    w = synthetic.packed(lengths, seed=701, slots=[4, 0, 8, 1, 7, 2, 3, 6, 5], state_std=0.02,
                         conv_std=1.0, n_slots=10)
    w["reset"] = np.array([0, 1, 0, 0, 0, 0, 1, 0, 0], np.uint8)
    o, S, _, _ = run_prefill(w, layer=make_layer(w, prefill_qkv_dtype=qkv, o_dtype=odt),
                             flags=GDN_PREFILL_RECURRENT, fused=False)
    assert device_status() == 0
    ref = oracle.layer(w)
    cu = w["cu_seqlens"]
    e_o, e_s = rel_l2(o, ref["o"]), rel_l2(S[w["slot_ids"]], ref["S"])
    print(f"recurrent {qkv}: o {e_o:.3e} S {e_s:.3e}")
    low = tol >= 2e-3
    r16 = operand_ref(ref, w) if qkv == torch.float16 else None
    assert_heads(o, ref["o"], tol, cu=cu, label="recurrent o", bf16_out=low, ref16=r16)
    assert_heads(S[w["slot_ids"]], ref["S"], tol if not low else 2e-3, label="recurrent S")
    assert np.all(S[3] == 0)  # the empty sequence with reset


def test_mixed_batch_routes_each_sequence_once():
    """Short and long sequences in one gdn_chunked_prefill call: against the oracle, and each
    side bit-identical to a call holding only its own sequences."""
    lengths = [1, 300, 1, 16, 17, 64, 2, 129, 0]
    slots = [3, 0, 8, 1, 7, 2, 4, 6, 5]
    w = synthetic.packed(lengths, seed=702, slots=slots, state_std=0.02, conv_std=1.0, n_slots=9)
    layer = make_layer(w)
    q, k, v, g, beta = _front(w, layer, torch.float16)
    dims, T = layer.dims, q.shape[0]
    cu, sl = t_i32(w["cu_seqlens"]), t_i32(w["slot_ids"])
    state0 = t_f32(w["state"])
    st = state0.clone()
    o = torch.full((T, dims.H_v, dims.d_v), float("nan"), dtype=torch.bfloat16, device="cuda")
    chunked_prefill(dims, q, k, v, g, beta, st, sl, cu, o)
    assert device_status() == 0
    # the same q, k, v through the oracle's recurrence (the front is checked elsewhere)
    ref = oracle.layer(w)
    on, Sn = o.float().cpu().numpy(), st.cpu().numpy()
    assert rel_l2(on, ref["o"]) < 2e-3
    assert_heads(on, ref["o"], 2e-3, cu=w["cu_seqlens"], label="mixed o", bf16_out=True,
                 ref16=operand_ref(ref, w), chunk=64)
    assert_heads(Sn[w["slot_ids"]], ref["S"], 2e-3, label="mixed S")
    # short sequences == the token-by-token kernel alone
    st_r = state0.clone()
    o_r = torch.full_like(o, float("nan"))
    chunked_prefill(dims, q, k, v, g, beta, st_r, sl, cu, o_r, flags=GDN_PREFILL_RECURRENT)
    cuh = np.asarray(w["cu_seqlens"])
    for n, L in enumerate(lengths):
        rows = slice(cuh[n], cuh[n + 1])
        if L <= 16:
            assert torch.equal(o[rows], o_r[rows]), n
            assert torch.equal(st[slots[n]], st_r[slots[n]]), n
    # long sequences == a call holding only them
    long_idx = [n for n, L in enumerate(lengths) if L > 16]
    rows = np.concatenate([np.arange(cuh[n], cuh[n + 1]) for n in long_idx])
    rt = torch.from_numpy(rows).cuda()
    cu_l = t_i32(np.concatenate([[0], np.cumsum([lengths[n] for n in long_idx])]))
    st_l = state0.clone()
    o_l = torch.empty((len(rows), dims.H_v, dims.d_v), dtype=torch.bfloat16, device="cuda")
    chunked_prefill(dims, q[rt].contiguous(), k[rt].contiguous(), v[rt].contiguous(),
                    g[rt].contiguous(), beta[rt].contiguous(), st_l,
                    t_i32([slots[n] for n in long_idx]), cu_l, o_l)
    assert device_status() == 0
    assert torch.equal(o[rt], o_l)
    for n in long_idx:
        assert torch.equal(st[slots[n]], st_l[slots[n]]), n


def test_single_tokens_through_prefill_equal_decode_step():
    """64 one-token sequences through gdn_chunked_prefill (all short: the token-by-token
    kernel) give exactly gdn_decode_step's outputs and states (same one-pass arithmetic)."""
    d = synthetic.decode(steps=1, n_seqs=64, n_slots=64)
    w = dict(d, x=d["x"][0], a=d["a"][0], b=d["b"][0])
    layer = make_layer(w)
    q, k, v, g, beta = _front(w, layer, torch.float16)  # fp16: the tensor-core path
    dims = layer.dims
    s1, s2 = t_f32(w["state"]), t_f32(w["state"])
    o1 = torch.empty((64, dims.H_v, dims.d_v), dtype=torch.bfloat16, device="cuda")
    o2 = torch.empty_like(o1)
    chunked_prefill(dims, q, k, v, g, beta, s1, t_i32(w["slot_ids"]), t_i32(w["cu_seqlens"]), o1)
    decode_step(dims, q, k, v, g, beta, s2, t_i32(w["slot_ids"]), o2)
    assert device_status() == 0
    assert torch.equal(o1, o2)
    assert torch.equal(s1, s2)


MIXED_SETS = {
    # 6 sequences: the one-kernel short path (front inside, a cluster per key head)
    "few": ([1, 300, 16, 17, 0, 5], [3, 0, 1, 4, 5, 2], [1, 0, 0, 0, 1, 0]),
    # 11 sequences: past the one-kernel path's grid limit, the front of the short sequences into
    # compact workspace rows, then the token-by-token kernel
    "many": ([1, 300, 1, 16, 17, 64, 2, 129, 0, 0, 5], [3, 0, 8, 1, 7, 2, 4, 6, 5, 9, 10],
             [0, 0, 1, 0, 0, 1, 0, 0, 1, 0, 0]),
}


@pytest.mark.parametrize("layout", [0, synthetic.GQA_TILED])
@pytest.mark.parametrize("which", ["few", "many"])
def test_layer_prefill_mixed_batch(layout, which):
    """A mixed batch through gdn_layer_prefill (the front inside the kernels): sequences of at
    most 16 tokens run in the short path, longer ones in the record and scan kernels; against
    the oracle per (sequence, head) and per chunk, the conv state bit for bit, and empty
    sequences (with and without reset) handled."""
    lengths, slots, reset = MIXED_SETS[which]
    w = synthetic.packed(lengths, seed=703, slots=slots, state_std=0.02, conv_std=1.0,
                         n_slots=len(lengths), layout=layout)
    w["reset"] = np.array(reset, np.uint8)
    o, S, conv, _ = run_prefill(w)
    assert device_status() == 0
    ref = oracle.layer(w)
    assert_heads(o, ref["o"], 2e-3, cu=w["cu_seqlens"], label="layer mixed o", bf16_out=True,
                 ref16=operand_ref(ref, w), chunk=64)
    assert_heads(S[w["slot_ids"]], ref["S"], 2e-3, label="layer mixed S")
    np.testing.assert_array_equal(conv[w["slot_ids"]],
                                  synthetic.f32_to_bf16_bits(ref["conv_state"].astype(np.float32)))
    e_slot_rst = slots[lengths.index(0)]
    assert np.all(S[e_slot_rst] == 0)                    # empty with reset: zero state
    if lengths.count(0) > 1:
        e_slot = slots[len(lengths) - 1 - lengths[::-1].index(0)]
        np.testing.assert_array_equal(S[e_slot], w["state"][e_slot])  # empty: unchanged


@pytest.mark.parametrize("lengths", [[4, 1, 16, 3], [4] * 8 + [1, 16]])
def test_layer_prefill_all_short(lengths):
    """Only short sequences (a multi-token step) through gdn_layer_prefill: the short path
    alone (4 sequences: one kernel; 10: front + token-by-token kernel), against the oracle."""
    n = len(lengths)
    w = synthetic.packed(lengths, seed=704, slots=list(range(n)), state_std=0.02,
                         conv_std=1.0, n_slots=n)
    o, S, conv, _ = run_prefill(w)
    assert device_status() == 0
    ref = oracle.layer(w)
    e_o = rel_l2(o, ref["o"])
    print(f"layer all-short: o {e_o:.3e}")
    assert_heads(o, ref["o"], 2e-3, cu=w["cu_seqlens"], label="layer short o", bf16_out=True,
                 ref16=operand_ref(ref, w))
    assert_heads(S[w["slot_ids"]], ref["S"], 2e-3, label="layer short S")
    np.testing.assert_array_equal(conv[w["slot_ids"]],
                                  synthetic.f32_to_bf16_bits(ref["conv_state"].astype(np.float32)))


def test_layer_prefill_short_only_flag():
    """gdn_layer_prefill with GDN_PREFILL_RECURRENT (every sequence promised to have at most
    16 tokens): the chunked kernels are skipped and the results are those of the routed call;
    a sequence longer than 16 tokens is skipped with GDN_EINVAL recorded, its rows untouched."""
    from gated_deltanet_linear_19_b200 import layer_prefill, prefill_workspace_size
    lengths = [4] * 12 + [1, 16]
    n = len(lengths)
    w = synthetic.packed(lengths, seed=705, slots=list(range(n)), state_std=0.02,
                         conv_std=1.0, n_slots=n)
    outs = []
    for flags in (0, GDN_PREFILL_RECURRENT):
        layer = make_layer(w)
        dims, T = layer.dims, int(w["cu_seqlens"][-1])
        o = torch.empty((T, dims.H_v, dims.d_v), dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(max(prefill_workspace_size(dims, T, n, 64, torch.float16, flags), 16),
                         dtype=torch.uint8, device="cuda")
        layer_prefill(dims, t_bits(w["x"]), layer.conv_w, layer.conv_state,
                      t_i32(w["cu_seqlens"]), t_i32(w["slot_ids"]), t_f32(w["a"]), t_f32(w["b"]),
                      layer.A_log, layer.dt_bias, layer.state, o, eps=w["eps"],
                      q_scale=w["q_scale"], workspace=ws, flags=flags)
        torch.cuda.synchronize()
        assert device_status() == 0
        outs.append((o, layer.state.clone(), layer.conv_state.clone()))
    for a, b in zip(outs[0], outs[1]):
        assert torch.equal(a, b)
    # a 17-token sequence under the promise: skipped, GDN_EINVAL
    lengths = [4, 17, 2]
    w = synthetic.packed(lengths, seed=706, slots=[0, 1, 2], state_std=0.02, conv_std=1.0,
                         n_slots=3)
    layer = make_layer(w)
    dims, T = layer.dims, int(w["cu_seqlens"][-1])
    o = torch.zeros((T, dims.H_v, dims.d_v), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(max(prefill_workspace_size(dims, T, 3, 64, torch.float16,
                                                GDN_PREFILL_RECURRENT), 16),
                     dtype=torch.uint8, device="cuda")
    layer_prefill(dims, t_bits(w["x"]), layer.conv_w, layer.conv_state, t_i32(w["cu_seqlens"]),
                  t_i32(w["slot_ids"]), t_f32(w["a"]), t_f32(w["b"]), layer.A_log,
                  layer.dt_bias, layer.state, o, eps=w["eps"], q_scale=w["q_scale"],
                  workspace=ws, flags=GDN_PREFILL_RECURRENT)
    torch.cuda.synchronize()
    assert device_status(clear=True) == -1  # GDN_EINVAL
    np.testing.assert_array_equal(layer.state[1].cpu().numpy(), w["state"][1])
    assert torch.all(o[4:21] == 0)
