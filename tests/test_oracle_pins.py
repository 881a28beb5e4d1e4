"""Pins for the fp64 oracle: each checks it against something other than itself.

The pages print no numeric worked example for this layer, so the pins come from the
definition of the single-token step (qwen3next.cpp, build_delta_net_autoregressive), the
chunk algebra (qwen3next.cpp, build_delta_net_chunking and the removed single-chunk path)
and the front (ik_llama.cpp src/llama-delta-net.cpp, build_layer_attn_linear_core):
closed forms, special cases, a hand-worked example, brute force on tiny inputs and
identities that any correct implementation satisfies.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _unit_rows(r, *shape):
    x = r.standard_normal(shape)
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _rand_core(seed, T, H_k, H_v, d_k, d_v, n_seqs=1, g_scale=0.3):
    r = np.random.default_rng(seed)
    q = _unit_rows(r, T, H_k, d_k) / math.sqrt(d_k)
    k = _unit_rows(r, T, H_k, d_k)
    v = r.standard_normal((T, H_v, d_v))
    g = -g_scale * r.random((T, H_v))
    beta = r.random((T, H_v))
    S0 = 0.1 * r.standard_normal((n_seqs, H_v, d_k, d_v))
    return q, k, v, g, beta, S0


def _relerr(a, b):
    return np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(np.asarray(b).ravel()), 1e-300)


# ---------------------------------------------------------------- core recurrence pins

def test_hand_worked_example():
    ex = json.load(open(os.path.join(GOLDEN, "hand_example_T2.json")))
    q = np.array(ex["q"])[:, None, :]
    k = np.array(ex["k"])[:, None, :]
    v = np.array(ex["v"])[:, None, :]
    g = np.array(ex["g"])[:, None]
    beta = np.array(ex["beta"])[:, None]
    o, S = oracle.recurrence(q, k, v, g, beta, None, [0, 2], threads=1)
    np.testing.assert_allclose(o[:, 0, :], np.array(ex["o"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(S[0, 0], np.array(ex["S_final"]), rtol=0, atol=1e-14)


def test_single_token_from_zero_state():
    # one token from S0 = 0: S = beta k v^T and o = beta (q.k) v
    q, k, v, g, beta, _ = _rand_core(1, 1, 2, 4, 16, 8)
    o, S = oracle.recurrence(q, k, v, g, beta, None, [0, 1], threads=1)
    for h in range(4):
        hk = h // 2
        exp_S = beta[0, h] * np.outer(k[0, hk], v[0, h])
        exp_o = beta[0, h] * float(q[0, hk] @ k[0, hk]) * v[0, h]
        np.testing.assert_allclose(S[0, h], exp_S, rtol=1e-13, atol=1e-15)
        np.testing.assert_allclose(o[0, h], exp_o, rtol=1e-13, atol=1e-15)


def test_beta0_g0_leaves_state_unchanged():
    q, k, v, g, beta, S0 = _rand_core(2, 7, 2, 2, 8, 8)
    g[:] = 0.0
    beta[:] = 0.0
    o, S = oracle.recurrence(q, k, v, g, beta, S0, [0, 7], threads=1)
    np.testing.assert_array_equal(S, S0)
    for t in range(7):
        for h in range(2):
            np.testing.assert_allclose(o[t, h], S0[0, h].T @ q[t, h], rtol=1e-13, atol=1e-15)


def test_very_negative_gate_erases_history():
    q, k, v, g, beta, S0 = _rand_core(3, 9, 1, 1, 8, 8)
    g[5, 0] = -800.0  # exp(-800) == 0 in fp64
    o, S = oracle.recurrence(q, k, v, g, beta, S0, [0, 9], threads=1)
    # token 5 acts as the first token of a fresh sequence
    exp_o5 = beta[5, 0] * float(q[5, 0] @ k[5, 0]) * v[5, 0]
    np.testing.assert_allclose(o[5, 0], exp_o5, rtol=1e-13, atol=1e-15)
    o2, S2 = oracle.recurrence(q[5:], k[5:], v[5:], g[5:], beta[5:], None, [0, 4], threads=1)
    np.testing.assert_allclose(o[5:], o2, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(S, S2, rtol=1e-13, atol=1e-15)


def test_orthonormal_keys_store_values_exactly():
    # beta = 1, g = 0, orthonormal keys: the delta rule writes each value at its key
    r = np.random.default_rng(4)
    d, T = 16, 10
    Qm, _ = np.linalg.qr(r.standard_normal((d, d)))
    k = Qm[:, :T].T[:, None, :]
    v = r.standard_normal((T, 1, d))
    q = k.copy()
    g = np.zeros((T, 1)); beta = np.ones((T, 1))
    o, S = oracle.recurrence(q, k, v, g, beta, None, [0, T], threads=1)
    for i in range(T):
        np.testing.assert_allclose(S[0, 0].T @ k[i, 0], v[i, 0], atol=1e-12)
    # reading with q = k_t right after writing returns v_t
    np.testing.assert_allclose(o[:, 0], v[:, 0], atol=1e-12)


def test_same_key_twice_overwrites():
    r = np.random.default_rng(5)
    d = 8
    kk = r.standard_normal(d); kk /= np.linalg.norm(kk)
    k = np.stack([kk, kk])[:, None, :]
    v = r.standard_normal((2, 1, d))
    q = k.copy()
    o, S = oracle.recurrence(q, k, v, np.zeros((2, 1)), np.ones((2, 1)), None, [0, 2],
                             threads=1)
    np.testing.assert_allclose(S[0, 0], np.outer(kk, v[1, 0]), atol=1e-13)


def _brute_force(q, k, v, g, beta, S0):
    """Affine-map expansion with explicit d_k x d_k matrices:
    S_t = A_t S_{t-1} + beta_t k_t v_t^T, A_t = exp(g_t) (I - beta_t k_t k_t^T); o_t = S_t^T q_t.
    The product form is unrolled: S_T = (prod_t A_t) S_0 + sum_t (prod_{s>t} A_s) beta_t k_t v_t^T.
    """
    T, d_k = k.shape
    I = np.eye(d_k)
    A = [math.exp(g[t]) * (I - beta[t] * np.outer(k[t], k[t])) for t in range(T)]
    outs = []
    for t_end in range(T):
        prod = I.copy()
        for t in range(t_end, -1, -1):
            prod = prod @ A[t]
        St = prod @ S0
        for t in range(t_end + 1):
            P = I.copy()
            for s in range(t_end, t, -1):
                P = P @ A[s]
            St = St + P @ (beta[t] * np.outer(k[t], v[t]))
        outs.append(St.T @ q[t_end])
    return np.array(outs), St


@pytest.mark.parametrize("T", [1, 3, 8])
def test_brute_force_unrolled_product(T):
    q, k, v, g, beta, S0 = _rand_core(10 + T, T, 1, 1, 6, 5, g_scale=1.0)
    o, S = oracle.recurrence(q, k, v, g, beta, S0, [0, T], threads=1)
    ob, Sb = _brute_force(q[:, 0], k[:, 0], v[:, 0], g[:, 0], beta[:, 0], S0[0, 0])
    assert _relerr(o[:, 0], ob) < 1e-12
    assert _relerr(S[0, 0], Sb) < 1e-12


@pytest.mark.parametrize("C", [1, 4, 16, 64])
def test_chunked_equals_recurrent(C):
    lengths = [37, 64, 5, 130]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    q, k, v, g, beta, S0 = _rand_core(20 + C, int(cu[-1]), 2, 4, 16, 12, n_seqs=4)
    o_r, S_r = oracle.recurrence(q, k, v, g, beta, S0, cu)
    o_c, S_c = oracle.chunked(q, k, v, g, beta, S0, cu, C)
    assert _relerr(o_c, o_r) < 1e-12
    assert _relerr(S_c, S_r) < 1e-12


def test_chunked_with_strong_decay():
    # cumulative gates of about -1000 inside a chunk: masking before exp keeps it finite
    cu = np.array([0, 100], np.int32)
    q, k, v, g, beta, S0 = _rand_core(30, 100, 1, 1, 8, 8)
    g[:] = -30.0
    o_r, S_r = oracle.recurrence(q, k, v, g, beta, S0, cu)
    o_c, S_c = oracle.chunked(q, k, v, g, beta, S0, cu, 64)
    assert np.all(np.isfinite(o_c)) and np.all(np.isfinite(S_c))
    assert _relerr(o_c, o_r) < 1e-12
    assert _relerr(S_c, S_r) < 1e-10 or np.linalg.norm(S_r) < 1e-200


def test_resume_is_bit_exact():
    q, k, v, g, beta, S0 = _rand_core(40, 50, 2, 4, 8, 8)
    o, S = oracle.recurrence(q, k, v, g, beta, S0, [0, 50], threads=1)
    o1, S1 = oracle.recurrence(q[:20], k[:20], v[:20], g[:20], beta[:20], S0, [0, 20])
    o2, S2 = oracle.recurrence(q[20:], k[20:], v[20:], g[20:], beta[20:], S1, [0, 30])
    np.testing.assert_array_equal(np.concatenate([o1, o2]), o)
    np.testing.assert_array_equal(S2, S)


def test_value_column_permutation():
    q, k, v, g, beta, S0 = _rand_core(50, 12, 1, 2, 8, 10)
    perm = np.random.default_rng(51).permutation(10)
    o, S = oracle.recurrence(q, k, v, g, beta, S0, [0, 12], threads=1)
    op, Sp = oracle.recurrence(q, k, v[:, :, perm], g, beta, S0[..., perm], [0, 12], threads=1)
    np.testing.assert_array_equal(op, o[:, :, perm])
    np.testing.assert_array_equal(Sp, S[..., perm])


def test_gqa_grouped_equals_duplicated_heads():
    q, k, v, g, beta, S0 = _rand_core(60, 15, 2, 6, 8, 8)
    o, S = oracle.recurrence(q, k, v, g, beta, S0, [0, 15], threads=1)
    # grouped mapping: v-head h reads k-head h // 3
    qd = np.repeat(q, 3, axis=1); kd = np.repeat(k, 3, axis=1)
    od, Sd = oracle.recurrence(qd, kd, v, g, beta, S0, [0, 15], threads=1)
    np.testing.assert_array_equal(o, od)
    np.testing.assert_array_equal(S, Sd)


def test_sequences_are_independent():
    lengths = [3, 11, 6]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    q, k, v, g, beta, S0 = _rand_core(70, 20, 1, 2, 8, 8, n_seqs=3)
    o, S = oracle.recurrence(q, k, v, g, beta, S0, cu, threads=1)
    for n in range(3):
        a, b = cu[n], cu[n + 1]
        on, Sn = oracle.recurrence(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b], S0[n:n + 1],
                                   [0, b - a], threads=1)
        np.testing.assert_array_equal(o[a:b], on)
        np.testing.assert_array_equal(S[n:n + 1], Sn)


def test_thread_count_invariance():
    lengths = [40, 17, 33]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    q, k, v, g, beta, S0 = _rand_core(80, 90, 2, 4, 16, 16, n_seqs=3)
    o1, S1 = oracle.recurrence(q, k, v, g, beta, S0, cu, threads=1)
    o8, S8 = oracle.recurrence(q, k, v, g, beta, S0, cu, threads=8)
    np.testing.assert_array_equal(o1, o8)
    np.testing.assert_array_equal(S1, S8)
    c1 = oracle.chunked(q, k, v, g, beta, S0, cu, 16, threads=1)
    c8 = oracle.chunked(q, k, v, g, beta, S0, cu, 16, threads=7)
    np.testing.assert_array_equal(c1[0], c8[0])


# ----------------------------------------------------------------------- front pins

def _front_case(seed, lengths, H_k=2, H_v=4, d_k=8, d_v=8, d_conv=4):
    r = np.random.default_rng(seed)
    conv_dim = 2 * H_k * d_k + H_v * d_v
    T = sum(lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    x = r.standard_normal((T, conv_dim))
    w = 0.5 * r.standard_normal((conv_dim, max(d_conv, 1)))
    st = r.standard_normal((len(lengths), max(d_conv - 1, 0), conv_dim))
    a = r.standard_normal((T, H_v)); b = r.standard_normal((T, H_v))
    A_log = np.log(r.uniform(1, 16, H_v)); dt_bias = r.standard_normal(H_v)
    return dict(x=x, conv_w=w, conv_state=st, cu_seqlens=cu, a=a, b=b, A_log=A_log,
                dt_bias=dt_bias, H_k=H_k, H_v=H_v, d_k=d_k, d_v=d_v, d_conv=d_conv)


def _call_front(c, **over):
    kw = dict(c)
    kw.update(over)
    return oracle.front(kw["x"], kw["conv_w"], kw["conv_state"], kw["cu_seqlens"], kw["a"],
                        kw["b"], kw["A_log"], kw["dt_bias"], H_k=kw["H_k"], H_v=kw["H_v"],
                        d_k=kw["d_k"], d_v=kw["d_v"], d_conv=kw["d_conv"],
                        eps=kw.get("eps", 1e-6), q_scale=kw.get("q_scale", 1 / math.sqrt(8)),
                        reset=kw.get("reset"), threads=1)


def _silu(y):
    return y * scipy.special.expit(y)


def test_front_one_hot_current_tap_is_identity_conv():
    c = _front_case(100, [6])
    w = np.zeros_like(c["conv_w"]); w[:, 3] = 1.0   # tap 3 = current token
    out = _call_front(c, conv_w=w)
    H_k, d_k = c["H_k"], c["d_k"]
    u = _silu(c["x"])
    np.testing.assert_allclose(out["v"].reshape(6, -1), u[:, 2 * H_k * d_k:], rtol=1e-14)
    uq = u[:, :H_k * d_k].reshape(6, H_k, d_k)
    uk = u[:, H_k * d_k:2 * H_k * d_k].reshape(6, H_k, d_k)
    exp_q = uq / np.sqrt((uq ** 2).sum(-1, keepdims=True) + 1e-6) / math.sqrt(8)
    exp_k = uk / np.sqrt((uk ** 2).sum(-1, keepdims=True) + 1e-6)
    np.testing.assert_allclose(out["q"], exp_q, rtol=1e-13)
    np.testing.assert_allclose(out["k"], exp_k, rtol=1e-13)


def test_front_oldest_tap_reads_conv_state_rows_in_order():
    c = _front_case(101, [5])
    w = np.zeros_like(c["conv_w"]); w[:, 0] = 1.0   # tap 0 = three tokens back
    out = _call_front(c, conv_w=w)
    ext = np.concatenate([c["conv_state"][0], c["x"]], axis=0)   # [state oldest..newest; x]
    u = _silu(ext[:5])
    np.testing.assert_allclose(out["v"].reshape(5, -1), u[:, 2 * 2 * 8:], rtol=1e-14)


def test_front_norms_and_scale():
    c = _front_case(102, [9])
    out = _call_front(c, eps=0.0)
    np.testing.assert_allclose(np.linalg.norm(out["k"], axis=-1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(np.linalg.norm(out["q"], axis=-1), 1 / math.sqrt(8), rtol=1e-14)


def test_front_gates_match_library_routines():
    c = _front_case(103, [7])
    c["a"][0, 0] = 40.0; c["a"][1, 0] = -40.0   # softplus tails
    out = _call_front(c)
    z = c["a"] + c["dt_bias"][None, :]
    exp_g = -np.exp(c["A_log"])[None, :] * np.logaddexp(0.0, z)
    np.testing.assert_allclose(out["g"], exp_g, rtol=1e-14)
    np.testing.assert_allclose(out["beta"], scipy.special.expit(c["b"]), rtol=1e-14)
    assert np.all(out["g"] < 0)


@pytest.mark.parametrize("L", [1, 2, 3, 4, 10])
def test_front_conv_state_rolls(L):
    c = _front_case(104 + L, [L])
    out = _call_front(c)
    ext = np.concatenate([c["conv_state"][0], c["x"]], axis=0)
    np.testing.assert_array_equal(out["conv_state"][0], ext[-3:])


def test_front_reset_zeroes_conv_state():
    c = _front_case(110, [2, 4])
    out_r = _call_front(c, reset=np.array([1, 0], np.uint8))
    zero = dict(c); zero["conv_state"] = c["conv_state"].copy(); zero["conv_state"][0] = 0.0
    out_z = _call_front(zero)
    for key in ("q", "k", "v", "conv_state"):
        np.testing.assert_array_equal(out_r[key], out_z[key])


def test_front_resume_is_bit_exact():
    c = _front_case(111, [12])
    full = _call_front(c)
    a = dict(c); a["x"] = c["x"][:5]; a["a"] = c["a"][:5]; a["b"] = c["b"][:5]
    a["cu_seqlens"] = np.array([0, 5], np.int32)
    first = _call_front(a)
    b2 = dict(c); b2["x"] = c["x"][5:]; b2["a"] = c["a"][5:]; b2["b"] = c["b"][5:]
    b2["cu_seqlens"] = np.array([0, 7], np.int32); b2["conv_state"] = first["conv_state"]
    second = _call_front(b2)
    for key in ("q", "k", "v", "g", "beta"):
        np.testing.assert_array_equal(np.concatenate([first[key], second[key]]), full[key])
    np.testing.assert_array_equal(second["conv_state"], full["conv_state"])


def test_front_without_conv_passes_x_through():
    c = _front_case(112, [4], d_conv=0)
    c["conv_w"] = None; c["conv_state"] = None
    out = _call_front(c)
    H_k, d_k = 2, 8
    xv = c["x"][:, 2 * H_k * d_k:]
    np.testing.assert_array_equal(out["v"].reshape(4, -1), xv)


def test_bf16_decode_is_exact():
    bits = np.array([0x3F80, 0xBF80, 0x4049, 0x0000, 0x8000, 0x7F7F], np.uint16)
    vals = oracle.bf16_bits_to_f64(bits)
    assert vals[0] == 1.0 and vals[1] == -1.0 and vals[3] == 0.0
    assert abs(vals[2] - 3.140625) == 0.0
    assert vals[5] == float(np.finfo(np.float32).max) - 0 or vals[5] > 3e38


# ---------------------------------------------------------------- the other weight family
def _layer_case(layout, seed=80, lengths=(7, 12), H_k=2, H_v=4, d=8):
    import synthetic
    w = synthetic.packed(list(lengths), seed=seed, state_std=0.02, conv_std=1.0, H_k=H_k,
                         H_v=H_v, d_k=d, d_v=d, n_slots=len(lengths), layout=layout)
    return w


def test_tiled_gqa_equals_grouped_with_value_heads_permuted():
    """Tiled GQA (value head h reads key head h % H_k) is the grouped mapping with the value
    heads renumbered: tiled head h = grouped head (h % H_k) r + h // H_k. Running the grouped
    oracle on inputs whose value heads (v channels, gates, A_log, dt_bias, state) are permuted
    that way must give the tiled results permuted the same way."""
    import synthetic
    H_k, H_v, d = 2, 6, 8
    r = H_v // H_k
    wt = _layer_case(synthetic.GQA_TILED, H_k=H_k, H_v=H_v, d=d)
    pi = [(h % H_k) * r + h // H_k for h in range(H_v)]  # tiled head h -> grouped head pi[h]
    inv = np.argsort(pi)
    wg = dict(wt)
    wg["dims"] = dict(wt["dims"], layout=0)
    vc0 = 2 * H_k * d
    # grouped head j holds tiled head inv[j]
    vperm = np.concatenate([np.arange(vc0 + inv[j] * d, vc0 + inv[j] * d + d) for j in range(H_v)])
    perm = np.concatenate([np.arange(vc0), vperm])
    wg["x"] = wt["x"][:, perm]
    wg["conv_state"] = wt["conv_state"][..., perm]
    wg["conv_w"] = wt["conv_w"][perm]
    wg["a"], wg["b"] = wt["a"][:, inv], wt["b"][:, inv]
    wg["A_log"], wg["dt_bias"] = wt["A_log"][inv], wt["dt_bias"][inv]
    wg["state"] = wt["state"][:, inv]
    rt = oracle.layer(wt, threads=1)
    rg = oracle.layer(wg, threads=1)
    np.testing.assert_allclose(rg["o"], rt["o"][:, inv], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(rg["S"], rt["S"][:, inv], rtol=1e-12, atol=1e-15)
    # and a tiled run really differs from reading the heads grouped
    rwrong = oracle.layer(dict(wt, dims=dict(wt["dims"], layout=0)), threads=1)
    assert _relerr(rwrong["o"], rt["o"]) > 1e-2


def test_mixed_beta_alpha_gates_hand_example():
    """The fused beta/alpha input: one key head, two value heads, mixed row [b0, b1, a0, a1]
    (ik_llama.cpp build_layer_attn_linear: per key head the beta logits first, then the
    alphas). The oracle's gates must be beta_h = sigmoid(b_h), g_h = -exp(A_log_h)
    softplus(a_h + dt_bias_h) for these literal values."""
    import synthetic
    w = _layer_case(synthetic.GATES_MIXED_BA, lengths=(1,), H_k=1, H_v=2)
    w["a"] = np.array([[[0.5, -1.25, 2.0, -0.75]]], np.float32)  # [T=1, H_k=1, 2r=4]
    w["A_log"] = np.array([0.25, 1.5], np.float32)
    w["dt_bias"] = np.array([-0.5, 0.3], np.float32)
    r = oracle.layer(w, threads=1)
    b_logit = np.array([0.5, -1.25]); alpha = np.array([2.0, -0.75])
    A = np.array([0.25, 1.5]); dtb = np.array([-0.5, 0.3])
    exp_beta = 1.0 / (1.0 + np.exp(-b_logit))
    exp_g = -np.exp(A) * np.log1p(np.exp(alpha + dtb))
    np.testing.assert_allclose(r["beta"][0], exp_beta, rtol=1e-6)
    np.testing.assert_allclose(r["g"][0], exp_g, rtol=1e-6)


# ---------------------------------------------------------------- output gate
def test_gated_norm_hand_example():
    """One row of d_v = 4: o = [3, 0, -4, 0] (mean square 25/4, RMS 2.5), w = [1, 2, 1, 0.5],
    z = [0, 2, -1, 30], eps = 0: out = o / 2.5 * w * z * sigmoid(z)."""
    o = np.array([[[3.0, 0.0, -4.0, 0.0]]])
    z = np.array([[[0.0, 2.0, -1.0, 30.0]]])
    w = np.array([1.0, 2.0, 1.0, 0.5])
    out = oracle.gated_norm(o, z, w, 0.0)
    silu = np.array([0.0, 2.0 * scipy.special.expit(2.0), -1.0 * scipy.special.expit(-1.0),
                     30.0 * scipy.special.expit(30.0)])
    expect = np.array([3.0 / 2.5, 0.0, -4.0 / 2.5, 0.0]) * w * silu
    np.testing.assert_allclose(out[0, 0], expect, rtol=1e-15, atol=1e-300)


def test_gated_norm_properties():
    g = np.random.default_rng(5)
    o = g.standard_normal((6, 3, 16))
    z = g.standard_normal((6, 3, 16))
    w = g.standard_normal(16)
    base = oracle.gated_norm(o, z, w, 0.0)
    # scale invariance of the RMS norm (eps = 0), per row
    np.testing.assert_allclose(oracle.gated_norm(o * 7.5, z, w, 0.0), base, rtol=1e-13)
    # with unit weight and large z the gate is the identity times z: RMS of out / z is 1
    big = np.full_like(z, 40.0)
    r = oracle.gated_norm(o, big, np.ones(16), 0.0) / 40.0
    np.testing.assert_allclose(np.sqrt(np.mean(r * r, axis=-1)), 1.0, rtol=1e-13)
    # z = 0 closes the gate
    assert np.all(oracle.gated_norm(o, np.zeros_like(z), w, 1e-6) == 0.0)
    # rows are independent: each (token, head) row depends only on itself
    o2 = o.copy(); o2[0, 0] *= 3.0; o2[0, 0, 0] += 1.0
    d = oracle.gated_norm(o2, z, w, 0.0) - base
    assert np.all(d[1:] == 0) and np.all(d[0, 1:] == 0)
