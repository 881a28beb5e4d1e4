"""gdn_chunked_prefill_noalloc: the prefill entry point for callers that cannot allocate
device memory (a host framework that owns all device allocations, or a latency-critical loop
that must not call cudaMalloc). It uses the library's fixed device scratch array instead of a
caller workspace and runs the same kernels as gdn_chunked_prefill's tensor-core path, so its
results must equal that entry point's bit for bit on two calls in a row (the second call must
not see anything left over from the first), and match the fp64 oracle; an input that does
not fit the fixed scratch must be rejected before any launch. Collected last on purpose."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from gated_deltanet_linear_19_b200 import (GDN_EWORKSPACE, GdnError, chunked_prefill,
                                           chunked_prefill_noalloc, conv_step, device_status)
from tests.gpu_util import dims_of, make_layer, rel_l2, t_bits, t_f32, t_i32

pytestmark = pytest.mark.gpu

TOL = 2e-3


def _front(w, layer):
    T = int(w["cu_seqlens"][-1])
    q, k, v, g, beta = (t.clone() for t in layer._front_bufs(T, torch.float16))
    conv_step(layer.dims, t_bits(w["x"]), layer.conv_w, layer.conv_state, t_i32(w["cu_seqlens"]),
              t_i32(w["slot_ids"]), t_f32(w["a"]), t_f32(w["b"]), layer.A_log, layer.dt_bias,
              q, k, v, g, beta, eps=w["eps"], q_scale=w["q_scale"])
    return q, k, v, g, beta


@pytest.mark.parametrize("seed,lengths", [(801, [700, 333]), (802, [64, 1, 900])])
def test_noalloc_matches_workspace_entry_point_twice(seed, lengths):
    w = synthetic.packed(lengths, seed=seed, state_std=0.02, conv_std=1.0,
                         n_slots=len(lengths))
    layer = make_layer(w)
    q, k, v, g, beta = _front(w, layer)
    T = q.shape[0]
    slots, cu = t_i32(w["slot_ids"]), t_i32(w["cu_seqlens"])
    dims = dims_of(w)
    state0 = t_f32(w["state"])
    # reference: the workspace entry point
    s_ref = state0.clone()
    o_ref = torch.empty((T, dims.H_v, dims.d_v), dtype=torch.bfloat16, device="cuda")
    chunked_prefill(dims, q, k, v, g, beta, s_ref, slots, cu, o_ref)
    assert device_status() == 0
    for _ in range(2):  # two calls in a row on the shared scratch
        s_na = state0.clone()
        o_na = torch.full_like(o_ref, float("nan"))
        chunked_prefill_noalloc(dims, q, k, v, g, beta, s_na, slots, cu, o_na)
        assert device_status() == 0
        assert torch.equal(o_na, o_ref)
        assert torch.equal(s_na, s_ref)
    # and against the fp64 oracle (front + per-token recurrence)
    ref = oracle.layer(w)
    assert rel_l2(o_na.float().cpu().numpy(), ref["o"]) < TOL
    assert rel_l2(s_na.cpu().numpy()[w["slot_ids"]], ref["S"]) < TOL


def test_noalloc_rejects_inputs_beyond_the_fixed_scratch():
    w = synthetic.packed([4000], seed=803, n_slots=1)
    layer = make_layer(w)
    dims = dims_of(w)
    T = 4000
    q, k, v, g, beta = layer._front_bufs(T, torch.float16)
    o = torch.empty((T, dims.H_v, dims.d_v), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(GdnError) as e:
        chunked_prefill_noalloc(dims, q, k, v, g, beta, layer.state, t_i32(w["slot_ids"]),
                                t_i32(w["cu_seqlens"]), o)
    assert e.value.status == GDN_EWORKSPACE
