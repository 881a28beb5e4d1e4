"""The host-buffer decode pipeline (gdn_decode_pipe_*): steps fed from pinned host memory and
returned to it give exactly the results of gdn_layer_decode on device buffers (outputs, state
and conv pools bit for bit), on both layer-decode paths (one kernel at small batches, front +
decode at large ones), with per-step slot ids and reset flags from the host and the fused
beta/alpha gate layout; and the first steps against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from gated_deltanet_linear_19_b200 import device_status
from tests.gpu_util import assert_heads, by_sequence, make_layer, t_bits, t_f32, t_i32

pytestmark = pytest.mark.gpu


def _pinned(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.pin_memory()


def _packed_rows(pipe, w, slots, steps):
    """One pinned host row per step: x, a, b, slot ids at the pipeline's packed offsets."""
    ox, oa, ob, osl = pipe.packed_offsets
    rows = torch.zeros((steps, pipe.packed_bytes), dtype=torch.uint8)
    for s in range(steps):
        parts = [(ox, np.ascontiguousarray(w["x"][s])),
                 (oa, np.ascontiguousarray(w["a"][s], np.float32)),
                 (osl, np.ascontiguousarray(slots[s], np.int32))]
        if ob is not None:
            parts.append((ob, np.ascontiguousarray(w["b"][s], np.float32)))
        for off, arr in parts:
            bts = torch.from_numpy(arr).view(torch.uint8).reshape(-1)
            rows[s, off:off + bts.numel()] = bts
    return rows.pin_memory()


@pytest.mark.parametrize("B,layout,packed", [(4, 0, False), (64, 0, False), (64, 0, True),
                                             (8, synthetic.GQA_TILED | synthetic.GATES_MIXED_BA,
                                              False),
                                             (8, synthetic.GQA_TILED | synthetic.GATES_MIXED_BA,
                                              True)])
def test_pipe_equals_layer_decode(B, layout, packed):
    steps = 6
    w = synthetic.decode(seed=880 + B, steps=steps, n_seqs=B, n_slots=B + 3, layout=layout)
    r = np.random.default_rng(881 + B)
    slots = [r.permutation(B + 3)[:B].astype(np.int32) for _ in range(steps)]
    resets = [(r.random(B) < 0.25).astype(np.uint8) if s in (0, 3) else None
              for s in range(steps)]
    l1, l2 = make_layer(w), make_layer(w)
    # reference: gdn_layer_decode on device buffers
    ref_o = []
    for s in range(steps):
        b = None if w["b"] is None else t_f32(w["b"][s])
        rs = None if resets[s] is None else torch.from_numpy(resets[s]).cuda()
        ref_o.append(l1.decode(t_bits(w["x"][s]), t_f32(w["a"][s]), b, t_i32(slots[s]),
                               reset=rs).cpu())
    # the pipeline, from pinned host buffers (kept alive until the end)
    pipe = l2.decode_pipe(B)
    xs = [_pinned(w["x"][s], torch.bfloat16) for s in range(steps)]
    as_ = [_pinned(np.asarray(w["a"][s], np.float32)) for s in range(steps)]
    bs = [None if w["b"] is None else _pinned(np.asarray(w["b"][s], np.float32))
          for s in range(steps)]
    ss = [_pinned(slots[s]) for s in range(steps)]
    rsh = [None if resets[s] is None else _pinned(resets[s]) for s in range(steps)]
    outs = [torch.empty((B, w["dims"]["H_v"], w["dims"]["d_v"]), dtype=torch.bfloat16)
            .pin_memory() for _ in range(steps)]
    rows = _packed_rows(pipe, w, slots, steps) if packed else None
    for s in range(steps):
        if packed:
            pipe.step_packed_ptr(rows[s].data_ptr(),
                                 None if rsh[s] is None else rsh[s].data_ptr(),
                                 outs[s].data_ptr())
        else:
            pipe.step(xs[s], as_[s], bs[s], ss[s], outs[s], reset=rsh[s])
    pipe.flush()
    torch.cuda.synchronize()
    assert device_status() == 0
    for s in range(steps):
        assert torch.equal(outs[s], ref_o[s]), s
    assert torch.equal(l1.state, l2.state)
    assert torch.equal(l1.conv_state, l2.conv_state)
    pipe.close()


def test_pipe_first_steps_against_oracle():
    B, steps = 16, 3
    w = synthetic.decode(seed=890, steps=steps, n_seqs=B)
    layer = make_layer(w)
    pipe = layer.decode_pipe(B, stream=torch.cuda.current_stream())
    keep = []
    outs = []
    for s in range(steps):
        x = _pinned(w["x"][s], torch.bfloat16)
        a = _pinned(np.asarray(w["a"][s], np.float32))
        b = _pinned(np.asarray(w["b"][s], np.float32))
        sl = _pinned(w["slot_ids"])
        o = torch.empty((B, 32, 128), dtype=torch.bfloat16).pin_memory()
        keep += [x, a, b, sl]
        outs.append(o)
        pipe.step(x, a, b, sl, o)
    pipe.flush()
    torch.cuda.synchronize()
    assert device_status() == 0
    ref = oracle.decode_steps(w, steps)
    og, cu = by_sequence(np.stack([o.float().numpy() for o in outs]))
    eg, _ = by_sequence(ref["o"])
    assert_heads(og, eg, 2e-3, cu=cu, label="pipe o", bf16_out=True)
    assert_heads(layer.state.cpu().numpy()[w["slot_ids"]], ref["S"], 1e-5, label="pipe S")
    pipe.close()
