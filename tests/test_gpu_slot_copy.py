"""gdn_state_slot_copy: bit-exact copies of recurrent and conv state rows, device-side slot
checks."""
import numpy as np
import pytest
import torch

from gated_deltanet_linear_19_b200 import Dims, device_status, state_slot_copy
from tests.gpu_util import t_i32

pytestmark = pytest.mark.gpu


def test_slot_copy_bit_exact():
    dims = Dims(n_slots=10, H_k=16, H_v=32, d_k=128, d_v=128, d_conv=4)
    g = torch.Generator(device="cuda").manual_seed(7)
    state = torch.randn((10, 32, 128, 128), device="cuda", generator=g)
    conv = torch.randn((10, 3, dims.conv_dim), device="cuda", generator=g).to(torch.bfloat16)
    s0, c0 = state.clone(), conv.clone()
    src, dst = [1, 4, 7], [9, 0, 2]
    state_slot_copy(dims, state, conv, t_i32(src), t_i32(dst))
    assert device_status() == 0
    for s, d in zip(src, dst):
        assert torch.equal(state[d], s0[s])
        assert torch.equal(conv[d], c0[s])
    rest = [i for i in range(10) if i not in dst]
    assert torch.equal(state[rest], s0[rest])
    assert torch.equal(conv[rest], c0[rest])


def test_slot_copy_repeated_or_read_destinations_are_skipped():
    """A pair whose dst repeats an earlier pair's dst, or is read as a source, is skipped
    (status GDN_ESLOT); the other pairs are copied and no other row changes."""
    dims = Dims(n_slots=8, H_k=2, H_v=4, d_k=32, d_v=32, d_conv=4)
    g = torch.Generator(device="cuda").manual_seed(9)
    state = torch.randn((8, 4, 32, 32), device="cuda", generator=g)
    conv = torch.randn((8, 3, dims.conv_dim), device="cuda", generator=g).to(torch.bfloat16)
    s0, c0 = state.clone(), conv.clone()
    # pair 1 repeats the dst 2 of pair 0; pair 3 writes slot 4, which pair 2 reads: pairs 1
    # and 3 are skipped, pairs 0 (0 -> 2) and 2 (4 -> 6) are copied
    state_slot_copy(dims, state, conv, t_i32([0, 1, 4, 5]), t_i32([2, 2, 6, 4]))
    assert device_status() == -2
    expect_s, expect_c = s0.clone(), c0.clone()
    expect_s[2], expect_c[2] = s0[0], c0[0]
    expect_s[6], expect_c[6] = s0[4], c0[4]
    assert torch.equal(state, expect_s)
    assert torch.equal(conv, expect_c)


def test_slot_copy_rejects_bad_slots():
    dims = Dims(n_slots=4, H_k=2, H_v=4, d_k=32, d_v=32, d_conv=4)
    state = torch.zeros((4, 4, 32, 32), device="cuda")
    state_slot_copy(dims, state, None, t_i32([0]), t_i32([4]))
    assert device_status() == -2
    state_slot_copy(dims, state, None, t_i32([0, 1]), t_i32([2, 2]))
    assert device_status() == -2
    state_slot_copy(dims, state, None, t_i32([0, 1]), t_i32([1, 3]))  # dst used as src
    assert device_status() == -2
