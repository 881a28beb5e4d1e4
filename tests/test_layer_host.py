"""Host-side dispatch of GDNLayer.prefill (no GPU needed): the layer prefill (front inside the
prefill's first kernel) is chosen exactly where the library supports it."""
import torch

from gated_deltanet_linear_19_b200 import (GDN_PREFILL_RECURRENT, GDN_PREFILL_SIMT,
                                           GDN_PREFILL_TC_HEAD_SCAN, Dims)
from gated_deltanet_linear_19_b200.layer import GDNLayer


def _layer(d=128, d_conv=4, conv_dtype=torch.bfloat16, qkv=torch.float16):
    dims = Dims(n_slots=2, H_k=2, H_v=4, d_k=d, d_v=d, d_conv=d_conv)
    conv_w = torch.zeros(dims.conv_dim, max(d_conv, 1))
    return GDNLayer(dims, conv_w if d_conv > 0 else None, torch.zeros(4), torch.zeros(4),
                    device="cpu", conv_dtype=conv_dtype, prefill_qkv_dtype=qkv)


def test_layer_prefill_applies_to_the_tensor_core_shape():
    L = _layer()
    x = torch.zeros(10, L.dims.conv_dim, dtype=torch.bfloat16)
    assert L.fused_prefill_applies(x)
    assert L.fused_prefill_applies(x, flags=GDN_PREFILL_TC_HEAD_SCAN)


def test_layer_prefill_does_not_apply_elsewhere():
    x16 = lambda L: torch.zeros(10, L.dims.conv_dim, dtype=torch.bfloat16)
    L = _layer()
    assert not L.fused_prefill_applies(x16(L), flags=GDN_PREFILL_SIMT)
    assert not L.fused_prefill_applies(x16(L), flags=GDN_PREFILL_RECURRENT)
    assert not L.fused_prefill_applies(x16(L), chunk=16)
    assert not L.fused_prefill_applies(torch.zeros(10, L.dims.conv_dim))      # fp32 x
    assert not L.fused_prefill_applies(x16(L), qkv_dtype=torch.float32)
    assert not _layer(d=64).fused_prefill_applies(x16(_layer(d=64)))
    assert not _layer(d_conv=3).fused_prefill_applies(x16(_layer(d_conv=3)))
    assert not _layer(conv_dtype=torch.float32).fused_prefill_applies(
        x16(_layer(conv_dtype=torch.float32)))
    assert not _layer(d_conv=0).fused_prefill_applies(x16(_layer(d_conv=0)))
