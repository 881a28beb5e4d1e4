"""CPU checks of the C ABI: the library loads, exports every symbol include/gdn.h declares,
and host-side argument validation returns the documented status codes without launching
anything (fake pointers are never dereferenced on the host)."""
import ctypes
import os
import re

import pytest

from gated_deltanet_linear_19_b200 import _lib, build as _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return _lib.load()


def _declared():
    text = open(os.path.join(ROOT, "include", "gdn.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    declared = _declared()
    assert declared, "no declarations parsed"
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) == set(_lib.EXPORTS)


def test_abi_version_and_strings(lib):
    assert lib.gdn_abi_version() == 2
    for code in (0, -1, -2, -3, -4, -5, -6, -7):
        s = lib.gdn_status_string(code).decode()
        assert s.startswith("GDN_")
    assert "unknown" in lib.gdn_status_string(-99).decode()


def _dims(**kw):
    d = dict(n_slots=4, H_k=2, H_v=4, d_k=128, d_v=128, d_conv=4)
    d.update(kw)
    return _lib.GdnDims(**d)


A = ctypes.c_void_p(0x100000)      # fake, aligned device pointers (never dereferenced)
B = ctypes.c_void_p(0x200000)
MIS = ctypes.c_void_p(0x100008)    # not 16-byte aligned


def _decode(lib, dims, **over):
    args = dict(q=A, k=A, v=A, qd=_lib.GDN_F32, g=A, beta=A, state=A, slots=B, reset=None,
                n=2, o=A, od=_lib.GDN_BF16)
    args.update(over)
    return lib.gdn_decode_step(ctypes.byref(dims), args["q"], args["k"], args["v"], args["qd"],
                               args["g"], args["beta"], args["state"], args["slots"],
                               args["reset"], args["n"], args["o"], args["od"], None)


def test_decode_host_validation(lib):
    assert lib.gdn_decode_step(None, A, A, A, 0, A, A, A, B, None, 1, A, 0, None) == _lib.GDN_EINVAL
    assert _decode(lib, _dims(), n=0) == _lib.GDN_OK                   # empty: nothing to do
    assert _decode(lib, _dims(), n=-1) == _lib.GDN_EINVAL
    assert _decode(lib, _dims(d_k=96)) == _lib.GDN_EUNSUPPORTED
    assert _decode(lib, _dims(H_v=3)) == _lib.GDN_EINVAL               # H_v % H_k != 0
    assert _decode(lib, _dims(n_slots=0)) == _lib.GDN_EINVAL
    assert _decode(lib, _dims(), state=None) == _lib.GDN_EINVAL
    assert _decode(lib, _dims(), slots=None) == _lib.GDN_EINVAL
    assert _decode(lib, _dims(), state=MIS) == _lib.GDN_EALIGN
    assert _decode(lib, _dims(), o=MIS) == _lib.GDN_EALIGN
    assert _decode(lib, _dims(), qd=7) == _lib.GDN_EINVAL
    assert _decode(lib, _dims(), od=_lib.GDN_F16) == _lib.GDN_EINVAL   # o is F32 or BF16


def test_prefill_host_validation(lib):
    d = _dims()

    def call(**over):
        a = dict(n=1, T=10, chunk=64, flags=0, q=A, state=A, cu=B, slots=B, o=A, ws=None,
                 wsb=0, qd=_lib.GDN_F32)
        a.update(over)
        return lib.gdn_chunked_prefill(ctypes.byref(d), a["q"], A, A, a["qd"], A, A, a["state"],
                                       a["slots"], a["cu"], None, a["n"], a["T"], a["chunk"],
                                       a["o"], _lib.GDN_BF16, a["ws"], a["wsb"], a["flags"],
                                       None)
    assert call(n=0) == _lib.GDN_OK
    assert call(chunk=48) == _lib.GDN_EINVAL
    assert call(T=-1) == _lib.GDN_EINVAL
    assert call(cu=None) == _lib.GDN_EINVAL
    assert call(flags=1 << 7) == _lib.GDN_EINVAL
    assert call(flags=1 << 1) == _lib.GDN_EINVAL  # reserved
    assert call(flags=_lib.GDN_PREFILL_TC_HEAD_SCAN | _lib.GDN_PREFILL_TC_TILE_SCAN) == \
        _lib.GDN_EINVAL
    assert call(q=MIS) == _lib.GDN_EALIGN
    assert call(ws=MIS) == _lib.GDN_EALIGN
    assert call(q=None) == _lib.GDN_EINVAL


def test_conv_step_host_validation(lib):
    d = _dims()

    def call(dims=d, **over):
        a = dict(x=A, xd=_lib.GDN_BF16, w=A, cs=A, csd=_lib.GDN_BF16, cu=B, slots=B, n=1, T=4,
                 eps=1e-6, q=A)
        a.update(over)
        return lib.gdn_conv_step(ctypes.byref(dims), a["x"], a["xd"], a["w"], a["cs"], a["csd"],
                                 a["cu"], a["slots"], None, a["n"], a["T"], A, A, A, A,
                                 a["eps"], 0.1, a["q"], A, A, _lib.GDN_F32, A, A, None)
    assert call(n=0) == _lib.GDN_OK
    assert call(w=None) == _lib.GDN_EINVAL                  # d_conv > 0 needs weights
    assert call(dims=_dims(d_conv=0)) == _lib.GDN_EINVAL    # d_conv == 0 forbids weights/state
    assert call(cs=None) == _lib.GDN_EINVAL
    assert call(xd=_lib.GDN_F16) == _lib.GDN_EINVAL
    assert call(eps=-1.0) == _lib.GDN_EINVAL
    assert call(x=MIS) == _lib.GDN_EALIGN
    assert call(dims=_dims(d_conv=5)) == _lib.GDN_EINVAL


def test_slot_copy_host_validation(lib):
    d = _dims()
    assert lib.gdn_state_slot_copy(ctypes.byref(d), A, None, 0, B, B, 0, None) == _lib.GDN_OK
    assert lib.gdn_state_slot_copy(ctypes.byref(d), None, None, 0, B, B, 1, None) == _lib.GDN_EINVAL
    assert lib.gdn_state_slot_copy(ctypes.byref(d), MIS, None, 0, B, B, 1, None) == _lib.GDN_EALIGN
    assert lib.gdn_state_slot_copy(ctypes.byref(d), A, None, 0, None, B, 1, None) == _lib.GDN_EINVAL


def test_workspace_size_is_host_only(lib):
    d = _dims()
    # fp32 inputs take the SIMT kernel, which needs no workspace
    assert lib.gdn_prefill_workspace_size(ctypes.byref(d), 4096, 1, 64, _lib.GDN_F32, 0) == 0
    assert lib.gdn_prefill_workspace_size(None, 4096, 1, 64, _lib.GDN_F16, 0) == 0


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        saved = _lib._lib
        try:
            _lib._lib = None
            _lib.load(str(tmp_path / "missing.so"))
        finally:
            _lib._lib = saved


def test_layer_prefill_host_validation(lib):
    d = _dims()

    def call(dims=d, **over):
        a = dict(x=A, xd=_lib.GDN_BF16, w=A, cs=A, csd=_lib.GDN_BF16, cu=B, slots=B, n=1,
                 T=100, chunk=64, state=A, o=A, od=_lib.GDN_BF16, ws=A, wsb=1 << 30, flags=0)
        a.update(over)
        return lib.gdn_layer_prefill(ctypes.byref(dims), a["x"], a["xd"], a["w"], a["cs"],
                                     a["csd"], a["cu"], a["slots"], None, a["n"], a["T"], A, A,
                                     A, A, 1e-6, 0.088, a["state"], a["chunk"], a["o"], a["od"],
                                     a["ws"], a["wsb"], a["flags"], a.get("gate"), None)
    assert call(n=0) == _lib.GDN_OK
    assert call(chunk=48) == _lib.GDN_EINVAL
    assert call(cs=None) == _lib.GDN_EINVAL                     # the conv state is required
    assert call(flags=_lib.GDN_PREFILL_SIMT) == _lib.GDN_EINVAL  # tensor-core path only
    assert call(flags=_lib.GDN_PREFILL_TC_HEAD_SCAN | _lib.GDN_PREFILL_TC_TILE_SCAN) == \
        _lib.GDN_EINVAL
    assert call(x=MIS) == _lib.GDN_EALIGN
    assert call(xd=_lib.GDN_F32) == _lib.GDN_EUNSUPPORTED       # bf16 x only
    assert call(csd=_lib.GDN_F32) == _lib.GDN_EUNSUPPORTED      # bf16 conv state only
    assert call(chunk=16) == _lib.GDN_EUNSUPPORTED
    assert call(dims=_dims(d_k=64, d_v=64)) == _lib.GDN_EUNSUPPORTED
    assert call(dims=_dims(d_conv=3)) == _lib.GDN_EUNSUPPORTED
    assert call(ws=None, wsb=0) == _lib.GDN_EWORKSPACE


def test_layer_decode_host_validation(lib):
    d = _dims()
    need = lib.gdn_decode_workspace_size(ctypes.byref(d), 2)
    # fp32 q, k (2 x 2 x 128), v (2 x 4 x 128), g, beta (2 x 4) and the pre-gate o
    # (2 x 4 x 128), each rounded up to 256 bytes
    assert need == 2 * 2048 + 4096 + 2 * 256 + 4096
    assert lib.gdn_decode_workspace_size(None, 2) == 0
    assert lib.gdn_layer_decode_launches(None, 2, 0) == 0
    assert lib.gdn_layer_decode_launches(ctypes.byref(d), 0, 0) == 0
    assert lib.gdn_layer_decode_launches(ctypes.byref(d), 2, 0) in (1, 2)
    assert lib.gdn_layer_decode_launches(ctypes.byref(d), 2, 1) in (1, 3)
    assert lib.gdn_decode_workspace_size(ctypes.byref(d), 0) == 0

    def call(dims=d, **over):
        a = dict(x=A, xd=_lib.GDN_BF16, w=A, cs=A, csd=_lib.GDN_BF16, slots=B, n=2, state=A,
                 o=A, od=_lib.GDN_BF16, ws=A, wsb=need, eps=1e-6)
        a.update(over)
        return lib.gdn_layer_decode(ctypes.byref(dims), a["x"], a["xd"], a["w"], a["cs"],
                                    a["csd"], a["slots"], None, a["n"], A, A, A, A, a["eps"],
                                    0.088, a["state"], a["o"], a["od"], a["ws"], a["wsb"],
                                    a.get("gate"), None)
    assert call(n=0) == _lib.GDN_OK
    assert call(n=-1) == _lib.GDN_EINVAL
    assert call(w=None) == _lib.GDN_EINVAL
    assert call(cs=None) == _lib.GDN_EINVAL
    assert call(slots=None) == _lib.GDN_EINVAL
    assert call(state=None) == _lib.GDN_EINVAL
    assert call(eps=-1.0) == _lib.GDN_EINVAL
    assert call(od=_lib.GDN_F16) == _lib.GDN_EINVAL
    assert call(x=MIS) == _lib.GDN_EALIGN
    assert call(ws=MIS) == _lib.GDN_EALIGN
    assert call(ws=None, wsb=0) == _lib.GDN_EWORKSPACE
    assert call(wsb=need - 1) == _lib.GDN_EWORKSPACE
    assert call(dims=_dims(d_k=96)) == _lib.GDN_EUNSUPPORTED


def test_conv_step_without_cu_seqlens_needs_one_token_per_sequence(lib):
    d = _dims()

    def call(**over):
        a = dict(cu=None, n=3, T=3)
        a.update(over)
        return lib.gdn_conv_step(ctypes.byref(d), A, _lib.GDN_BF16, A, A, _lib.GDN_BF16, a["cu"],
                                 B, None, a["n"], a["T"], A, A, A, A, 1e-6, 0.1, A, A, A,
                                 _lib.GDN_F32, A, A, None)
    assert call(T=4) == _lib.GDN_EINVAL   # NULL cu_seqlens: T_total must equal n_seqs


def test_output_gate_host_validation(lib):
    d = _dims()
    good = _lib.GdnOutGate(0x300000, _lib.GDN_BF16, 0x400000, 1e-6)
    bad_eps = _lib.GdnOutGate(0x300000, _lib.GDN_BF16, 0x400000, -1.0)
    no_w = _lib.GdnOutGate(0x300000, _lib.GDN_BF16, None, 1e-6)
    mis_z = _lib.GdnOutGate(0x300008, _lib.GDN_BF16, 0x400000, 1e-6)
    f16_z = _lib.GdnOutGate(0x300000, _lib.GDN_F16, 0x400000, 1e-6)

    def gn(gate, o=A, od=_lib.GDN_BF16, T=5):
        return lib.gdn_gated_norm(ctypes.byref(d), o, od, None if gate is None else ctypes.byref(gate),
                                  B, _lib.GDN_BF16, T, None)
    assert gn(None) == _lib.GDN_EINVAL
    assert gn(good, T=0) == _lib.GDN_OK
    assert gn(bad_eps) == _lib.GDN_EINVAL
    assert gn(no_w) == _lib.GDN_EINVAL
    assert gn(f16_z) == _lib.GDN_EINVAL
    assert gn(mis_z) == _lib.GDN_EALIGN
    assert gn(good, o=MIS) == _lib.GDN_EALIGN
    assert gn(good, od=_lib.GDN_F16) == _lib.GDN_EINVAL


def test_layout_flags_host_validation(lib):
    # unknown layout bits
    assert _decode(lib, _dims(layout=4)) == _lib.GDN_EINVAL
    # mixed beta/alpha gates: b must be NULL (the fused array is passed as a)
    d = _dims(layout=_lib.GDN_GATES_MIXED_BA)

    def conv(b):
        return lib.gdn_conv_step(ctypes.byref(d), A, _lib.GDN_BF16, A, A, _lib.GDN_BF16, B, B,
                                 None, 1, 4, A, b, A, A, 1e-6, 0.1, A, A, A, _lib.GDN_F32, A, A,
                                 None)
    assert conv(A) == _lib.GDN_EINVAL
    # separate gates need both
    d2 = _dims()
    assert lib.gdn_conv_step(ctypes.byref(d2), A, _lib.GDN_BF16, A, A, _lib.GDN_BF16, B, B, None,
                             1, 4, A, None, A, A, 1e-6, 0.1, A, A, A, _lib.GDN_F32, A, A,
                             None) == _lib.GDN_EINVAL


def test_decode_pipe_host_validation(lib):
    """The host-buffer decode pipeline: its buffer size from the staging layout, and every
    argument check of create / step / flush / destroy that returns before any CUDA call."""
    d = _dims()  # H_k 2, H_v 4, d 128, conv_dim 2 x 2 x 128 + 4 x 128 = 1024
    n = 2
    ws = lib.gdn_decode_workspace_size(ctypes.byref(d), n)
    up = lambda v: (v + 255) // 256 * 256  # noqa: E731
    # per staging set: x (bf16), a, b, slot ids, reset, o (bf16), each rounded up to 256 bytes
    one_set = up(n * 1024 * 2) + 2 * up(n * 4 * 4) + up(n * 4) + up(n) + up(n * 4 * 128 * 2)
    need = lib.gdn_decode_pipe_buffer_size(ctypes.byref(d), n, _lib.GDN_BF16, _lib.GDN_BF16)
    assert need == 2 * one_set + up(ws)
    # the fused beta/alpha layout stages a [n][H_k][2 r] (twice a's size) and no b
    dm = _dims(layout=_lib.GDN_GATES_MIXED_BA)
    one_m = up(n * 1024 * 2) + up(n * 8 * 4) + up(n * 4) + up(n) + up(n * 4 * 128 * 2)
    assert lib.gdn_decode_pipe_buffer_size(ctypes.byref(dm), n, _lib.GDN_BF16,
                                           _lib.GDN_BF16) == 2 * one_m + up(ws)
    assert lib.gdn_decode_pipe_buffer_size(None, n, _lib.GDN_BF16, _lib.GDN_BF16) == 0
    assert lib.gdn_decode_pipe_buffer_size(ctypes.byref(d), 0, _lib.GDN_BF16, _lib.GDN_BF16) == 0
    assert lib.gdn_decode_pipe_buffer_size(ctypes.byref(d), n, _lib.GDN_F16, _lib.GDN_BF16) == 0

    # the packed input row: x, a, b, slot ids, each from a multiple of 256 bytes
    assert lib.gdn_decode_pipe_packed_bytes(ctypes.byref(d), n, _lib.GDN_BF16) == \
        up(n * 1024 * 2) + 2 * up(n * 4 * 4) + n * 4
    assert lib.gdn_decode_pipe_packed_bytes(ctypes.byref(dm), n, _lib.GDN_BF16) == \
        up(n * 1024 * 2) + up(n * 8 * 4) + n * 4
    assert lib.gdn_decode_pipe_packed_bytes(None, n, _lib.GDN_BF16) == 0
    assert lib.gdn_decode_pipe_step_packed(None, A, None, A) == _lib.GDN_EINVAL

    h = ctypes.c_void_p(1)

    def create(**over):
        a = dict(dims=d, n=n, buf=A, bytes=need, state=A, eps=1e-6)
        a.update(over)
        return lib.gdn_decode_pipe_create(ctypes.byref(a["dims"]), a["n"], _lib.GDN_BF16, A, A,
                                          _lib.GDN_BF16, A, A, a["eps"], 0.088, a["state"],
                                          _lib.GDN_BF16, a["buf"], a["bytes"], None,
                                          ctypes.byref(h))
    assert create(n=0) == _lib.GDN_EINVAL and h.value is None
    assert create(state=None) == _lib.GDN_EINVAL
    assert create(eps=-1.0) == _lib.GDN_EINVAL
    assert create(buf=None) == _lib.GDN_EWORKSPACE
    assert create(bytes=need - 1) == _lib.GDN_EWORKSPACE
    assert create(buf=ctypes.c_void_p(0x100010)) == _lib.GDN_EALIGN  # 16- but not 256-aligned
    assert lib.gdn_decode_pipe_create(ctypes.byref(d), n, _lib.GDN_BF16, A, A, _lib.GDN_BF16,
                                      A, A, 1e-6, 0.088, A, _lib.GDN_BF16, A, need, None,
                                      None) == _lib.GDN_EINVAL
    assert lib.gdn_decode_pipe_step(None, A, A, A, A, None, A) == _lib.GDN_EINVAL
    assert lib.gdn_decode_pipe_flush(None) == _lib.GDN_EINVAL
    assert lib.gdn_decode_pipe_destroy(None) == _lib.GDN_OK
