"""tcgen05 building blocks: a single M=128 kind::f16 GEMM through every canonical operand
layout the prefill kernels use (K-major / MN-major A and B, either group stride outermost),
compared with a float64 matmul of the same fp16 inputs."""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def selftest_lib(tmp_path_factory):
    out = tmp_path_factory.mktemp("umma") / "libumma_selftest.so"
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-std=c++17",
                    "-shared", "-Xcompiler", "-fPIC", os.path.join(HERE, "csrc", "umma_selftest.cu"),
                    "-o", str(out)], check=True)
    lib = ctypes.CDLL(str(out))
    lib.umma_selftest.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 5 + [ctypes.c_void_p]
    lib.umma_selftest.restype = ctypes.c_int
    return lib


@pytest.mark.parametrize("N,K", [(32, 128), (64, 64), (64, 128)])
@pytest.mark.parametrize("a_mn", [0, 1])
@pytest.mark.parametrize("b_mn", [0, 1])
@pytest.mark.parametrize("outer_k", [0, 1])
def test_umma_gemm_layouts(selftest_lib, N, K, a_mn, b_mn, outer_k):
    g = torch.Generator().manual_seed(N * 1000 + K + 10 * a_mn + 100 * b_mn + outer_k)
    A = torch.randn(128, K, generator=g).half()
    B = torch.randn(K, N, generator=g).half()
    dA, dB = A.cuda(), B.cuda()
    dD = torch.zeros(128, N, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = selftest_lib.umma_selftest(dA.data_ptr(), dB.data_ptr(), dD.data_ptr(), N, K, a_mn,
                                    b_mn, outer_k, err.data_ptr())
    assert rc == 0 and int(err.item()) == 0
    ref = A.double().numpy() @ B.double().numpy()
    got = dD.cpu().double().numpy()
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel < 1e-6, rel


@pytest.mark.parametrize("N,K", [(32, 128), (128, 64), (64, 128)])
@pytest.mark.parametrize("b_mn", [0, 1])
def test_umma_gemm_a_in_tmem(selftest_lib, N, K, b_mn):
    """A held in tensor memory (row m in lane m, K packed two fp16 per 32-bit column)."""
    selftest_lib.umma_selftest_tmem_a.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 3 + \
        [ctypes.c_void_p]
    selftest_lib.umma_selftest_tmem_a.restype = ctypes.c_int
    g = torch.Generator().manual_seed(7 * N + K + b_mn)
    A = torch.randn(128, K, generator=g).half()
    B = torch.randn(K, N, generator=g).half()
    dA, dB = A.cuda(), B.cuda()
    dD = torch.zeros(128, N, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = selftest_lib.umma_selftest_tmem_a(dA.data_ptr(), dB.data_ptr(), dD.data_ptr(), N, K,
                                           b_mn, err.data_ptr())
    assert rc == 0 and int(err.item()) == 0
    ref = A.double().numpy() @ B.double().numpy()
    got = dD.cpu().double().numpy()
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel < 1e-6, rel


@pytest.mark.parametrize("abort_first", [0, 1])
def test_bounded_wait_gives_up_and_drains(selftest_lib, abort_first):
    """The time-out path of the kernels' bounded mbarrier waits (umma.cuh mbar_wait): a wait
    on a barrier that nothing completes gives up (after a short cycle limit, or once the abort
    flag is seen), the kernel records GDN_ETIMEOUT, drains the MMA it issued, frees its TMEM
    and returns; the device then still runs a normal GEMM correctly."""
    lib = selftest_lib
    lib.umma_selftest_timeout.argtypes = [ctypes.c_void_p, ctypes.c_longlong, ctypes.c_int,
                                          ctypes.c_void_p]
    lib.umma_selftest_timeout.restype = ctypes.c_int
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    drained = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = lib.umma_selftest_timeout(status.data_ptr(), 200000, abort_first, drained.data_ptr())
    assert rc == 0
    assert int(status.item()) == -5   # GDN_ETIMEOUT
    assert int(drained.item()) == 1
    # the context is still usable
    test_umma_gemm_layouts(selftest_lib, 64, 64, 0, 1, 0)


@pytest.mark.parametrize("N,K,a_mn,b_mn", [(64, 64, 0, 0), (128, 128, 0, 0), (64, 128, 0, 1),
                                           (128, 64, 1, 1), (128, 128, 1, 0), (256, 64, 0, 1),
                                           (32, 128, 0, 0), (64, 64, 1, 1)])
def test_umma_gemm_swizzle128(selftest_lib, N, K, a_mn, b_mn):
    """Operands in the 128-byte swizzled layouts that TMA writes (K-major and MN-major)."""
    lib = selftest_lib
    lib.umma_selftest_sw128.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 4 + \
        [ctypes.c_void_p]
    lib.umma_selftest_sw128.restype = ctypes.c_int
    g = torch.Generator().manual_seed(11 * N + K + 3 * a_mn + 5 * b_mn)
    A = torch.randn(128, K, generator=g).half()
    B = torch.randn(K, N, generator=g).half()
    dA, dB = A.cuda(), B.cuda()
    dD = torch.zeros(128, N, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = lib.umma_selftest_sw128(dA.data_ptr(), dB.data_ptr(), dD.data_ptr(), N, K, a_mn, b_mn,
                                 err.data_ptr())
    assert rc == 0 and int(err.item()) == 0
    ref = A.double().numpy() @ B.double().numpy()
    got = dD.cpu().double().numpy()
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel < 1e-6, rel


def test_prefill_wait_time_out_path():
    """The tensor-core prefill's record kernel with its wait limit cut to one cycle: a wait
    runs out (the TMA loads or MMAs it waits for cannot be done that soon), the call records
    GDN_ETIMEOUT, the blocks drain what they issued and end; with the default limit restored
    the next call on the same context matches the oracle again."""
    import oracle
    import synthetic
    from gated_deltanet_linear_19_b200 import _lib, device_status
    from tests.gpu_util import rel_l2, run_prefill
    lib = _lib.load()
    w = synthetic.packed([200, 70], seed=750, slots=[1, 0], state_std=0.02, conv_std=1.0,
                         n_slots=2)
    assert lib.gdn_debug_set_wait_limit(1) == 0
    try:
        run_prefill(w, fused=False)
        assert device_status() == -5  # GDN_ETIMEOUT
    finally:
        assert lib.gdn_debug_set_wait_limit(0) == 0
    o, S, _, _ = run_prefill(w, fused=False)
    assert device_status() == 0
    ref = oracle.layer(w)
    assert rel_l2(o, ref["o"]) < 2e-3
    assert rel_l2(S[w["slot_ids"]], ref["S"]) < 2e-3
