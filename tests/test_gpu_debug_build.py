"""The bounds-checked debug build (libw4a8_debug.so, compiled with
W4A8_DEBUG) on the shapes that exercise every schedule and ragged edge: its
kernels check every global store and workspace access of the GEMM, the
chain and the quantizers against the buffer's extent and report a failed
check as W4A8_DEVERR_BOUNDS instead of performing the access. The results
must still match the CPU oracle, with the device error word clear.

This build and the canary regions of the parity tests stand in for a memory
checker: one catches an out-of-extent index inside the kernel, the other a
write that lands next to a buffer.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import w4a8_quantized_gemm_quantize_b200 as w4a8
from w4a8_quantized_gemm_quantize_b200 import build as w4a8_build
from w4a8_quantized_gemm_quantize_b200 import inputs as I

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from tests import test_gpu_chain as TC  # noqa: E402
from tests import test_gpu_parity as TP  # noqa: E402

DEV = torch.device("cuda:0")


@pytest.fixture
def debug_lib():
    """Swaps the binding onto the debug library for one test."""
    path = w4a8_build.build(debug=True)
    saved = (w4a8._lib, w4a8.library_path)
    w4a8._lib, w4a8.library_path = None, path
    w4a8._default_ws.clear()
    try:
        w4a8.lib()
        w4a8.clear_device_error(DEV)
        yield
        assert w4a8.get_device_error(DEV) == 0
    finally:
        w4a8._lib, w4a8.library_path = saved
        w4a8._default_ws.clear()


def test_debug_library_is_the_debug_build(debug_lib):
    assert w4a8.library_path.endswith("libw4a8_debug.so")


@pytest.mark.parametrize("M", [1, 16, 33])
def test_debug_build_every_schedule(debug_lib, M):
    N, K = 256, 512
    q, z, s2, s1 = I.uniform_codes(N, K, I.weight_seed("tiny", N, K))
    A = I.activations(M, K, I.activation_seed("tiny", M, K))
    TP.check_gemm(A, q, z, s2, s1, TP.ALL_SCHEDULES)


@pytest.mark.parametrize("M,N,K", [(3, 384, 1024), (129, 384, 512), (200, 128, 384), (1, 1024, 4096)])
def test_debug_build_ragged_shapes(debug_lib, M, N, K):
    q, z, s2, s1 = I.uniform_codes(N, K, I.seed_of("t-g", N, K))
    A = I.activations(M, K, I.seed_of("t-a", M, K))
    scheds = [(0, 0, 0), (1, 0, 0), (2, 0, 0), (2, 16, 5), (1, 128, 3)]
    if (N // 128) * -(-M // 16) <= 32:
        scheds += TP.CLUSTER
    TP.check_gemm(A, q, z, s2, s1, scheds)


def test_debug_build_chain(debug_lib):
    links = [TC.make_link(M, N, K, 500 + i) for i, (M, N, K) in enumerate(TC.SHAPES)]
    g = TC.gpu_links(links)
    ws = TC.run_chain(g)
    for L, gl in zip(links, g):
        TC.check_link(gl, L["A_host"], L["codes"])
    assert not ws.any().item()
