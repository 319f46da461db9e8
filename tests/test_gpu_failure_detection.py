"""Failure detection on the GPU without a GPU fault: every wait in the
library's kernels is bounded in time and, when it runs out, records a code in
the device error word and lets the kernel return. The self-test entry point
runs that same bounded wait on an mbarrier nothing ever completes (a flag that
nothing sets), with a short limit; the host then reads the code, clears it and
checks that the context still computes correct results."""
import time

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import w4a8_quantized_gemm_quantize_b200 as w4a8
from w4a8_quantized_gemm_quantize_b200 import inputs as I
from oracle import w4a8_oracle as O

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

DEV = torch.device("cuda:0")


def _small_gemm_matches_oracle():
    M, N, K = 4, 256, 512
    q, z, s2, s1 = I.uniform_codes(N, K, I.seed_of("t-fd", N, K))
    A = I.activations(M, K, I.seed_of("t-fda", M, K))
    blob = w4a8.pack_weights(*(torch.from_numpy(x).to(DEV) for x in (q, z, s2, s1)))
    A8, sA, rs = w4a8.quantize_act(torch.from_numpy(A).to(DEV))
    acc = w4a8.gemm_debug_acc(A8, rs, blob, N, K)
    oA8, _, _ = O.quantize_act(A)
    return (acc.cpu().numpy() == O.gemm_acc(oA8, O.dequant_weights(q, z, s2))).all()


def test_bounded_wait_gives_up_and_reports():
    w4a8.clear_device_error(DEV)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    w4a8.selftest_bounded_wait(20_000_000)  # 20 ms
    code = w4a8.get_device_error(DEV)  # synchronizes the stream
    dt = time.perf_counter() - t0
    assert code == w4a8.DEVERR_SELFTEST_WAIT
    assert 0.015 <= dt < 1.5, dt
    # the first code stays until cleared
    w4a8.selftest_bounded_wait(1_000)
    assert w4a8.get_device_error(DEV) == w4a8.DEVERR_SELFTEST_WAIT
    w4a8.clear_device_error(DEV)
    assert w4a8.get_device_error(DEV) == 0


def test_context_usable_after_a_wait_gave_up():
    w4a8.selftest_bounded_wait(5_000_000)
    assert w4a8.get_device_error(DEV) == w4a8.DEVERR_SELFTEST_WAIT
    w4a8.clear_device_error(DEV)
    assert _small_gemm_matches_oracle()
    torch.cuda.synchronize()
    assert w4a8.get_device_error(DEV) == 0
