"""The allocation-free GEMM entry point (w4a8_gemm_noalloc).

Some callers cannot give the library a workspace: a plugin inside a host
engine that owns and plans all device memory, or a serving loop that must
not call the allocator after start-up. For them the library keeps its own
scratch array in device memory. This file checks, through the C ABI, that
two calls in a row give exactly the output of the regular entry point
(w4a8_gemm with a caller workspace: the same kernel on a zeroed scratch, so
bit for bit), that the output is within 1 fp16 ulp of the CPU oracle (the
tolerance of the other GEMM tests), that a call after a larger one (whose
partial sums covered more of the array) is still exact, and that a shape
needing more scratch than the array holds, or a misaligned pointer, is
refused before anything is launched. It runs last and also passes alone in
a fresh process.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import w4a8_quantized_gemm_quantize_b200 as w4a8
from w4a8_quantized_gemm_quantize_b200 import build as w4a8_build
from w4a8_quantized_gemm_quantize_b200 import inputs as I
from oracle import w4a8_oracle as O
from tests._util import max_ulp_fp16

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

DEV = torch.device("cuda:0")


def _case(M, N, K, seed):
    codes = I.uniform_codes(N, K, seed)
    q, z, s2, s1 = (torch.from_numpy(x).to(DEV) for x in codes)
    blob = w4a8.pack_weights(q, z, s2, s1)
    A_host = I.activations(M, K, seed + 1)
    A8, sA, rs = w4a8.quantize_act(torch.from_numpy(A_host).to(DEV))
    # the expected output, from the oracle alone
    oA8, osA, _ = O.quantize_act(A_host)
    oq, oz, os2, os1 = codes
    Y_oracle = O.epilogue(O.gemm_acc(oA8, O.dequant_weights(oq, oz, os2)), osA, os1)
    return A8, sA, rs, blob, Y_oracle


def _workspace_gemm(L, A8, sA, rs, blob, M, N, K):
    ws = torch.zeros(w4a8.workspace_bytes(M, N, K), dtype=torch.uint8, device=DEV)
    Y = torch.empty((M, N), dtype=torch.float16, device=DEV)
    code = L.w4a8_gemm(ctypes.c_void_p(A8.data_ptr()), ctypes.c_void_p(sA.data_ptr()),
                       ctypes.c_void_p(rs.data_ptr()), ctypes.c_void_p(blob.data_ptr()), M, N, K,
                       ctypes.c_void_p(Y.data_ptr()), ctypes.c_void_p(ws.data_ptr()), ws.numel(),
                       ctypes.c_void_p(torch.cuda.current_stream(DEV).cuda_stream))
    assert code == 0, w4a8.status_string(code)
    return Y


def _noalloc(L, A8, sA, rs, blob, M, N, K, Y):
    stream = ctypes.c_void_p(torch.cuda.current_stream(DEV).cuda_stream)
    return L.w4a8_gemm_noalloc(ctypes.c_void_p(A8.data_ptr()), ctypes.c_void_p(sA.data_ptr()),
                               ctypes.c_void_p(rs.data_ptr()), ctypes.c_void_p(blob.data_ptr()), M, N, K, ctypes.c_void_p(Y.data_ptr()), stream)


# cluster-split shapes (no scratch used) and stream-K shapes (partial sums
# and tickets in the scratch array)
@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (16, 6144, 4096), (32, 4096, 14336), (33, 1024, 512),
                                   (16, 28672, 4096), (64, 16384, 1024)])
def test_noalloc_matches_workspace_entry_point_twice(M, N, K):
    w4a8_build.build()
    L = w4a8.lib()
    A8, sA, rs, blob, Y_oracle = _case(M, N, K, I.seed_of("noalloc", M, N, K))
    Y_ref = _workspace_gemm(L, A8, sA, rs, blob, M, N, K)
    for _ in range(2):  # the second call finds the scratch array used by the first
        Y = torch.full((M, N), float("nan"), dtype=torch.float16, device=DEV)
        code = _noalloc(L, A8, sA, rs, blob, M, N, K, Y)
        assert code == 0, w4a8.status_string(code)
        torch.cuda.synchronize()
        assert torch.equal(Y, Y_ref)
        assert max_ulp_fp16(Y.cpu().numpy(), Y_oracle) <= 1
    assert w4a8.get_device_error(DEV) == 0


def test_noalloc_after_a_larger_call():
    """A larger stream-K call first (its partial sums span more of the array),
    then a smaller one: the second must still be exact."""
    w4a8_build.build()
    L = w4a8.lib()
    for (M, N, K) in [(32, 28672, 4096), (16, 28672, 4096), (5, 8192, 1024)]:
        A8, sA, rs, blob, Y_oracle = _case(M, N, K, I.seed_of("noalloc-seq", M, N, K))
        Y_ref = _workspace_gemm(L, A8, sA, rs, blob, M, N, K)
        Y = torch.full((M, N), float("nan"), dtype=torch.float16, device=DEV)
        code = _noalloc(L, A8, sA, rs, blob, M, N, K, Y)
        assert code == 0, w4a8.status_string(code)
        torch.cuda.synchronize()
        assert torch.equal(Y, Y_ref)
        assert max_ulp_fp16(Y.cpu().numpy(), Y_oracle) <= 1
    assert w4a8.get_device_error(DEV) == 0


def test_noalloc_rejects_bad_arguments_before_launching():
    w4a8_build.build()
    L = w4a8.lib()
    M, N, K = 16, 1024, 512
    A8, sA, rs, blob, _ = _case(M, N, K, I.seed_of("noalloc-bad", M, N, K))
    Yb = torch.zeros((M * N + 8,), dtype=torch.float16, device=DEV)
    Y_mis = Yb[1:1 + M * N].view(M, N)  # 2-byte offset: not 16-byte aligned
    assert w4a8.status_string(_noalloc(L, A8, sA, rs, blob, M, N, K, Y_mis)) == "W4A8_ERR_MISALIGNED"
    assert w4a8.status_string(_noalloc(L, A8, sA, rs, blob, M, N, 100, Yb)) == "W4A8_ERR_UNSUPPORTED_SHAPE"
    torch.cuda.synchronize()
    assert not Yb.any()  # nothing was launched


def test_noalloc_refuses_shapes_beyond_its_scratch():
    w4a8_build.build()
    L = w4a8.lib()
    M, N, K = 64, 49152, 128       # needs 12.6 MB of scratch > 8 MiB
    assert w4a8.workspace_bytes(M, N, K) > w4a8.NOALLOC_SCRATCH_BYTES
    A8 = torch.zeros((M, K), dtype=torch.int8, device=DEV)
    sA = torch.zeros((M,), dtype=torch.float16, device=DEV)
    rs = torch.zeros((M,), dtype=torch.int32, device=DEV)
    blob = torch.zeros((w4a8.packed_bytes(N, K),), dtype=torch.uint8, device=DEV)
    Y = torch.zeros((M, N), dtype=torch.float16, device=DEV)
    code = _noalloc(L, A8, sA, rs, blob, M, N, K, Y)
    assert w4a8.status_string(code) == "W4A8_ERR_WORKSPACE"
    torch.cuda.synchronize()
    assert not Y.any()  # nothing was launched
