"""The allocation-free GEMM entry point (w4a8_gemm_noalloc).

Some callers cannot give the library a workspace: a plugin inside a host
engine that owns and plans all device memory, or a serving loop that must
not call the allocator after start-up. For them the library keeps its own
scratch array in device memory. This file checks, through the C ABI, that
two calls in a row give the same output as the regular entry point
(w4a8_gemm with a caller workspace), within the tolerance the other GEMM
tests use, and that a shape needing more scratch than the array holds is
refused. It runs last and also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import w4a8_quantized_gemm_quantize_b200 as w4a8
from w4a8_quantized_gemm_quantize_b200 import build as w4a8_build
from w4a8_quantized_gemm_quantize_b200 import inputs as I
from tests._util import max_ulp_fp16

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

DEV = torch.device("cuda:0")


def _case(M, N, K, seed):
    q, z, s2, s1 = (torch.from_numpy(x).to(DEV) for x in I.uniform_codes(N, K, seed))
    blob = w4a8.pack_weights(q, z, s2, s1)
    A = torch.from_numpy(I.activations(M, K, seed + 1)).to(DEV)
    A8, sA, rs = w4a8.quantize_act(A)
    return A8, sA, rs, blob


def _noalloc(L, A8, sA, rs, blob, M, N, K, Y):
    stream = ctypes.c_void_p(torch.cuda.current_stream(DEV).cuda_stream)
    return L.w4a8_gemm_noalloc(ctypes.c_void_p(A8.data_ptr()), ctypes.c_void_p(sA.data_ptr()),
                               ctypes.c_void_p(rs.data_ptr()), ctypes.c_void_p(blob.data_ptr()), M, N, K, ctypes.c_void_p(Y.data_ptr()), stream)


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (16, 6144, 4096), (32, 4096, 14336), (33, 1024, 512)])
def test_noalloc_matches_workspace_entry_point_twice(M, N, K):
    w4a8_build.build()
    L = w4a8.lib()
    A8, sA, rs, blob = _case(M, N, K, I.seed_of("noalloc", M, N, K))
    ws = torch.zeros(w4a8.workspace_bytes(M, N, K), dtype=torch.uint8, device=DEV)
    Y_ref = torch.empty((M, N), dtype=torch.float16, device=DEV)
    code = L.w4a8_gemm(ctypes.c_void_p(A8.data_ptr()), ctypes.c_void_p(sA.data_ptr()),
                       ctypes.c_void_p(rs.data_ptr()), ctypes.c_void_p(blob.data_ptr()), M, N, K, ctypes.c_void_p(Y_ref.data_ptr()),
                       ctypes.c_void_p(ws.data_ptr()), ws.numel(),
                       ctypes.c_void_p(torch.cuda.current_stream(DEV).cuda_stream))
    assert code == 0, w4a8.status_string(code)
    for _ in range(2):  # the second call finds the scratch array used by the first
        Y = torch.full((M, N), float("nan"), dtype=torch.float16, device=DEV)
        code = _noalloc(L, A8, sA, rs, blob, M, N, K, Y)
        assert code == 0, w4a8.status_string(code)
        torch.cuda.synchronize()
        assert max_ulp_fp16(Y.cpu().numpy(), Y_ref.cpu().numpy()) <= 1
    assert w4a8.get_device_error(DEV) == 0


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
