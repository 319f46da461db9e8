"""The C-ABI library builds for sm_100a, loads without a GPU, exports every
entry point that include/w4a8.h declares, and rejects bad arguments on the
host before any launch (no CUDA call is reached by these cases)."""
import ctypes
import os
import re

import numpy as np
import pytest

import w4a8_quantized_gemm_quantize_b200 as w4a8
from w4a8_quantized_gemm_quantize_b200 import build as w4a8_build
from oracle import w4a8_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4a8.h")


@pytest.fixture(scope="module")
def L():
    w4a8_build.build()
    return w4a8.lib()


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"W4A8_API\s+[\w\s\*]+?\b(w4(?:a[48]|lut3?|kv)_\w+)\s*\(", src)))


def test_header_declares_entry_points():
    names = declared_functions()
    assert set(names) == set(w4a8.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value


def test_status_strings(L):
    assert w4a8.status_string(0) == "W4A8_OK"
    assert w4a8.status_string(2) == "W4A8_ERR_UNSUPPORTED_SHAPE"
    assert w4a8.status_string(99) == "W4A8_ERR_UNKNOWN"
    assert L.w4a8_version() == 100


@pytest.mark.parametrize("N,K", [(128, 128), (256, 512), (4096, 14336), (49152, 8192)])
def test_packed_bytes_matches_layout(L, N, K):
    assert w4a8.packed_bytes(N, K) == O.packed_bytes(N, K)


def test_packed_bytes_rejects(L):
    assert w4a8.packed_bytes(100, 128) == 0
    assert w4a8.packed_bytes(128, 100) == 0
    assert w4a8.packed_bytes(128, 128, 64) == 0
    assert w4a8.packed_bytes(128, 65536 + 128) == 0


def test_workspace_bytes(L):
    assert w4a8.workspace_bytes(0, 4096, 4096) == 0
    ws = w4a8.workspace_bytes(32, 4096, 4096)
    assert ws >= 32 * 4096 * 4 + 32 * 4
    assert w4a8.workspace_bytes(16, 4096, 4096) <= ws


FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: validation fails first
FAKE_ODD = ctypes.c_void_p(0x10001)


def test_quantize_act_validation(L):
    f = L.w4a8_quantize_act
    assert f(FAKE, 4, 7, FAKE, FAKE, None, None) == 2        # K % 8
    assert f(FAKE, 4, 0, FAKE, FAKE, None, None) == 2
    assert f(FAKE, 4, 65544, FAKE, FAKE, None, None) == 2    # K too large
    assert f(FAKE, -1, 128, FAKE, FAKE, None, None) == 1
    assert f(None, 4, 128, FAKE, FAKE, None, None) == 1
    assert f(FAKE_ODD, 4, 128, FAKE, FAKE, None, None) == 3
    assert f(FAKE, 0, 128, None, None, None, None) == 0      # M == 0: no-op


def test_quantize_act_static_validation(L):
    f = L.w4a8_quantize_act_static
    assert f(FAKE, 4, 7, FAKE, FAKE, FAKE, None, None) == 2        # K % 8
    assert f(FAKE, 4, 128, None, FAKE, FAKE, None, None) == 1      # no scale
    assert f(FAKE, 4, 128, FAKE_ODD, FAKE, FAKE, None, None) == 3  # scale alignment
    assert f(FAKE_ODD, 4, 128, FAKE, FAKE, FAKE, None, None) == 3
    assert f(FAKE, 0, 128, None, None, None, None, None) == 0      # M == 0: no-op


def test_quantize_weights_validation(L):
    f = L.w4a8_quantize_weights
    assert f(FAKE, 128, 100, 128, FAKE, FAKE, FAKE, FAKE, None) == 2
    assert f(FAKE, 128, 128, 64, FAKE, FAKE, FAKE, FAKE, None) == 2
    assert f(None, 128, 128, 128, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert f(FAKE, 0, 128, 128, None, None, None, None, None) == 0


def test_pack_validation(L):
    f = L.w4a8_pack_weights
    nb = w4a8.packed_bytes(256, 256)
    assert f(FAKE, FAKE, FAKE, FAKE, 200, 256, 128, FAKE, nb, None) == 2
    assert f(FAKE, FAKE, FAKE, FAKE, 256, 256, 128, FAKE, nb - 1, None) == 1
    assert f(FAKE_ODD, FAKE, FAKE, FAKE, 256, 256, 128, FAKE, nb, None) == 3


def test_gemm_validation(L):
    g = L.w4a8_gemm
    assert g(FAKE, FAKE, FAKE, FAKE, 4, 100, 256, FAKE, None, 0, None) == 2      # N % 128
    assert g(FAKE, FAKE, FAKE, FAKE, 4, 128, 200, FAKE, None, 0, None) == 2      # K % 128
    assert g(FAKE, FAKE, FAKE, FAKE, 4, 128, 65536 + 128, FAKE, None, 0, None) == 2
    assert g(FAKE, FAKE, FAKE, FAKE, -2, 128, 256, FAKE, None, 0, None) == 1
    assert g(FAKE, FAKE, FAKE, FAKE, 4, 128, 256, None, None, 0, None) == 1      # no Y
    assert g(FAKE, FAKE, None, FAKE, 4, 128, 256, FAKE, None, 0, None) == 1      # no rowsum
    assert g(FAKE_ODD, FAKE, FAKE, FAKE, 4, 128, 256, FAKE, None, 0, None) == 3
    assert g(FAKE, FAKE, FAKE_ODD, FAKE, 4, 128, 256, FAKE, None, 0, None) == 3  # rowsum alignment
    assert g(FAKE, FAKE, FAKE, FAKE, 0, 128, 256, FAKE, None, 0, None) == 0      # M == 0: no-op
    ex = L.w4a8_gemm_ex
    bad = w4a8.GemmOpts(0, 48, 0, 0)                                             # block_m not supported
    assert ex(FAKE, FAKE, FAKE, FAKE, 4, 128, 256, FAKE, None, None, 0, ctypes.byref(bad), None) == 1
    bad = w4a8.GemmOpts(4, 0, 0, 0)
    assert ex(FAKE, FAKE, FAKE, FAKE, 4, 128, 256, FAKE, None, None, 0, ctypes.byref(bad), None) == 1
    both = FAKE
    assert ex(FAKE, FAKE, FAKE, FAKE, 4, 128, 256, FAKE, both, None, 0, None, None) == 1  # Y and acc
    assert L.w4a8_gemm_debug_acc(FAKE, FAKE, FAKE, 4, 128, 256, None, None, 0, None) == 1  # no acc
    assert ex(None, None, None, None, 0, 128, 256, None, None, None, 0, None, None) == 0   # M == 0


def test_w4a4_validation(L):
    q = L.w4a4_quantize_act
    assert q(FAKE, 4, 7, FAKE, FAKE, None, None) == 2                # K % 8
    assert q(FAKE, 4, 128, None, FAKE, None, None) == 1              # no output
    assert q(FAKE, 4, 128, FAKE_ODD, FAKE, None, None) == 3          # packed codes alignment
    assert q(FAKE, 0, 128, None, None, None, None) == 0              # M == 0: no-op
    qs = L.w4a4_quantize_act_static
    assert qs(FAKE, 4, 128, None, FAKE, FAKE, None, None) == 1       # no scale
    assert qs(FAKE, 4, 128, FAKE_ODD, FAKE, FAKE, None, None) == 3   # scale alignment
    g = L.w4a4_gemm
    assert g(FAKE, FAKE, FAKE, FAKE, 4, 100, 256, FAKE, None, 0, None) == 2   # N % 128
    assert g(FAKE, FAKE, FAKE, FAKE, 4, 128, 200, FAKE, None, 0, None) == 2   # K % 128
    assert g(FAKE, FAKE, None, FAKE, 4, 128, 256, FAKE, None, 0, None) == 1   # no rowsum
    assert g(FAKE_ODD, FAKE, FAKE, FAKE, 4, 128, 256, FAKE, None, 0, None) == 3
    assert g(FAKE, FAKE, FAKE, FAKE, 0, 128, 256, FAKE, None, 0, None) == 0   # M == 0: no-op
    ex = L.w4a4_gemm_ex
    assert ex(FAKE, FAKE, FAKE, FAKE, 4, 128, 256, FAKE, FAKE, None, 0, None, None) == 1  # Y and acc


def test_python_binding_refuses_cpu_tensors(L):
    torch = pytest.importorskip("torch")
    with pytest.raises(w4a8.W4A8Error):
        w4a8.quantize_act(torch.zeros((2, 128), dtype=torch.float16))


def test_lut_validation(L):
    assert L.w4lut_packed_bytes(256, 512, 128) == 64 + 2 * 4 * 8448 + 64
    assert L.w4lut_packed_bytes(200, 512, 128) == 0
    p = L.w4lut_pack_weights
    nb = L.w4lut_packed_bytes(256, 256, 128)
    assert p(FAKE, FAKE, FAKE, 200, 256, 128, FAKE, nb, None) == 2
    assert p(FAKE, FAKE, None, 256, 256, 128, FAKE, nb, None) == 1       # no table
    assert p(FAKE, FAKE, FAKE, 256, 256, 128, FAKE, nb - 1, None) == 1
    assert p(FAKE_ODD, FAKE, FAKE, 256, 256, 128, FAKE, nb, None) == 3
    g = L.w4lut_gemm
    assert g(FAKE, FAKE, 4, 100, 256, FAKE, None, 0, None) == 2           # N % 128
    assert g(FAKE, FAKE, 4, 128, 200, FAKE, None, 0, None) == 2           # K % 128
    assert g(FAKE, FAKE, 4, 128, 256, None, None, 0, None) == 1           # no Y
    assert g(FAKE_ODD, FAKE, 4, 128, 256, FAKE, None, 0, None) == 3
    assert g(FAKE, FAKE, 0, 128, 256, FAKE, None, 0, None) == 0           # M == 0: no-op
    bad = w4a8.GemmOpts(0, 64, 0, 0)                                       # 64-token tiles: not for this GEMM
    assert L.w4lut_gemm_ex(FAKE, FAKE, 4, 128, 256, FAKE, None, None, 0, ctypes.byref(bad), None) == 1


def test_kv4_validation(L):
    q = L.w4kv_quantize
    assert q(FAKE, 4, 64, FAKE, FAKE, None) == 2                           # D != 128
    assert q(FAKE, -1, 128, FAKE, FAKE, None) == 1
    assert q(None, 4, 128, FAKE, FAKE, None) == 1
    assert q(FAKE_ODD, 4, 128, FAKE, FAKE, None) == 3
    assert q(None, 0, 128, None, None, None) == 0                         # n == 0: no-op
    ws = L.w4kv_attention_workspace_bytes
    assert ws(2, 32, 8, 4096, 128) == 2 * 32 * 32 * 130 * 4               # partials of 128-token chunks
    assert ws(2, 6, 4, 4096, 128) == 0                                    # Hq % Hkv
    assert ws(2, 32, 8, 4096, 64) == 0                                    # D
    a = L.w4kv_attention_decode
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE]
    assert a(*args, 2, 32, 8, 0, 128, 1.0, FAKE, FAKE, 1 << 30, None) == 2   # Lmax == 0
    assert a(*args, 2, 32, 8, 1024, 128, 1.0, FAKE, FAKE, 16, None) == 4     # workspace too small
    assert a(*args, 2, 32, 8, 1024, 128, 1.0, FAKE, None, 1 << 30, None) == 4
    assert a(*args, 2, 32, 8, 1024, 128, 1.0, None, FAKE, 1 << 30, None) == 1
    assert a(FAKE_ODD, *args[1:], 2, 32, 8, 1024, 128, 1.0, FAKE, FAKE, 1 << 30, None) == 3
    assert a(*args, 0, 32, 8, 1024, 128, 1.0, None, None, 0, None) == 0     # B == 0: no-op
    ap = L.w4kv_append
    assert ap(FAKE, FAKE, FAKE, 2, 8, 1024, 64, FAKE, FAKE, FAKE, FAKE, None) == 2
    assert ap(FAKE, FAKE, None, 2, 8, 1024, 128, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert ap(FAKE, FAKE, FAKE, 0, 8, 1024, 128, FAKE, FAKE, FAKE, FAKE, None) == 0


def test_lut3_validation(L):
    assert L.w4lut3_packed_bytes(256, 512, 128) == 64 + 2 * 4 * 6400 + 64
    assert L.w4lut3_packed_bytes(200, 512, 128) == 0
    p = L.w4lut3_pack_weights
    nb = L.w4lut3_packed_bytes(256, 256, 128)
    assert p(FAKE, FAKE, FAKE, 200, 256, 128, FAKE, nb, None) == 2
    assert p(FAKE, FAKE, None, 256, 256, 128, FAKE, nb, None) == 1        # no table
    assert p(FAKE, FAKE, FAKE, 256, 256, 128, FAKE, nb - 1, None) == 1
    assert p(FAKE, FAKE, FAKE, 256, 256, 128, FAKE_ODD, nb, None) == 3    # blob alignment
    g = L.w4lut3_gemm
    assert g(FAKE, FAKE, 4, 100, 256, FAKE, None, 0, None) == 2
    assert g(FAKE, FAKE, 4, 128, 256, None, None, 0, None) == 1
    assert g(FAKE, FAKE, 0, 128, 256, FAKE, None, 0, None) == 0
    bad = w4a8.GemmOpts(0, 64, 0, 0)
    assert L.w4lut3_gemm_ex(FAKE, FAKE, 4, 128, 256, FAKE, None, None, 0, ctypes.byref(bad), None) == 1


def test_chain_validation_on_the_host():
    """w4a8_chain checks its links before touching the device."""
    import ctypes
    L = w4a8.lib()
    Link = w4a8.ChainLink
    buf = ctypes.create_string_buffer(1 << 16)
    base = (ctypes.addressof(buf) + 255) // 256 * 256

    def link(**kw):
        d = dict(A=base, packed=base, M=4, N=256, K=512, A8=base, sA=base, rowsum=base, Y=base)
        d.update(kw)
        return Link(*(d[f] for f, _ in Link._fields_))

    def status(links, ws=base, nbytes=1 << 15):
        arr = (Link * max(len(links), 1))(*links)
        return w4a8.status_string(L.w4a8_chain(arr, len(links), ctypes.c_void_p(ws), nbytes, None))

    assert status([]) == "W4A8_ERR_INVALID_ARG"
    assert status([link()] * 17) == "W4A8_ERR_INVALID_ARG"
    assert status([link(M=33)]) == "W4A8_ERR_UNSUPPORTED_SHAPE"
    assert status([link(M=0)]) == "W4A8_ERR_INVALID_ARG"
    assert status([link(N=200)]) == "W4A8_ERR_UNSUPPORTED_SHAPE"
    assert status([link(K=65536 + 128)]) == "W4A8_ERR_UNSUPPORTED_SHAPE"
    assert status([link(Y=0)]) == "W4A8_ERR_INVALID_ARG"
    assert status([link(A=base + 8)]) == "W4A8_ERR_MISALIGNED"
    assert status([link(rowsum=base + 2)]) == "W4A8_ERR_MISALIGNED"
    assert status([link()], ws=base + 16) == "W4A8_ERR_MISALIGNED"
    arr = (Link * 1)(link(M=40))
    assert L.w4a8_chain_workspace_bytes(arr, 1) == 0
