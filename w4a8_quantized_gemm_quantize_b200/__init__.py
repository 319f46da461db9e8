"""Python binding of the B200 W4A8 quantized GEMM library (libw4a8.so).

Argument marshalling only: every computation runs in the CUDA kernels of
libw4a8.so, called through its C ABI (include/w4a8.h) on the caller's
current torch CUDA stream. There is no CPU or PyTorch fallback: if the
library is missing or the tensors are not on a CUDA device, the calls raise.

    A8, sA, rowsum = quantize_act(A)             # fp16 [M,K] -> int8, fp16, int32
    q, z, s2, s1 = quantize_weights(W)           # fp32 [N,K] -> two-level codes
    blob = pack_weights(q, z, s2, s1)            # offline reordering
    Y = gemm(A8, sA, rowsum, blob, N, K)         # fp16 [M,N]
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "W4A8Error", "lib", "library_path", "EXPORTED_SYMBOLS", "status_string", "quantize_act",
    "quantize_weights", "packed_bytes", "pack_weights", "workspace_bytes", "Workspace", "gemm",
    "gemm_debug_acc", "gemm_ex", "gemm_noalloc", "get_device_error", "clear_device_error",
    "selftest_bounded_wait", "quantize_act_static", "w4a4_quantize_act", "w4a4_quantize_act_static",
    "w4a4_gemm", "w4a4_gemm_ex", "w4a4_workspace_bytes", "lut_packed_bytes", "lut_pack_weights", "lut_gemm",
    "lut_gemm_ex", "lut3_packed_bytes", "lut3_pack_weights", "lut3_gemm", "lut3_gemm_ex", "kv4_quantize", "kv4_append", "kv4_workspace_bytes", "kv4_attention_decode",
    "ChainLink", "chain_links", "chain_workspace_bytes", "chain",
]

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_PKG_DIR, "libw4a8.so")

EXPORTED_SYMBOLS = (
    "w4a8_status_string", "w4a8_version", "w4a8_quantize_act", "w4a8_quantize_weights",
    "w4a8_packed_bytes", "w4a8_pack_weights", "w4a8_gemm_workspace_bytes", "w4a8_gemm",
    "w4a8_gemm_debug_acc", "w4a8_gemm_ex", "w4a8_get_device_error", "w4a8_clear_device_error",
    "w4a8_gemm_noalloc", "w4a8_selftest_bounded_wait", "w4a8_quantize_act_static",
    "w4a4_quantize_act", "w4a4_quantize_act_static", "w4a4_gemm", "w4a4_gemm_ex", "w4a4_gemm_workspace_bytes",
    "w4lut_packed_bytes", "w4lut_pack_weights", "w4lut_gemm", "w4lut_gemm_ex",
    "w4kv_quantize", "w4kv_append", "w4kv_attention_workspace_bytes", "w4kv_attention_decode",
    "w4lut3_packed_bytes", "w4lut3_pack_weights", "w4lut3_gemm", "w4lut3_gemm_ex",
    "w4a8_chain_workspace_bytes", "w4a8_chain",
)

SCHEDULE_AUTO, SCHEDULE_WHOLE_TILES, SCHEDULE_SPLIT_K, SCHEDULE_CLUSTER = 0, 1, 2, 3


class W4A8Error(RuntimeError):
    pass


class GemmOpts(ctypes.Structure):
    _fields_ = [("schedule", ctypes.c_int32), ("block_m", ctypes.c_int32),
                ("max_ctas", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class ChainLink(ctypes.Structure):
    """w4a8_chain_link_t: one GEMM of a chain (device pointers and shape)."""
    _fields_ = [("A", ctypes.c_void_p), ("packed", ctypes.c_void_p), ("M", ctypes.c_int64), ("N", ctypes.c_int64),
                ("K", ctypes.c_int64), ("A8", ctypes.c_void_p), ("sA", ctypes.c_void_p), ("rowsum", ctypes.c_void_p),
                ("Y", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """Loads libw4a8.so (built in-tree by the package's build module)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(library_path):
        raise W4A8Error(
            f"{library_path} is missing: build it with `python -m w4a8_quantized_gemm_quantize_b200.build`")
    L = ctypes.CDLL(library_path)
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
    sig = {
        "w4a8_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "w4a8_version": (ctypes.c_int, []),
        "w4a8_quantize_act": (ctypes.c_int, [vp, i64, i64, vp, vp, vp, vp]),
        "w4a8_quantize_weights": (ctypes.c_int, [vp, i64, i64, i32, vp, vp, vp, vp, vp]),
        "w4a8_packed_bytes": (sz, [i64, i64, i32]),
        "w4a8_pack_weights": (ctypes.c_int, [vp, vp, vp, vp, i64, i64, i32, vp, sz, vp]),
        "w4a8_gemm_workspace_bytes": (sz, [i64, i64, i64]),
        "w4a8_gemm": (ctypes.c_int, [vp, vp, vp, vp, i64, i64, i64, vp, vp, sz, vp]),
        "w4a8_gemm_debug_acc": (ctypes.c_int, [vp, vp, vp, i64, i64, i64, vp, vp, sz, vp]),
        "w4a8_gemm_ex": (ctypes.c_int, [vp, vp, vp, vp, i64, i64, i64, vp, vp, vp, sz,
                                        ctypes.POINTER(GemmOpts), vp]),
        "w4a8_get_device_error": (ctypes.c_int, [vp, ctypes.POINTER(ctypes.c_int32)]),
        "w4a8_clear_device_error": (ctypes.c_int, [vp]),
        "w4a8_gemm_noalloc": (ctypes.c_int, [vp, vp, vp, vp, i64, i64, i64, vp, vp]),
        "w4a8_selftest_bounded_wait": (ctypes.c_int, [i64, vp]),
        "w4a8_quantize_act_static": (ctypes.c_int, [vp, i64, i64, vp, vp, vp, vp, vp]),
        "w4a4_quantize_act": (ctypes.c_int, [vp, i64, i64, vp, vp, vp, vp]),
        "w4a4_quantize_act_static": (ctypes.c_int, [vp, i64, i64, vp, vp, vp, vp, vp]),
        "w4a4_gemm": (ctypes.c_int, [vp, vp, vp, vp, i64, i64, i64, vp, vp, sz, vp]),
        "w4a4_gemm_workspace_bytes": (sz, [i64, i64, i64]),
        "w4lut_packed_bytes": (sz, [i64, i64, i32]),
        "w4lut_pack_weights": (ctypes.c_int, [vp, vp, vp, i64, i64, i32, vp, sz, vp]),
        "w4lut_gemm": (ctypes.c_int, [vp, vp, i64, i64, i64, vp, vp, sz, vp]),
        "w4lut_gemm_ex": (ctypes.c_int, [vp, vp, i64, i64, i64, vp, vp, vp, sz, ctypes.POINTER(GemmOpts), vp]),
        "w4a4_gemm_ex": (ctypes.c_int, [vp, vp, vp, vp, i64, i64, i64, vp, vp, vp, sz,
                                        ctypes.POINTER(GemmOpts), vp]),
        "w4lut3_packed_bytes": (sz, [i64, i64, i32]),
        "w4lut3_pack_weights": (ctypes.c_int, [vp, vp, vp, i64, i64, i32, vp, sz, vp]),
        "w4lut3_gemm": (ctypes.c_int, [vp, vp, i64, i64, i64, vp, vp, sz, vp]),
        "w4lut3_gemm_ex": (ctypes.c_int, [vp, vp, i64, i64, i64, vp, vp, vp, sz, ctypes.POINTER(GemmOpts), vp]),
        "w4kv_quantize": (ctypes.c_int, [vp, i64, i32, vp, vp, vp]),
        "w4kv_append": (ctypes.c_int, [vp, vp, vp, i64, i64, i64, i32, vp, vp, vp, vp, vp]),
        "w4kv_attention_workspace_bytes": (sz, [i64, i64, i64, i64, i32]),
        "w4kv_attention_decode": (ctypes.c_int, [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i32, ctypes.c_float,
                                                 vp, vp, sz, vp]),
        "w4a8_chain_workspace_bytes": (sz, [ctypes.POINTER(ChainLink), i32]),
        "w4a8_chain": (ctypes.c_int, [ctypes.POINTER(ChainLink), i32, vp, sz, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def status_string(code: int) -> str:
    return lib().w4a8_status_string(int(code)).decode()


def _check(code: int, what: str):
    if code != 0:
        raise W4A8Error(f"{what}: {status_string(code)}")


# --------------------------------------------------------------- helpers
def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    torch = _torch()
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _require_cuda(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise W4A8Error("tensors must live on a CUDA device (no CPU path exists)")
            if not t.is_contiguous():
                raise W4A8Error("tensors must be contiguous")


# ------------------------------------------------------------------- API
def quantize_act(A, out=None):
    """fp16 [M, K] -> (A8 int8 [M, K], sA fp16 [M], rowsum int32 [M])."""
    torch = _torch()
    _require_cuda(A)
    if A.dtype != torch.float16 or A.dim() != 2:
        raise W4A8Error("A must be a 2-D fp16 tensor")
    M, K = A.shape
    if out is None:
        A8 = torch.empty((M, K), dtype=torch.int8, device=A.device)
        sA = torch.empty((M,), dtype=torch.float16, device=A.device)
        rowsum = torch.empty((M,), dtype=torch.int32, device=A.device)
    else:
        A8, sA, rowsum = out
        _require_cuda(A8, sA, rowsum)
    _check(lib().w4a8_quantize_act(_ptr(A), M, K, _ptr(A8), _ptr(sA), _ptr(rowsum), _stream(A.device)),
           "w4a8_quantize_act")
    return A8, sA, rowsum


def quantize_act_static(A, s, out=None):
    """Per-tensor static quantization with the fp16 scale `s` (a 1-element
    CUDA tensor): fp16 [M, K] -> (A8 int8 [M, K], sA fp16 [M] = s, rowsum int32 [M])."""
    torch = _torch()
    _require_cuda(A, s)
    if A.dtype != torch.float16 or A.dim() != 2 or s.dtype != torch.float16 or s.numel() != 1:
        raise W4A8Error("A must be a 2-D fp16 tensor and s a 1-element fp16 tensor")
    M, K = A.shape
    if out is None:
        A8 = torch.empty((M, K), dtype=torch.int8, device=A.device)
        sA = torch.empty((M,), dtype=torch.float16, device=A.device)
        rowsum = torch.empty((M,), dtype=torch.int32, device=A.device)
    else:
        A8, sA, rowsum = out
        _require_cuda(A8, sA, rowsum)
    _check(lib().w4a8_quantize_act_static(_ptr(A), M, K, _ptr(s), _ptr(A8), _ptr(sA), _ptr(rowsum),
                                          _stream(A.device)), "w4a8_quantize_act_static")
    return A8, sA, rowsum


def quantize_weights(W, group: int = 128):
    """fp32 [N, K] -> (q uint8 [N,K], z uint8 [N,K/g], s2 uint8 [N,K/g], s1 fp16 [N])."""
    torch = _torch()
    _require_cuda(W)
    if W.dtype != torch.float32 or W.dim() != 2:
        raise W4A8Error("W must be a 2-D fp32 tensor")
    N, K = W.shape
    G = K // group if group > 0 else 0
    q = torch.empty((N, K), dtype=torch.uint8, device=W.device)
    z = torch.empty((N, G), dtype=torch.uint8, device=W.device)
    s2 = torch.empty((N, G), dtype=torch.uint8, device=W.device)
    s1 = torch.empty((N,), dtype=torch.float16, device=W.device)
    _check(lib().w4a8_quantize_weights(_ptr(W), N, K, group, _ptr(q), _ptr(z), _ptr(s2), _ptr(s1),
                                       _stream(W.device)), "w4a8_quantize_weights")
    return q, z, s2, s1


def packed_bytes(N: int, K: int, group: int = 128) -> int:
    return int(lib().w4a8_packed_bytes(N, K, group))


def pack_weights(q, z, s2, s1, group: int = 128):
    """Codes -> packed blob (uint8 tensor of packed_bytes(N, K))."""
    torch = _torch()
    _require_cuda(q, z, s2, s1)
    N, K = q.shape
    nbytes = packed_bytes(N, K, group)
    if nbytes == 0:
        raise W4A8Error(f"unsupported weight shape {N}x{K} (group {group})")
    blob = torch.empty((nbytes,), dtype=torch.uint8, device=q.device)
    _check(lib().w4a8_pack_weights(_ptr(q), _ptr(z), _ptr(s2), _ptr(s1), N, K, group, _ptr(blob), nbytes,
                                   _stream(q.device)), "w4a8_pack_weights")
    return blob


def workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib().w4a8_gemm_workspace_bytes(M, N, K))


class Workspace:
    """A zero-filled GEMM workspace that grows on demand (kept zero by the kernels)."""

    def __init__(self, device=None):
        self.device = device
        self.buf = None

    def get(self, M: int, N: int, K: int):
        torch = _torch()
        need = workspace_bytes(M, N, K)
        if need == 0:
            return None
        if self.buf is None or self.buf.numel() < need:
            self.buf = torch.zeros((need,), dtype=torch.uint8, device=self.device)
        return self.buf


_default_ws = {}


def _workspace_for(device, M, N, K):
    key = str(device)
    ws = _default_ws.get(key)
    if ws is None:
        ws = _default_ws[key] = Workspace(device)
    return ws.get(M, N, K)


def _gemm_common(A8, sA, rowsum, blob, N, K, Y, acc, workspace, opts):
    torch = _torch()
    _require_cuda(A8, sA, rowsum, blob, Y, acc, workspace)
    M = A8.shape[0]
    if A8.dtype != torch.int8 or A8.shape[1] != K:
        raise W4A8Error("A8 must be int8 [M, K]")
    if workspace is None:
        workspace = _workspace_for(A8.device, M, N, K)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    o = None if opts is None else ctypes.byref(GemmOpts(*opts))
    code = lib().w4a8_gemm_ex(_ptr(A8), _ptr(sA), _ptr(rowsum), _ptr(blob), M, N, K, _ptr(Y), _ptr(acc),
                              _ptr(workspace), ws_bytes, o, _stream(A8.device))
    _check(code, "w4a8_gemm_ex")


def gemm(A8, sA, rowsum, blob, N: int, K: int, out=None, workspace=None, opts=None):
    """Y fp16 [M, N] = fp16(sA * s1 * (A8 @ W8^T)); rowsum as from quantize_act."""
    torch = _torch()
    M = A8.shape[0]
    Y = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=A8.device)
    _gemm_common(A8, sA, rowsum, blob, N, K, Y, None, workspace, opts)
    return Y


def gemm_debug_acc(A8, rowsum, blob, N: int, K: int, out=None, workspace=None, opts=None):
    """int32 [M, N] accumulators sum_k A8[m,k] * W8[n,k]."""
    torch = _torch()
    M = A8.shape[0]
    acc = out if out is not None else torch.empty((M, N), dtype=torch.int32, device=A8.device)
    _gemm_common(A8, None, rowsum, blob, N, K, None, acc, workspace, opts)
    return acc


def gemm_ex(A8, sA, rowsum, blob, N: int, K: int, Y=None, acc=None, workspace=None, schedule=0, block_m=0,
            max_ctas=0):
    """GEMM with explicit scheduling overrides (for tests and tuning)."""
    _gemm_common(A8, sA, rowsum, blob, N, K, Y, acc, workspace, (schedule, block_m, max_ctas, 0))
    return Y if Y is not None else acc


# ------------------------------------------------------------------ W4A4
def w4a4_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib().w4a4_gemm_workspace_bytes(M, N, K))


def _w4a4_workspace_for(device, M, N, K):
    """A cached W4A4 workspace shared by all shapes: its zero-filled prefix
    covers the largest w4a8 part seen and its scratch end the largest M * K
    seen, so no shape's scratch (at the buffer's end) reaches another shape's
    zero-filled prefix."""
    torch = _torch()
    if w4a4_workspace_bytes(M, N, K) == 0:
        return None
    key = ("w4a4", str(device))
    buf, base, codes = _default_ws.get(key, (None, 0, 0))
    base2, codes2 = max(base, workspace_bytes(M, N, K)), max(codes, M * K)
    if buf is None or base2 > base or codes2 > codes:
        need = (base2 + 255) // 256 * 256 + codes2 + 256
        buf = torch.zeros((need,), dtype=torch.uint8, device=device)
        _default_ws[key] = (buf, base2, codes2)
    return buf


def _act4_outputs(A, out):
    torch = _torch()
    M, K = A.shape
    if out is None:
        return (torch.empty((M, K // 2), dtype=torch.uint8, device=A.device),
                torch.empty((M,), dtype=torch.float16, device=A.device),
                torch.empty((M,), dtype=torch.int32, device=A.device))
    _require_cuda(*out)
    return out


def w4a4_quantize_act(A, out=None):
    """fp16 [M, K] -> (A4 uint8 [M, K/2] packed 4-bit codes, sA fp16 [M], rowsum int32 [M])."""
    torch = _torch()
    _require_cuda(A)
    if A.dtype != torch.float16 or A.dim() != 2:
        raise W4A8Error("A must be a 2-D fp16 tensor")
    A4, sA, rowsum = _act4_outputs(A, out)
    M, K = A.shape
    _check(lib().w4a4_quantize_act(_ptr(A), M, K, _ptr(A4), _ptr(sA), _ptr(rowsum), _stream(A.device)),
           "w4a4_quantize_act")
    return A4, sA, rowsum


def w4a4_quantize_act_static(A, s, out=None):
    """Per-tensor static 4-bit codes with the fp16 scale `s` (a 1-element CUDA
    tensor): fp16 [M, K] -> (A4 uint8 [M, K/2], sA fp16 [M] = s, rowsum int32 [M])."""
    torch = _torch()
    _require_cuda(A, s)
    if A.dtype != torch.float16 or A.dim() != 2 or s.dtype != torch.float16 or s.numel() != 1:
        raise W4A8Error("A must be a 2-D fp16 tensor and s a 1-element fp16 tensor")
    A4, sA, rowsum = _act4_outputs(A, out)
    M, K = A.shape
    _check(lib().w4a4_quantize_act_static(_ptr(A), M, K, _ptr(s), _ptr(A4), _ptr(sA), _ptr(rowsum),
                                          _stream(A.device)), "w4a4_quantize_act_static")
    return A4, sA, rowsum


def w4a4_gemm_ex(A4, sA, rowsum, blob, N: int, K: int, Y=None, acc=None, workspace=None, schedule=0, block_m=0,
                 max_ctas=0):
    """W4A4 GEMM on packed 4-bit activation codes A4 uint8 [M, K/2]: fp16 Y
    and/or (acc given) the raw int32 accumulators; scheduling overrides as gemm_ex."""
    torch = _torch()
    _require_cuda(A4, sA, rowsum, blob, Y, acc, workspace)
    M = A4.shape[0]
    if A4.dtype != torch.uint8 or A4.dim() != 2 or A4.shape[1] * 2 != K:
        raise W4A8Error("A4 must be uint8 [M, K/2]")
    if workspace is None:
        workspace = _w4a4_workspace_for(A4.device, M, N, K)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    o = ctypes.byref(GemmOpts(schedule, block_m, max_ctas, 0))
    _check(lib().w4a4_gemm_ex(_ptr(A4), _ptr(sA), _ptr(rowsum), _ptr(blob), M, N, K, _ptr(Y), _ptr(acc),
                              _ptr(workspace), ws_bytes, o, _stream(A4.device)), "w4a4_gemm_ex")
    return Y if Y is not None else acc


def w4a4_gemm(A4, sA, rowsum, blob, N: int, K: int, out=None, workspace=None):
    """Y fp16 [M, N] = fp16(sA * s1 * (A4 @ W8^T)) on packed 4-bit activation codes."""
    torch = _torch()
    _require_cuda(A4, sA, rowsum, blob, out, workspace)
    M = A4.shape[0]
    if A4.dtype != torch.uint8 or A4.dim() != 2 or A4.shape[1] * 2 != K:
        raise W4A8Error("A4 must be uint8 [M, K/2]")
    Y = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=A4.device)
    if workspace is None:
        workspace = _w4a4_workspace_for(A4.device, M, N, K)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().w4a4_gemm(_ptr(A4), _ptr(sA), _ptr(rowsum), _ptr(blob), M, N, K, _ptr(Y), _ptr(workspace),
                           ws_bytes, _stream(A4.device)), "w4a4_gemm")
    return Y


# ---------------------------------------------- lookup-table weight-only GEMM
def lut_packed_bytes(N: int, K: int, group: int = 128) -> int:
    return int(lib().w4lut_packed_bytes(N, K, group))


def lut_pack_weights(q, s, table, group: int = 128):
    """Indices q uint8 [N, K], scales s fp16 [N, K/128], table fp16 [16] -> blob."""
    torch = _torch()
    _require_cuda(q, s, table)
    N, K = q.shape
    nbytes = lut_packed_bytes(N, K, group)
    if nbytes == 0:
        raise W4A8Error(f"unsupported weight shape {N}x{K} (group {group})")
    blob = torch.empty((nbytes,), dtype=torch.uint8, device=q.device)
    _check(lib().w4lut_pack_weights(_ptr(q), _ptr(s), _ptr(table), N, K, group, _ptr(blob), nbytes,
                                    _stream(q.device)), "w4lut_pack_weights")
    return blob


def lut_gemm_ex(A, blob, N: int, K: int, Y=None, acc=None, workspace=None, schedule=0, block_m=0, max_ctas=0):
    """Lookup-table GEMM of fp16 A [M, K]: fp16 Y and/or (acc given) the fp32
    sums before rounding; scheduling overrides as gemm_ex (block_m 0/16/32)."""
    torch = _torch()
    _require_cuda(A, blob, Y, acc, workspace)
    if A.dtype != torch.float16 or A.dim() != 2 or A.shape[1] != K:
        raise W4A8Error("A must be fp16 [M, K]")
    M = A.shape[0]
    if workspace is None:
        workspace = _workspace_for(A.device, M, N, K)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    o = ctypes.byref(GemmOpts(schedule, block_m, max_ctas, 0))
    _check(lib().w4lut_gemm_ex(_ptr(A), _ptr(blob), M, N, K, _ptr(Y), _ptr(acc), _ptr(workspace), ws_bytes, o,
                               _stream(A.device)), "w4lut_gemm_ex")
    return Y if Y is not None else acc


def lut_gemm(A, blob, N: int, K: int, out=None, workspace=None):
    """Y fp16 [M, N] = fp16(sum_k A[m,k] * fp16(T[q[n,k]] * s[n,k/128]))."""
    torch = _torch()
    _require_cuda(A, blob, out, workspace)
    if A.dtype != torch.float16 or A.dim() != 2 or A.shape[1] != K:
        raise W4A8Error("A must be fp16 [M, K]")
    M = A.shape[0]
    Y = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=A.device)
    if workspace is None:
        workspace = _workspace_for(A.device, M, N, K)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().w4lut_gemm(_ptr(A), _ptr(blob), M, N, K, _ptr(Y), _ptr(workspace), ws_bytes, _stream(A.device)),
           "w4lut_gemm")
    return Y


def lut3_packed_bytes(N: int, K: int, group: int = 128) -> int:
    return int(lib().w4lut3_packed_bytes(N, K, group))


def lut3_pack_weights(q, s, table, group: int = 128):
    """3-bit indices q uint8 [N, K] (0..7), scales s fp16 [N, K/128], table fp16 [8] -> blob."""
    torch = _torch()
    _require_cuda(q, s, table)
    N, K = q.shape
    nbytes = lut3_packed_bytes(N, K, group)
    if nbytes == 0:
        raise W4A8Error(f"unsupported weight shape {N}x{K} (group {group})")
    blob = torch.empty((nbytes,), dtype=torch.uint8, device=q.device)
    _check(lib().w4lut3_pack_weights(_ptr(q), _ptr(s), _ptr(table), N, K, group, _ptr(blob), nbytes,
                                     _stream(q.device)), "w4lut3_pack_weights")
    return blob


def lut3_gemm_ex(A, blob, N: int, K: int, Y=None, acc=None, workspace=None, schedule=0, block_m=0, max_ctas=0):
    """3-bit lookup-table GEMM (as lut_gemm_ex)."""
    torch = _torch()
    _require_cuda(A, blob, Y, acc, workspace)
    if A.dtype != torch.float16 or A.dim() != 2 or A.shape[1] != K:
        raise W4A8Error("A must be fp16 [M, K]")
    M = A.shape[0]
    if workspace is None:
        workspace = _workspace_for(A.device, M, N, K)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    o = ctypes.byref(GemmOpts(schedule, block_m, max_ctas, 0))
    _check(lib().w4lut3_gemm_ex(_ptr(A), _ptr(blob), M, N, K, _ptr(Y), _ptr(acc), _ptr(workspace), ws_bytes, o,
                                _stream(A.device)), "w4lut3_gemm_ex")
    return Y if Y is not None else acc


def lut3_gemm(A, blob, N: int, K: int, out=None, workspace=None):
    """Y fp16 [M, N] = fp16(sum_k A[m,k] * fp16(T[q[n,k]] * s[n,k/128])), 3-bit q."""
    torch = _torch()
    _require_cuda(A, blob, out, workspace)
    if A.dtype != torch.float16 or A.dim() != 2 or A.shape[1] != K:
        raise W4A8Error("A must be fp16 [M, K]")
    M = A.shape[0]
    Y = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=A.device)
    if workspace is None:
        workspace = _workspace_for(A.device, M, N, K)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().w4lut3_gemm(_ptr(A), _ptr(blob), M, N, K, _ptr(Y), _ptr(workspace), ws_bytes, _stream(A.device)),
           "w4lut3_gemm")
    return Y


NOALLOC_SCRATCH_BYTES = 8 << 20


def gemm_noalloc(A8, sA, rowsum, blob, N: int, K: int, out=None):
    """The GEMM through the allocation-free entry point: the library's own
    built-in scratch array replaces the workspace (see w4a8_gemm_noalloc in
    include/w4a8.h), so no workspace is passed or allocated."""
    torch = _torch()
    _require_cuda(A8, sA, rowsum, blob, out)
    M = A8.shape[0]
    Y = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=A8.device)
    _check(lib().w4a8_gemm_noalloc(_ptr(A8), _ptr(sA), _ptr(rowsum), _ptr(blob), M, N, K, _ptr(Y),
                                   _stream(A8.device)),
           "w4a8_gemm_noalloc")
    return Y


def get_device_error(device=None) -> int:
    code = ctypes.c_int32(0)
    _check(lib().w4a8_get_device_error(_stream(device), ctypes.byref(code)), "w4a8_get_device_error")
    return int(code.value)


def clear_device_error(device=None):
    _check(lib().w4a8_clear_device_error(_stream(device)), "w4a8_clear_device_error")


DEVERR_SELFTEST_WAIT = 6
DEVERR_KV_RANGE = 7
DEVERR_PACK_RANGE = 8
DEVERR_CHAIN_WAIT = 9
DEVERR_BOUNDS = 10


def selftest_bounded_wait(limit_ns: int, device=None):
    """Launches the failure-path self-test (a bounded wait that must give up
    after `limit_ns`); its code shows in get_device_error()."""
    _check(lib().w4a8_selftest_bounded_wait(int(limit_ns), _stream(device)), "w4a8_selftest_bounded_wait")


# ------------------------------------------------------- 4-bit KV cache
KV_HEAD_DIM = 128


def kv4_quantize(X, codes=None, params=None):
    """fp16 vectors X [..., 128] -> (codes uint8 [..., 64], parameter words
    int32 [...] holding the fp16 pair (s, z), s in the low half)."""
    torch = _torch()
    _require_cuda(X, codes, params)
    if X.dtype != torch.float16 or X.shape[-1] != KV_HEAD_DIM or not X.is_contiguous():
        raise W4A8Error("X must be contiguous fp16 [..., 128]")
    lead = tuple(X.shape[:-1])
    n = X.numel() // KV_HEAD_DIM
    codes = codes if codes is not None else torch.empty(lead + (KV_HEAD_DIM // 2,), dtype=torch.uint8,
                                                        device=X.device)
    params = params if params is not None else torch.empty(lead, dtype=torch.int32, device=X.device)
    _check(lib().w4kv_quantize(_ptr(X), n, KV_HEAD_DIM, _ptr(codes), _ptr(params), _stream(X.device)),
           "w4kv_quantize")
    return codes, params


def kv4_append(K_new, V_new, positions, k_codes, k_params, v_codes, v_params):
    """Quantizes one token per (sequence, kv head), K_new and V_new fp16
    [B, Hkv, 128], into the caches (codes [B, Hkv, Lmax, 64], parameter
    words [B, Hkv, Lmax]) at positions int32 [B]."""
    _require_cuda(K_new, V_new, positions, k_codes, k_params, v_codes, v_params)
    B, Hkv, D = K_new.shape
    Lmax = k_codes.shape[2]
    _check(lib().w4kv_append(_ptr(K_new), _ptr(V_new), _ptr(positions), B, Hkv, Lmax, D, _ptr(k_codes),
                             _ptr(k_params), _ptr(v_codes), _ptr(v_params), _stream(K_new.device)), "w4kv_append")


def kv4_workspace_bytes(B: int, Hq: int, Hkv: int, Lmax: int) -> int:
    return int(lib().w4kv_attention_workspace_bytes(B, Hq, Hkv, Lmax, KV_HEAD_DIM))


_kv_ws = {}


def _kv_workspace_for(device, nbytes: int):
    """A workspace per device for the chunks' partial results, grown on
    demand and reused (any contents will do)."""
    torch = _torch()
    key = str(device)
    ws = _kv_ws.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = _kv_ws[key] = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)
    return ws


def kv4_attention_decode(q, k_codes, k_params, v_codes, v_params, seq_lens, scale, out=None, workspace=None):
    """Y fp16 [B, Hq, 128] = decode attention of q fp16 [B, Hq, 128] over the
    4-bit caches with lengths seq_lens int32 [B]; workspace: zero-filled
    uint8 (a per-device one is kept here if none is given; calls on one
    device that share it must not overlap on the GPU)."""
    torch = _torch()
    _require_cuda(q, k_codes, k_params, v_codes, v_params, seq_lens, out, workspace)
    if q.dtype != torch.float16 or q.dim() != 3 or q.shape[2] != KV_HEAD_DIM:
        raise W4A8Error("q must be fp16 [B, Hq, 128]")
    B, Hq, D = q.shape
    Hkv, Lmax = k_codes.shape[1], k_codes.shape[2]
    Y = out if out is not None else torch.empty((B, Hq, D), dtype=torch.float16, device=q.device)
    if workspace is None:
        workspace = _kv_workspace_for(q.device, kv4_workspace_bytes(B, Hq, Hkv, Lmax))
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().w4kv_attention_decode(_ptr(q), _ptr(k_codes), _ptr(k_params), _ptr(v_codes), _ptr(v_params),
                                       _ptr(seq_lens), B, Hq, Hkv, Lmax, D, float(scale), _ptr(Y), _ptr(workspace),
                                       ws_bytes, _stream(q.device)), "w4kv_attention_decode")
    return Y


# ------------------------------------------------------------- GEMM chain
def chain_links(links):
    """ctypes array of w4a8_chain_link_t from dicts with the tensors A (fp16
    [M, K]), blob, N, K, Y (fp16 [M, N]) and A8 / sA / rowsum (int8 [M, K],
    fp16 [M], int32 [M]: where the link's quantized activations go)."""
    torch = _torch()
    arr = (ChainLink * len(links))()
    for i, d in enumerate(links):
        A, Y = d["A"], d["Y"]
        _require_cuda(A, d["blob"], Y, d["A8"], d["sA"], d["rowsum"])
        if A.dtype != torch.float16 or A.dim() != 2 or A.shape[1] != d["K"]:
            raise W4A8Error("A must be fp16 [M, K]")
        if Y.dtype != torch.float16 or tuple(Y.shape) != (A.shape[0], d["N"]):
            raise W4A8Error("Y must be fp16 [M, N]")
        arr[i] = ChainLink(_ptr(A), _ptr(d["blob"]), A.shape[0], d["N"], d["K"], _ptr(d["A8"]), _ptr(d["sA"]),
                           _ptr(d["rowsum"]), _ptr(Y))
    return arr


def chain_workspace_bytes(links) -> int:
    arr = links if isinstance(links, ctypes.Array) else chain_links(links)
    return int(lib().w4a8_chain_workspace_bytes(arr, len(arr)))


def chain(links, workspace):
    """Runs the links in order in one launch (w4a8_chain): link j quantizes
    its A after link j - 1's Y is complete, then computes its Y. `workspace`
    is a zero-filled uint8 CUDA tensor of at least chain_workspace_bytes."""
    arr = links if isinstance(links, ctypes.Array) else chain_links(links)
    _require_cuda(workspace)
    ws_bytes = workspace.numel() * workspace.element_size()
    dev = workspace.device
    _check(lib().w4a8_chain(arr, len(arr), _ptr(workspace), ws_bytes, _stream(dev)), "w4a8_chain")
