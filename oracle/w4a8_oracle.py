"""CPU oracle for the W4A8 quantized GEMM — TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import this module. The product (the CUDA library and its Python binding)
never calls it, and it shares no code with the product.

It is a plain, slow, obviously-correct restatement of what the path
computes, with numpy. Every step is the definition itself; nothing is
blocked, fused or reordered.

What the pages fix and what this file reads into them
-----------------------------------------------------
* W4A8: 4-bit weights against 8-bit activations, with a *progressive*
  (two-level) weight quantization chosen so that dequantizing a weight inside
  the GEMM is cheap ("QServe/QoQ" abstract quoted in lmdeploy issue
  "[Feature] Support W4A8KV4 Quantization(QServe/QoQ)", Motivation).
  The two levels used here: a per-output-channel fp16 scale s1 (level 1) and,
  per group of 128 inputs, a uint4 zero z and an integer scale s2 in [1, 8]
  (level 2), so that the level-2 dequantized weight W8 = (q - z) * s2 is an
  exact int8 in [-120, 120] and the GEMM runs on int8 tensor cores.
* Dequantization must not overflow the 8-bit lanes it is computed in
  ("LiquidGEMM: Hardware-Efficient W4A8 GEMM Kernel ...", Method: LiquidQuant
  dequantizes four elements with two arithmetic operations and no overflow).
  The oracle dequantizes element by element; the bytewise form is pinned in
  the tests.
* Activations: 8-bit, per-token symmetric with a dynamic scale (the dynamic
  per-token baseline that "PrefixQuant: Static Quantization Beats Dynamic
  through Prefixed Outliers in LLMs" compares against, Key Findings).
* 4-bit activations (W4A4): the W4A4KV4 models of "PrefixQuant ..." (Key
  Findings) with per-tensor static scales; readings of the 4-bit code range,
  rounding and nibble order are stated at `quantize_act4`.
* Lookup-table weight-only GEMM ("Fast Matrix Multiplications for Lookup
  Table-Quantized LLMs", FLUTE, abstract): readings at `lut_dequant` and
  the section heading there.
* Offline weight reordering ("QServe/QoQ" abstract: compute-aware weight
  reordering; "QUICK: Quantization-aware Interleaving and Conflict-free
  Kernel ...", abstract: offline interleaving; "Fast Matrix Multiplications
  for Lookup Table-Quantized LLMs", abstract: offline restructuring). The
  packed byte layout below is this library's own; the oracle writes it from
  its definition so the CUDA packer can be checked byte for byte.

Readings where the pages are silent (each is listed in the design notes):
activation codes are rint (half to even) of A / float(sA) with an IEEE fp32
divide, where sA = fp16(amax / 127) is the *stored* scale, clamped to
[-127, 127]; amax == 0 gives sA = 0 and zero codes; the epilogue is
fp16_rn(float(acc) * (float(sA) * float(s1))) in fp32; the weight quantizer's
s1 / s2 / z selection rule is this file's `quantize_weights`.
"""
from __future__ import annotations

import numpy as np

GROUP = 128
TILE_N = 128
TILE_K = 128
TILE_CODE_BYTES = TILE_N * TILE_K // 2  # 8192
TILE_META_BYTES = TILE_N  # 128
TILE_BYTES = TILE_CODE_BYTES + TILE_META_BYTES  # 8320
HEADER_BYTES = 64
MAGIC = 0x38413457  # b"W4A8" little-endian
LAYOUT_VERSION = 1


# ---------------------------------------------------------------------------
# Activation quantization (per token, symmetric int8)
# ---------------------------------------------------------------------------
def quantize_act(A: np.ndarray):
    """Per-token symmetric int8 quantization of fp16 activations.

    For each row m:  amax = max_k |A[m,k]|;  sA = fp16_rn(amax / 127) with an
    fp32 divide;  A8 = clamp(rint(A / float(sA)), -127, 127) with an fp32
    divide (rint: half to even); sA == 0 gives all-zero codes.
    rowsum[m] = sum_k A8[m,k] (int32).

    Returns (A8 int8 [M,K], sA fp16 [M], rowsum int32 [M]).
    """
    assert A.dtype == np.float16 and A.ndim == 2
    Af = A.astype(np.float32)
    amax = np.max(np.abs(Af), axis=1) if A.shape[1] else np.zeros(A.shape[0], np.float32)
    s = amax / np.float32(127.0)
    sA = s.astype(np.float16)
    sf = sA.astype(np.float32)
    A8 = np.zeros(A.shape, dtype=np.int8)
    nz = sf != 0
    if np.any(nz):
        quot = Af[nz] / sf[nz][:, None]
        A8[nz] = np.clip(np.rint(quot), -127, 127).astype(np.int8)
    rowsum = A8.astype(np.int64).sum(axis=1).astype(np.int32)
    return A8, sA, rowsum


def quantize_act_static(A: np.ndarray, s: np.float16):
    """Per-tensor static symmetric int8 quantization of fp16 activations.

    One fp16 scale s for the whole tensor, fixed offline by calibration
    instead of measured per token at run time ("PrefixQuant: Static
    Quantization Beats Dynamic through Prefixed Outliers in LLMs",
    Methodology and Key Findings: per-tensor static quantization once the
    outlier tokens are prefixed). Rounding and range as quantize_act:
    A8 = clamp(rint(A / float(s)), -127, 127) with an fp32 divide (rint: half
    to even); s == 0 gives all-zero codes. sA[m] = s for every token, so the
    GEMM's per-token epilogue applies the tensor scale unchanged;
    rowsum[m] = sum_k A8[m,k] (int32).

    Returns (A8 int8 [M,K], sA fp16 [M], rowsum int32 [M]).
    """
    assert A.dtype == np.float16 and A.ndim == 2
    sf = np.float32(np.float16(s))
    A8 = np.zeros(A.shape, dtype=np.int8)
    if sf != 0:
        A8 = np.clip(np.rint(A.astype(np.float32) / sf), -127, 127).astype(np.int8)
    sA = np.full(A.shape[0], np.float16(s), dtype=np.float16)
    rowsum = A8.astype(np.int64).sum(axis=1).astype(np.int32)
    return A8, sA, rowsum


# ---------------------------------------------------------------------------
# 4-bit activations (W4A4)
# ---------------------------------------------------------------------------
# "PrefixQuant: Static Quantization Beats Dynamic through Prefixed Outliers
# in LLMs" (Key Findings) runs W4A4KV4 models: 4-bit weights against 4-bit
# activations, with per-tensor static activation scales once the outlier
# tokens are prefixed. The pages fix no code range, rounding or storage for
# the 4-bit activations; the readings here are the 8-bit scheme's with the
# symmetric 4-bit range: codes in [-7, 7] (-8 never occurs), rint half to even
# of A / float(s) with an fp32 divide, per-tensor static s (the pages'
# scheme) or a per-token dynamic s = fp16_rn(amax / 7); two codes per byte,
# code k = 2j in the low nibble and k = 2j + 1 in the high nibble of byte j of
# the row, each as a 4-bit two's complement value.
A4_MAX = 7


def quantize_act4(A: np.ndarray):
    """Per-token symmetric 4-bit quantization of fp16 activations.

    For each row m: amax = max_k |A[m,k]|; sA = fp16_rn(amax / 7) with an fp32
    divide; A4 = clamp(rint(A / float(sA)), -7, 7) with an fp32 divide (rint:
    half to even); sA == 0 gives all-zero codes; rowsum[m] = sum_k A4[m,k].

    Returns (A4 int8 [M,K] with values in [-7, 7], sA fp16 [M], rowsum int32 [M]).
    """
    assert A.dtype == np.float16 and A.ndim == 2
    Af = A.astype(np.float32)
    amax = np.max(np.abs(Af), axis=1) if A.shape[1] else np.zeros(A.shape[0], np.float32)
    sA = (amax / np.float32(A4_MAX)).astype(np.float16)
    sf = sA.astype(np.float32)
    A4 = np.zeros(A.shape, dtype=np.int8)
    nz = sf != 0
    if np.any(nz):
        A4[nz] = np.clip(np.rint(Af[nz] / sf[nz][:, None]), -A4_MAX, A4_MAX).astype(np.int8)
    rowsum = A4.astype(np.int64).sum(axis=1).astype(np.int32)
    return A4, sA, rowsum


def quantize_act4_static(A: np.ndarray, s: np.float16):
    """Per-tensor static symmetric 4-bit quantization (the PrefixQuant scheme):
    A4 = clamp(rint(A / float(s)), -7, 7) with an fp32 divide (rint: half to
    even); s == 0 gives all-zero codes; sA[m] = s; rowsum[m] = sum_k A4[m,k].

    Returns (A4 int8 [M,K], sA fp16 [M], rowsum int32 [M]).
    """
    assert A.dtype == np.float16 and A.ndim == 2
    sf = np.float32(np.float16(s))
    A4 = np.zeros(A.shape, dtype=np.int8)
    if sf != 0:
        A4 = np.clip(np.rint(A.astype(np.float32) / sf), -A4_MAX, A4_MAX).astype(np.int8)
    sA = np.full(A.shape[0], np.float16(s), dtype=np.float16)
    rowsum = A4.astype(np.int64).sum(axis=1).astype(np.int32)
    return A4, sA, rowsum


def pack_act4(A4: np.ndarray) -> np.ndarray:
    """[M, K] codes in [-8, 7] -> [M, K/2] bytes: byte j of a row holds code
    2j in bits 0-3 and code 2j+1 in bits 4-7 (4-bit two's complement)."""
    assert A4.ndim == 2 and A4.shape[1] % 2 == 0
    nib = (A4.astype(np.int16) & 0xF).astype(np.uint8)
    return (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)


def unpack_act4(P: np.ndarray) -> np.ndarray:
    """Inverse of `pack_act4`: [M, K/2] bytes -> [M, K] int8 codes."""
    assert P.dtype == np.uint8 and P.ndim == 2
    lo = (P & 0xF).astype(np.int16)
    hi = (P >> 4).astype(np.int16)
    out = np.empty((P.shape[0], 2 * P.shape[1]), dtype=np.int16)
    out[:, 0::2] = np.where(lo >= 8, lo - 16, lo)
    out[:, 1::2] = np.where(hi >= 8, hi - 16, hi)
    return out.astype(np.int8)


# ---------------------------------------------------------------------------
# Progressive (two-level) weight quantization
# ---------------------------------------------------------------------------
def quantize_weights(W: np.ndarray, group: int = GROUP):
    """Two-level quantization of fp32 weights W [N, K].

    Level 1, per output channel n: the range of group g is
    r_g = max(max W_g, 0) - min(min W_g, 0); s1[n] = fp16_rn(max_g r_g / 120)
    (fp32 divide); a zero s1 is replaced by 1.  t = W / float(s1) (fp32).
    Level 2, per (n, group): lo = min(min t, 0), hi = max(max t, 0);
    s2 = clamp(ceil((hi - lo) / 15), 1, 8); z = clamp(rint(-lo / s2), 0, 15);
    q = clamp(rint(t / s2) + z, 0, 15).  All divides are fp32.

    Returns (q uint8 [N,K], z uint8 [N,G], s2 uint8 [N,G], s1 fp16 [N]).
    """
    assert W.dtype == np.float32 and W.ndim == 2
    N, K = W.shape
    assert K % group == 0
    G = K // group
    Wg = W.reshape(N, G, group)
    r = np.maximum(Wg.max(axis=2), np.float32(0)) - np.minimum(Wg.min(axis=2), np.float32(0))
    R = r.max(axis=1)
    s1 = (R / np.float32(120.0)).astype(np.float16)
    s1[s1 == 0] = np.float16(1.0)
    t = Wg / s1.astype(np.float32)[:, None, None]
    lo = np.minimum(t.min(axis=2), np.float32(0))
    hi = np.maximum(t.max(axis=2), np.float32(0))
    s2 = np.clip(np.ceil((hi - lo) / np.float32(15.0)), 1, 8).astype(np.int32)
    s2f = s2.astype(np.float32)
    z = np.clip(np.rint(-lo / s2f), 0, 15).astype(np.int32)
    q = np.clip(np.rint(t / s2f[:, :, None]) + z[:, :, None], 0, 15).astype(np.uint8)
    return q.reshape(N, K), z.astype(np.uint8), s2.astype(np.uint8), s1


def dequant_weights(q: np.ndarray, z: np.ndarray, s2: np.ndarray, group: int = GROUP) -> np.ndarray:
    """Level-2 dequantization: W8[n,k] = (q[n,k] - z[n,k//g]) * s2[n,k//g], exact int8."""
    N, K = q.shape
    zk = np.repeat(z.astype(np.int32), group, axis=1)
    sk = np.repeat(s2.astype(np.int32), group, axis=1)
    w8 = (q.astype(np.int32) - zk) * sk
    return w8.astype(np.int8)


# ---------------------------------------------------------------------------
# Packed weight blob (offline reordering)
# ---------------------------------------------------------------------------
def packed_bytes(N: int, K: int, group: int = GROUP) -> int:
    """Header + (N/128)*(K/128) tiles of 8320 bytes + s1 padded to 16 bytes."""
    tiles = (N // TILE_N) * (K // TILE_K)
    s1_bytes = (2 * N + 15) // 16 * 16
    return HEADER_BYTES + tiles * TILE_BYTES + s1_bytes


def code_byte_offset(r: int, kk: int):
    """Byte offset inside a tile's code area of row r, in-tile k index kk,
    and whether the code is the high nibble.

    Row r's codes for k = 8j .. 8j+7 form 32-bit word j (j = 0..15): byte b
    holds k = 8j+b in its low nibble and k = 8j+4+b in its high nibble.
    Word j of row r sits at word index ((j // 4) * 128 + r) * 4 + j % 4, so
    the four words j = 4c .. 4c+3 (k = 32c .. 32c+31) of a row are one
    16-byte vector and 32 consecutive rows read 512 contiguous bytes.
    """
    j, within = divmod(kk, 8)
    high = within >= 4
    b = within - 4 if high else within
    word = ((j // 4) * TILE_N + r) * 4 + (j % 4)
    return word * 4 + b, high


def pack_weights(q, z, s2, s1, group: int = GROUP) -> np.ndarray:
    """Writes the packed blob element by element from the layout definition.

    Header (64 bytes, little-endian): u32 magic 'W4A8', u32 version 1,
    i64 N, i64 K, i32 group, u32 tile bytes (8320), u64 byte offset of s1;
    the rest zero.  Tile (nt, kt) starts at 64 + (nt*(K/128) + kt)*8320: 8192
    code bytes (see `code_byte_offset`), then 128 meta bytes, row r's being
    z | ((s2 - 1) << 4) of group kt.  After the tiles: s1 as N fp16 values,
    zero padded to a multiple of 16 bytes.
    """
    assert group == GROUP
    N, K = q.shape
    assert N % TILE_N == 0 and K % TILE_K == 0
    KT = K // TILE_K
    out = np.zeros(packed_bytes(N, K, group), dtype=np.uint8)
    s1_off = HEADER_BYTES + (N // TILE_N) * KT * TILE_BYTES
    hdr = bytearray(HEADER_BYTES)
    hdr[0:4] = MAGIC.to_bytes(4, "little")
    hdr[4:8] = LAYOUT_VERSION.to_bytes(4, "little")
    hdr[8:16] = int(N).to_bytes(8, "little", signed=True)
    hdr[16:24] = int(K).to_bytes(8, "little", signed=True)
    hdr[24:28] = int(group).to_bytes(4, "little", signed=True)
    hdr[28:32] = TILE_BYTES.to_bytes(4, "little")
    hdr[32:40] = int(s1_off).to_bytes(8, "little")
    out[:HEADER_BYTES] = np.frombuffer(bytes(hdr), dtype=np.uint8)
    # code bytes: byte b of word j of row r in tile (nt, kt) holds
    # k = 8j+b (low nibble) and k = 8j+4+b (high nibble)
    n = np.arange(N)[:, None, None, None]
    kt = np.arange(KT)[None, :, None, None]
    j = np.arange(16)[None, None, :, None]
    b = np.arange(4)[None, None, None, :]
    r = n % TILE_N
    k_lo = kt * TILE_K + 8 * j + b
    k_hi = k_lo + 4
    byte = (q[n, k_lo].astype(np.uint16) | (q[n, k_hi].astype(np.uint16) << 4)).astype(np.uint8)
    word = ((j // 4) * TILE_N + r) * 4 + (j % 4)
    dest = HEADER_BYTES + ((n // TILE_N) * KT + kt) * TILE_BYTES + word * 4 + b
    out[dest.ravel()] = byte.ravel()
    n = np.arange(N)[:, None]
    # meta bytes
    g = np.arange(K // group)[None, :]
    meta = (z.astype(np.uint16) | ((s2.astype(np.uint16) - 1) << 4)).astype(np.uint8)
    mdest = HEADER_BYTES + (n // TILE_N * KT + g) * TILE_BYTES + TILE_CODE_BYTES + n % TILE_N
    out[mdest.ravel()] = meta.ravel()
    out[s1_off:s1_off + 2 * N] = np.frombuffer(s1.astype(np.float16).tobytes(), dtype=np.uint8)
    return out


def unpack_weights(blob: np.ndarray):
    """Inverse of `pack_weights`: returns (q, z, s2, s1, N, K)."""
    hdr = bytes(blob[:HEADER_BYTES])
    assert int.from_bytes(hdr[0:4], "little") == MAGIC
    N = int.from_bytes(hdr[8:16], "little", signed=True)
    K = int.from_bytes(hdr[16:24], "little", signed=True)
    group = int.from_bytes(hdr[24:28], "little", signed=True)
    s1_off = int.from_bytes(hdr[32:40], "little")
    KT = K // TILE_K
    q = np.zeros((N, K), dtype=np.uint8)
    z = np.zeros((N, K // group), dtype=np.uint8)
    s2 = np.zeros((N, K // group), dtype=np.uint8)
    n = np.arange(N)[:, None]
    k = np.arange(K)[None, :]
    nt, r = n // TILE_N, n % TILE_N
    kt, kk = k // TILE_K, k % TILE_K
    j, within = kk // 8, kk % 8
    high = within >= 4
    b = np.where(high, within - 4, within)
    word = ((j // 4) * TILE_N + r) * 4 + (j % 4)
    src = HEADER_BYTES + (nt * KT + kt) * TILE_BYTES + word * 4 + b
    byte = blob[src]
    q[:] = np.where(high, byte >> 4, byte & 0x0F)
    g = np.arange(K // group)[None, :]
    msrc = HEADER_BYTES + (nt * KT + g) * TILE_BYTES + TILE_CODE_BYTES + r
    meta = blob[msrc]
    z[:] = meta & 0x0F
    s2[:] = (meta >> 4) + 1
    s1 = np.frombuffer(bytes(blob[s1_off:s1_off + 2 * N]), dtype=np.float16).copy()
    return q, z, s2, s1, N, K


# ---------------------------------------------------------------------------
# GEMM
# ---------------------------------------------------------------------------
def gemm_acc(A8: np.ndarray, W8: np.ndarray) -> np.ndarray:
    """acc[m,n] = sum_k A8[m,k] * W8[n,k] (int32).

    Computed as an fp64 matmul of the integer values, which is exact here:
    every product and partial sum is an integer of magnitude below
    127 * 120 * K < 2**53.
    """
    assert A8.dtype == np.int8 and W8.dtype == np.int8
    assert A8.shape[1] == W8.shape[1]
    assert 127 * 120 * A8.shape[1] < 2 ** 31
    acc = A8.astype(np.float64) @ W8.astype(np.float64).T
    return acc.astype(np.int64).astype(np.int32)


def epilogue(acc: np.ndarray, sA: np.ndarray, s1: np.ndarray) -> np.ndarray:
    """Y[m,n] = fp16_rn(float(acc[m,n]) * (float(sA[m]) * float(s1[n]))), fp32."""
    scale = sA.astype(np.float32)[:, None] * s1.astype(np.float32)[None, :]
    with np.errstate(over="ignore"):
        return (acc.astype(np.float32) * scale).astype(np.float16)


def w4a8_gemm(A8, sA, q, z, s2, s1, group: int = GROUP) -> np.ndarray:
    """Y = fp16(sA[m] * s1[n] * sum_k A8[m,k] * (q[n,k] - z) * s2)."""
    return epilogue(gemm_acc(A8, dequant_weights(q, z, s2, group)), sA, s1)


def w4a8_gemm_packed(A8, sA, blob) -> np.ndarray:
    q, z, s2, s1, N, K = unpack_weights(blob)
    return w4a8_gemm(A8, sA, q, z, s2, s1)


def w4a4_gemm(A4_packed, sA, q, z, s2, s1, group: int = GROUP) -> np.ndarray:
    """W4A4: Y = fp16(sA[m] * s1[n] * sum_k A4[m,k] * (q[n,k] - z) * s2) with the
    4-bit activation codes A4 = unpack_act4(A4_packed); the same int32 sum and
    fp32 epilogue as the 8-bit GEMM."""
    return epilogue(gemm_acc(unpack_act4(A4_packed), dequant_weights(q, z, s2, group)), sA, s1)


# ---------------------------------------------------------------------------
# Lookup-table weight-only GEMM (FLUTE)
# ---------------------------------------------------------------------------
# "Fast Matrix Multiplications for Lookup Table-Quantized LLMs" (FLUTE,
# abstract): weight-only quantization in which every weight is an index into
# a non-uniform table (NormalFloat being the example), with a scale per group
# of 128 inputs; the activations stay in 16-bit floating point, and the GEMM
# fuses the table lookup with the matrix multiplication. The pages fix no
# arithmetic; the readings here: 4-bit indices q into a 16-entry fp16 table
# T, one fp16 scale s per (output channel, group of 128 inputs), the weight
# W[n,k] = fp16_rn(float(T[q[n,k]]) * float(s[n, k // 128])) (the exact
# product rounded once), fp16 activations A, and
#   Y[m,n] = fp16_rn(sum_k A[m,k] * W[n,k]),
# the sum exact here (fp64 of exact fp16 x fp16 products); the GPU sums in
# fp32 in an unspecified order, within `lut_error_bound` of it.
LUT_MAGIC = 0x544C3457  # b"W4LT" little-endian
LUT_TILE_SCALE_BYTES = 2 * TILE_N  # 256
LUT_TILE_BYTES = TILE_CODE_BYTES + LUT_TILE_SCALE_BYTES  # 8448


def lut_dequant(q: np.ndarray, s: np.ndarray, T: np.ndarray, group: int = GROUP) -> np.ndarray:
    """W[n,k] = fp16_rn(float(T[q[n,k]]) * float(s[n, k // group])): fp16 [N, K].
    (The product of two fp16 values is exact in fp32, so this is one rounding.)"""
    Tv = T.astype(np.float32)[q]
    sk = np.repeat(s.astype(np.float32), group, axis=1)
    return (Tv * sk).astype(np.float16)


def lut_gemm_exact(A: np.ndarray, q, s, T, group: int = GROUP) -> np.ndarray:
    """sum_k A[m,k] * W[n,k] in fp64 (exact products; fp64 sums, relative error
    below K * 2**-53), [M, N] float64."""
    W = lut_dequant(q, s, T, group)
    return A.astype(np.float64) @ W.astype(np.float64).T


def lut_gemm(A: np.ndarray, q, s, T, group: int = GROUP) -> np.ndarray:
    """Y = fp16_rn(sum_k A[m,k] * W[n,k]) with the sum exact (fp64)."""
    with np.errstate(over="ignore"):
        return lut_gemm_exact(A, q, s, T, group).astype(np.float16)


def lut_error_bound(A: np.ndarray, W: np.ndarray) -> np.ndarray:
    """Bound on |fp32-accumulated sum - exact sum| for sum_k A[m,k] W[n,k]:
    gamma_K * sum_k |A W|, gamma_K = K u / (1 - K u), with u = 2**-23 (one
    fp32 ulp per addition, which also covers additions that truncate rather
    than round). The products themselves are exact in fp32."""
    K = A.shape[1]
    u = 2.0 ** -23
    gamma = K * u / (1 - K * u)
    return gamma * (np.abs(A.astype(np.float64)) @ np.abs(W.astype(np.float64)).T)


def lut_quantize_weights(W: np.ndarray, T: np.ndarray, group: int = GROUP):
    """Offline lookup-table quantization of fp32 W [N, K] with table T:
    s[n,g] = fp16_rn(max |W_g| / max |T|) (fp32 divide; 0 -> 1), and q[n,k] the
    index of the table entry nearest to W[n,k] / float(s) (fp32 divide; ties
    to the lower index). Returns (q uint8 [N,K], s fp16 [N, K/group])."""
    N, K = W.shape
    G = K // group
    Wg = W.reshape(N, G, group)
    tmax = np.float32(np.max(np.abs(T.astype(np.float32))))
    s = (np.max(np.abs(Wg), axis=2) / tmax).astype(np.float16)
    s[s == 0] = np.float16(1.0)
    t = Wg / s.astype(np.float32)[:, :, None]
    dist = np.abs(t[..., None] - T.astype(np.float32)[None, None, None, :])
    q = np.argmin(dist, axis=3).astype(np.uint8)  # argmin takes the first (lowest) index on ties
    return q.reshape(N, K), s


def lut_packed_bytes(N: int, K: int, group: int = GROUP) -> int:
    """Header + (N/128)*(K/128) tiles of 8448 bytes + the table (16 fp16) padded to 64 bytes."""
    return HEADER_BYTES + (N // TILE_N) * (K // TILE_K) * LUT_TILE_BYTES + 64


def lut_code_byte_offset(r: int, kk: int):
    """Byte offset inside a tile's code area of row r, in-tile k index kk, and
    whether the index is the high nibble. Row r's indices for in-tile
    k = 2j, 2j+1 share byte j of the row (k = 2j in bits 0-3); the row's 64
    bytes are four 16-byte vectors, vector c at ((c * 128) + r) * 16, so 32
    consecutive rows read 512 contiguous bytes."""
    j, high = divmod(kk, 2)
    c, b = divmod(j, 16)
    return (c * TILE_N + r) * 16 + b, bool(high)


def lut_pack_weights(q, s, T, group: int = GROUP) -> np.ndarray:
    """Writes the lookup-table weight blob from its definition.

    Header (64 bytes, little-endian): u32 magic 'W4LT', u32 version 1,
    i64 N, i64 K, i32 group, u32 tile bytes (8448), u64 byte offset of the
    table; the rest zero. Tile (nt, kt) starts at 64 + (nt*(K/128) + kt)*8448:
    8192 index bytes (see `lut_code_byte_offset`), then the 128 rows' fp16
    scales of group kt (256 bytes, row r at 8192 + 2r). After the tiles: the
    16 fp16 table entries, zero padded to 64 bytes."""
    assert group == GROUP
    N, K = q.shape
    KT = K // TILE_K
    out = np.zeros(lut_packed_bytes(N, K, group), dtype=np.uint8)
    t_off = HEADER_BYTES + (N // TILE_N) * KT * LUT_TILE_BYTES
    hdr = bytearray(HEADER_BYTES)
    hdr[0:4] = LUT_MAGIC.to_bytes(4, "little")
    hdr[4:8] = (1).to_bytes(4, "little")
    hdr[8:16] = int(N).to_bytes(8, "little", signed=True)
    hdr[16:24] = int(K).to_bytes(8, "little", signed=True)
    hdr[24:28] = int(group).to_bytes(4, "little", signed=True)
    hdr[28:32] = LUT_TILE_BYTES.to_bytes(4, "little")
    hdr[32:40] = int(t_off).to_bytes(8, "little")
    out[:HEADER_BYTES] = np.frombuffer(bytes(hdr), dtype=np.uint8)
    n = np.arange(N)[:, None, None]
    kt = np.arange(KT)[None, :, None]
    j = np.arange(64)[None, None, :]
    r = n % TILE_N
    k_lo = kt * TILE_K + 2 * j
    byte = (q[n, k_lo].astype(np.uint16) | (q[n, k_lo + 1].astype(np.uint16) << 4)).astype(np.uint8)
    c, b = j // 16, j % 16
    dest = HEADER_BYTES + ((n // TILE_N) * KT + kt) * LUT_TILE_BYTES + (c * TILE_N + r) * 16 + b
    out[dest.ravel()] = byte.ravel()
    n = np.arange(N)[:, None]
    g = np.arange(KT)[None, :]
    sb = s.astype(np.float16).view(np.uint8).reshape(N, KT, 2)
    sdest = HEADER_BYTES + (n // TILE_N * KT + g) * LUT_TILE_BYTES + TILE_CODE_BYTES + 2 * (n % TILE_N)
    out[sdest.ravel()] = sb[:, :, 0].ravel()
    out[sdest.ravel() + 1] = sb[:, :, 1].ravel()
    out[t_off:t_off + 32] = np.frombuffer(T.astype(np.float16).tobytes(), dtype=np.uint8)
    return out


def lut_unpack_weights(blob: np.ndarray):
    """Inverse of `lut_pack_weights`: returns (q, s, T, N, K)."""
    hdr = bytes(blob[:HEADER_BYTES])
    assert int.from_bytes(hdr[0:4], "little") == LUT_MAGIC
    N = int.from_bytes(hdr[8:16], "little", signed=True)
    K = int.from_bytes(hdr[16:24], "little", signed=True)
    t_off = int.from_bytes(hdr[32:40], "little")
    KT = K // TILE_K
    n = np.arange(N)[:, None]
    k = np.arange(K)[None, :]
    nt, r = n // TILE_N, n % TILE_N
    kt, kk = k // TILE_K, k % TILE_K
    j, high = kk // 2, kk % 2
    c, b = j // 16, j % 16
    src = HEADER_BYTES + (nt * KT + kt) * LUT_TILE_BYTES + (c * TILE_N + r) * 16 + b
    byte = blob[src]
    q = np.where(high == 1, byte >> 4, byte & 0x0F).astype(np.uint8)
    g = np.arange(KT)[None, :]
    ssrc = HEADER_BYTES + (nt * KT + g) * LUT_TILE_BYTES + TILE_CODE_BYTES + 2 * r
    s = (blob[ssrc].astype(np.uint16) | (blob[ssrc + 1].astype(np.uint16) << 8)).view(np.float16)
    T = np.frombuffer(bytes(blob[t_off:t_off + 32]), dtype=np.float16).copy()
    return q, s, T, N, K


# ---------------------------------------------------------------------------
# 3-bit lookup-table weights ("Fast Matrix Multiplications for Lookup
# Table-Quantized LLMs", abstract: bit widths that do not divide a byte).
# Same arithmetic as above with an 8-entry table (`lut_dequant`,
# `lut_gemm_exact`, `lut_error_bound` and `lut_quantize_weights` apply as they
# stand). The storage is this file's reading: a tile row's 128 indices are
# three 16-byte bit planes, plane c holding bit c of every index (bit kk of
# the plane, i.e. bit kk % 8 of byte kk // 8, is bit c of the index at in-tile
# k = kk), plane c of row r at (c * 128 + r) * 16, so no index straddles two
# 16-byte vectors; then the tile's 128 fp16 row scales.
LUT3_MAGIC = 0x544C3357  # b"W3LT" little-endian
LUT3_TILE_CODE_BYTES = 3 * 16 * TILE_N  # 6144
LUT3_TILE_BYTES = LUT3_TILE_CODE_BYTES + LUT_TILE_SCALE_BYTES  # 6400


def lut3_packed_bytes(N: int, K: int, group: int = GROUP) -> int:
    """Header + (N/128)*(K/128) tiles of 6400 bytes + the table (8 fp16) padded to 64 bytes."""
    return HEADER_BYTES + (N // TILE_N) * (K // TILE_K) * LUT3_TILE_BYTES + 64


def lut3_bit_position(r: int, kk: int, c: int):
    """(byte offset inside a tile's index area, bit) of bit c of the index of
    row r at in-tile k = kk."""
    return (c * TILE_N + r) * 16 + kk // 8, kk % 8


def lut3_pack_weights(q, s, T, group: int = GROUP) -> np.ndarray:
    """Writes the 3-bit lookup-table blob from its definition. Header as the
    4-bit blob's with magic 'W3LT' and tile bytes 6400; tile (nt, kt) at
    64 + (nt*(K/128) + kt)*6400: the three bit planes of each row, then the
    128 rows' fp16 scales of group kt (row r at 6144 + 2r); after the tiles
    the 8 fp16 table entries, zero padded to 64 bytes."""
    assert group == GROUP
    q = np.asarray(q, dtype=np.uint8)
    assert q.max(initial=0) < 8 and len(T) == 8
    N, K = q.shape
    KT = K // TILE_K
    out = np.zeros(lut3_packed_bytes(N, K, group), dtype=np.uint8)
    t_off = HEADER_BYTES + (N // TILE_N) * KT * LUT3_TILE_BYTES
    hdr = bytearray(HEADER_BYTES)
    hdr[0:4] = LUT3_MAGIC.to_bytes(4, "little")
    hdr[4:8] = (1).to_bytes(4, "little")
    hdr[8:16] = int(N).to_bytes(8, "little", signed=True)
    hdr[16:24] = int(K).to_bytes(8, "little", signed=True)
    hdr[24:28] = int(group).to_bytes(4, "little", signed=True)
    hdr[28:32] = LUT3_TILE_BYTES.to_bytes(4, "little")
    hdr[32:40] = int(t_off).to_bytes(8, "little")
    out[:HEADER_BYTES] = np.frombuffer(bytes(hdr), dtype=np.uint8)
    for n in range(N):
        nt, r = divmod(n, TILE_N)
        for kt in range(KT):
            base = HEADER_BYTES + (nt * KT + kt) * LUT3_TILE_BYTES
            row = q[n, kt * TILE_K:(kt + 1) * TILE_K]
            for c in range(3):
                bits = (row >> c) & 1
                plane = np.packbits(bits, bitorder="little")  # bit kk -> byte kk // 8, bit kk % 8
                off = base + (c * TILE_N + r) * 16
                out[off:off + 16] = plane
            sb = np.frombuffer(np.float16(s[n, kt]).tobytes(), dtype=np.uint8)
            out[base + LUT3_TILE_CODE_BYTES + 2 * r:base + LUT3_TILE_CODE_BYTES + 2 * r + 2] = sb
    out[t_off:t_off + 16] = np.frombuffer(np.asarray(T, dtype=np.float16).tobytes(), dtype=np.uint8)
    return out


def lut3_unpack_weights(blob: np.ndarray):
    """Inverse of `lut3_pack_weights`: returns (q, s, T, N, K)."""
    hdr = bytes(blob[:HEADER_BYTES])
    assert int.from_bytes(hdr[0:4], "little") == LUT3_MAGIC
    N = int.from_bytes(hdr[8:16], "little", signed=True)
    K = int.from_bytes(hdr[16:24], "little", signed=True)
    t_off = int.from_bytes(hdr[32:40], "little")
    KT = K // TILE_K
    q = np.zeros((N, K), dtype=np.uint8)
    s = np.zeros((N, KT), dtype=np.float16)
    for n in range(N):
        nt, r = divmod(n, TILE_N)
        for kt in range(KT):
            base = HEADER_BYTES + (nt * KT + kt) * LUT3_TILE_BYTES
            for c in range(3):
                off = base + (c * TILE_N + r) * 16
                bits = np.unpackbits(blob[off:off + 16], bitorder="little")
                q[n, kt * TILE_K:(kt + 1) * TILE_K] |= (bits << c).astype(np.uint8)
            so = base + LUT3_TILE_CODE_BYTES + 2 * r
            s[n, kt] = np.frombuffer(bytes(blob[so:so + 2]), dtype=np.float16)[0]
    T = np.frombuffer(bytes(blob[t_off:t_off + 16]), dtype=np.float16).copy()
    return q, s, T, N, K
