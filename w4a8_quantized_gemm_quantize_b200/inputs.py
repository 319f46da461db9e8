"""Seeded synthetic inputs for the W4A8 GEMM workloads.

This module only draws random numbers and names the layer shapes. It holds
none of the quantization or GEMM arithmetic: both the CUDA path and the CPU
oracle consume what it returns.

Workloads (the low-bit LLM-serving layers the pages study: Llama-3-8B and
Qwen1.5-72B linears, "QServe/QoQ" abstract on the lmdeploy issue
"[Feature] Support W4A8KV4 Quantization(QServe/QoQ)", Motivation):

* ``tiny``     M=16, K=512, N=256; codes drawn directly (q, z ~ U[0,15],
               s2 ~ U{1..8}, s1 ~ U[0.001, 0.01] as fp16).
* ``decode``   M in {1, 8, 16, 32} on the four Llama-3-8B linears.
* ``serving``  M in {64, 128, 256, 512} on the same linears.
* ``prefill``  M in {2048, 8192} on the same linears.
* ``qwen72b``  M in {1, 32, 256, 4096} on the four Qwen1.5-72B linears.

Activations are fp16 N(0, 1) with round(0.01*K) outlier channels scaled by
20; the outlier channels depend on K only, so every token of a layer shares
them. Dense weights are fp32 N(0, std) with std 0.02 (Llama) or 0.015 (Qwen).

Lookup-table weights (`lut_table`, `lut_codes`, 3-bit `lut3_table`,
`lut3_codes`): NormalFloat-style tables, uniform indices, group scales on
[0.005, 0.05].

KV-cache attention (`KV_WORKLOADS`): ``kv-tiny`` (3 sequences, 4 query / 2 kv
heads, <= 300 tokens), ``kv-decode`` (Llama-3-8B attention, 32 / 8 heads of
128, 16 sequences of 2048..4096 tokens), ``kv-long`` (4 x 32768),
``kv-qwen72b`` (64 / 64 heads, 8 x 2048..4096). Keys N(0, 1) with
round(0.04*D) outlier channels x10 per head, values and queries N(0, 1).
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass

import numpy as np

GROUP = 128

LLAMA3_8B_LINEARS = (
    ("qkv", 6144, 4096),
    ("o", 4096, 4096),
    ("gate_up", 28672, 4096),
    ("down", 4096, 14336),
)
QWEN15_72B_LINEARS = (
    ("qkv", 24576, 8192),
    ("o", 8192, 8192),
    ("gate_up", 49152, 8192),
    ("down", 8192, 24576),
)


@dataclass(frozen=True)
class Workload:
    name: str
    ms: tuple
    linears: tuple  # (layer name, N, K)
    weight_std: float  # 0.0 means: draw codes directly (tiny case)


WORKLOADS = {
    "tiny": Workload("tiny", (16,), (("tiny", 256, 512),), 0.0),
    "decode": Workload("decode", (1, 8, 16, 32), LLAMA3_8B_LINEARS, 0.02),
    "serving": Workload("serving", (64, 128, 256, 512), LLAMA3_8B_LINEARS, 0.02),
    "prefill": Workload("prefill", (2048, 8192), LLAMA3_8B_LINEARS, 0.02),
    "qwen72b": Workload("qwen72b", (1, 32, 256, 4096), QWEN15_72B_LINEARS, 0.015),
}


def seed_of(*parts) -> int:
    """A 63-bit seed derived from a descriptor tuple (stable across runs)."""
    h = hashlib.sha256(repr(parts).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def n_outlier_channels(K: int) -> int:
    """round(0.01*K), halves rounded up (K=512 -> 5, 4096 -> 41, 14336 -> 143)."""
    return int(np.floor(0.01 * K + 0.5))


def outlier_channels(K: int) -> np.ndarray:
    rng = np.random.default_rng(seed_of("outlier-channels", K))
    return np.sort(rng.choice(K, size=n_outlier_channels(K), replace=False))


def activations(M: int, K: int, seed: int, outlier_scale: float = 20.0) -> np.ndarray:
    """fp16 [M, K] row-major: N(0,1) with the layer's outlier channels x20."""
    rng = np.random.default_rng(seed)
    a = rng.standard_normal((M, K), dtype=np.float32)
    ch = outlier_channels(K)
    if ch.size:
        a[:, ch] *= np.float32(outlier_scale)
    return a.astype(np.float16)


def dense_weights(N: int, K: int, std: float, seed: int) -> np.ndarray:
    """fp32 [N, K] row-major, N(0, std)."""
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((N, K), dtype=np.float32)
    w *= np.float32(std)
    return w


def uniform_codes(N: int, K: int, seed: int, group: int = GROUP):
    """Codes drawn directly: q, z ~ U[0,15]; s2 ~ U{1..8}; s1 ~ U[0.001, 0.01] fp16.

    Returns (q uint8 [N,K], z uint8 [N,K/group], s2 uint8 [N,K/group], s1 fp16 [N]).
    """
    rng = np.random.default_rng(seed)
    G = K // group
    q = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    z = rng.integers(0, 16, size=(N, G), dtype=np.uint8)
    s2 = rng.integers(1, 9, size=(N, G), dtype=np.uint8)
    s1 = rng.uniform(0.001, 0.01, size=N).astype(np.float16)
    return q, z, s2, s1


def activation_seed(workload: str, M: int, K: int) -> int:
    return seed_of("act", workload, M, K)


def weight_seed(workload: str, N: int, K: int) -> int:
    return seed_of("weight", workload, N, K)


# ------------------------------------------------ lookup-table weights (LUT)
def lut_table(delta: float = 0.03) -> np.ndarray:
    """A NormalFloat-style 16-entry table (input data for the lookup-table
    GEMM): standard-normal quantiles at evenly spaced probabilities, 8 below
    and 7 above an exact zero, each side scaled to reach -1 / +1; fp16."""
    from scipy.special import ndtri
    neg = ndtri(np.linspace(delta, 0.5, 9)[:-1])
    pos = ndtri(np.linspace(0.5, 1.0 - delta, 8)[1:])
    t = np.concatenate([neg / -neg.min(), [0.0], pos / pos.max()])
    return t.astype(np.float16)


def lut_codes(N: int, K: int, seed: int, group: int = GROUP):
    """Lookup-table weights drawn directly: indices q ~ U[0,15] (uint8 [N,K])
    and per-(row, group) scales s ~ U[0.005, 0.05] (fp16 [N, K/group])."""
    rng = np.random.default_rng(seed)
    q = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    s = rng.uniform(0.005, 0.05, size=(N, K // group)).astype(np.float16)
    return q, s


# ------------------------------------------------ 4-bit KV-cache attention
# Attention geometry of the workloads' models: (query heads, kv heads, head dim).
LLAMA3_8B_ATTN = (32, 8, 128)
QWEN15_72B_ATTN = (64, 64, 128)


@dataclass(frozen=True)
class KvWorkload:
    name: str
    batch: int
    max_len: int      # cache capacity per sequence (tokens)
    heads: tuple      # (Hq, Hkv, D)
    ragged: bool      # lengths drawn in [max_len / 2, max_len], else all max_len


KV_WORKLOADS = {
    "kv-tiny": KvWorkload("kv-tiny", 3, 300, (4, 2, 128), True),
    "kv-decode": KvWorkload("kv-decode", 16, 4096, LLAMA3_8B_ATTN, True),
    "kv-long": KvWorkload("kv-long", 4, 32768, LLAMA3_8B_ATTN, False),
    "kv-qwen72b": KvWorkload("kv-qwen72b", 8, 4096, QWEN15_72B_ATTN, True),
}


def kv_vectors(B: int, H: int, L: int, D: int, seed: int, outlier_scale: float = 10.0) -> np.ndarray:
    """fp16 [B, H, L, D]: N(0, 1), with round(0.04 D) channels per head
    scaled by `outlier_scale` (the same channels for every token of a head,
    as keys have; pass 1.0 for values)."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, H, L, D), dtype=np.float32)
    n_out = int(np.floor(0.04 * D + 0.5))
    if outlier_scale != 1.0 and n_out > 0:
        for h in range(H):
            ch = rng.choice(D, size=n_out, replace=False)
            x[:, h, :, ch] *= outlier_scale
    return x.astype(np.float16)


def kv_queries(B: int, Hq: int, D: int, seed: int) -> np.ndarray:
    """fp16 [B, Hq, D] decode queries, N(0, 1)."""
    rng = np.random.default_rng(seed)
    return rng.standard_normal((B, Hq, D), dtype=np.float32).astype(np.float16)


def kv_seq_lens(wl: KvWorkload, seed: int) -> np.ndarray:
    """int32 [B] cache lengths of a workload (ragged: uniform on
    [max_len / 2, max_len], the first sequence always full)."""
    if not wl.ragged:
        return np.full(wl.batch, wl.max_len, dtype=np.int32)
    rng = np.random.default_rng(seed)
    lens = rng.integers(wl.max_len // 2, wl.max_len + 1, size=wl.batch).astype(np.int32)
    lens[0] = wl.max_len
    return lens


def lut3_table(delta: float = 0.06) -> np.ndarray:
    """An 8-entry NormalFloat-style table for 3-bit indices (input data):
    standard-normal quantiles at evenly spaced probabilities, 4 below and 3
    above an exact zero, each side scaled to reach -1 / +1; fp16."""
    from scipy.special import ndtri
    neg = ndtri(np.linspace(delta, 0.5, 5)[:-1])
    pos = ndtri(np.linspace(0.5, 1.0 - delta, 4)[1:])
    t = np.concatenate([neg / -neg.min(), [0.0], pos / pos.max()])
    return t.astype(np.float16)


def lut3_codes(N: int, K: int, seed: int, group: int = GROUP):
    """3-bit lookup-table weights drawn directly: indices q ~ U[0,7] (uint8
    [N,K]) and per-(row, group) scales s ~ U[0.005, 0.05] (fp16 [N, K/group])."""
    rng = np.random.default_rng(seed)
    q = rng.integers(0, 8, size=(N, K), dtype=np.uint8)
    s = rng.uniform(0.005, 0.05, size=(N, K // group)).astype(np.float16)
    return q, s
