"""CPU oracle for decode attention over a 4-bit KV cache — TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import this module. The product (the CUDA library and its Python binding)
never calls it, and it shares no code with the product.

What the pages fix: QoQ is W4A8KV4, i.e. the key/value cache is stored in 4
bits, and QServe makes the fused attention kernel memory-bound so that the
smaller cache turns into speed ("QServe/QoQ" abstract quoted in lmdeploy
issue "[Feature] Support W4A8KV4 Quantization(QServe/QoQ)", Motivation);
"PrefixQuant: Static Quantization Beats Dynamic through Prefixed Outliers in
LLMs" (Methodology, Key Findings) quantizes the KV cache to 4 bits as well
(W4A4KV4), with static per-tensor parameters. Neither page fixes a code
range, a rounding rule, the granularity of the parameters or the attention
arithmetic. Readings (each listed in the design notes):

* One cached vector = one token of one kv head, D values (D = 128 in the
  workloads). It is quantized asymmetrically on its own range widened to
  include zero: lo = min(min x, 0), hi = max(max x, 0),
  s = fp16_rn((hi - lo) / 15) (fp32 subtract and divide),
  z = clamp(rint(-lo / s), 0, 15), code = clamp(rint(x / s) + z, 0, 15),
  all in fp32 with IEEE divides, rint half to even; s == 0 (an all-zero
  vector) gives z = 0 and zero codes. Dequantized value (code - z) * s, exact
  in fp32. A static per-tensor scheme is the same format with the same
  (s, z) stored for every token.
* Storage: codes two per byte, element 2i in bits 0-3 and 2i+1 in bits 4-7
  of byte i of the vector's D/2 bytes; per vector one (s, z) pair of fp16
  values (z is an integer 0..15, exact in fp16).
* Decode attention, one new query token per sequence: for sequence b with
  cache length L_b and query head h, kv head g = h // (Hq / Hkv) (grouped
  queries), s_j = scale * sum_d q[d] * K^[j, d] over the L_b cached tokens,
  o = sum_j softmax(s)_j V^[j] with softmax over those L_b tokens; Y =
  fp16_rn(o); L_b = 0 gives Y = 0. `scale` is an fp32 number (typically
  1/sqrt(D)).
"""
from __future__ import annotations

import math

import numpy as np

KV_CODE_MAX = 15
U32 = 2.0 ** -23  # one fp32 ulp at 1: covers rounding and truncating operations


# ---------------------------------------------------------------------------
# Quantizing cached vectors
# ---------------------------------------------------------------------------
def quantize_kv(X: np.ndarray):
    """fp16 [..., D] -> (codes uint8 [..., D] in 0..15, s fp16 [...], z fp16 [...]).

    Follows the reading above step by step, in fp32."""
    x = np.asarray(X, dtype=np.float16).astype(np.float32)
    lo = np.minimum(x.min(axis=-1), np.float32(0))
    hi = np.maximum(x.max(axis=-1), np.float32(0))
    s = ((hi - lo) / np.float32(KV_CODE_MAX)).astype(np.float16)
    sf = s.astype(np.float32)
    pos = sf > 0
    safe = np.where(pos, sf, np.float32(1))
    # z is an integer 0..15; stored as that integer's fp16 value (a range with
    # lo = 0 gives rint(-0 / s) = -0, whose integer is 0, encoded +0)
    z = np.where(pos, np.clip(np.rint(-lo / safe), 0, KV_CODE_MAX), 0).astype(np.int32).astype(np.float32)
    codes = np.clip(np.rint(x / safe[..., None]) + z[..., None], 0, KV_CODE_MAX)
    codes = np.where(pos[..., None], codes, 0)
    return codes.astype(np.uint8), s, z.astype(np.float16)


def dequant_kv(codes: np.ndarray, s: np.ndarray, z: np.ndarray) -> np.ndarray:
    """(code - z) * s, exact, as float64 [..., D]."""
    return (codes.astype(np.float64) - z.astype(np.float64)[..., None]) * s.astype(np.float64)[..., None]


def pack_kv(codes: np.ndarray) -> np.ndarray:
    """uint8 [..., D] (0..15) -> uint8 [..., D/2]: element 2i low nibble, 2i+1 high."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_kv(P: np.ndarray) -> np.ndarray:
    p = np.asarray(P, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = p & 0x0F
    out[..., 1::2] = p >> 4
    return out


def kv_params(s: np.ndarray, z: np.ndarray) -> np.ndarray:
    """The stored per-vector parameters: fp16 pairs (s, z), shape [..., 2]."""
    return np.stack([np.asarray(s, np.float16), np.asarray(z, np.float16)], axis=-1)


# ---------------------------------------------------------------------------
# Decode attention
# ---------------------------------------------------------------------------
def _group_of(h: int, Hq: int, Hkv: int) -> int:
    assert Hq % Hkv == 0
    return h // (Hq // Hkv)


def attention_decode_exact(q, kc, kp, vc, vp, seq_lens, scale) -> np.ndarray:
    """float64 [B, Hq, D] outputs before the final rounding.

    q fp16 [B, Hq, D]; kc, vc packed codes uint8 [B, Hkv, Lmax, D/2];
    kp, vp fp16 (s, z) pairs [B, Hkv, Lmax, 2]; seq_lens [B]; scale fp32."""
    q = np.asarray(q, dtype=np.float16)
    B, Hq, D = q.shape
    Hkv = kc.shape[1]
    sc = float(np.float32(scale))
    out = np.zeros((B, Hq, D), dtype=np.float64)
    for b in range(B):
        L = int(seq_lens[b])
        if L == 0:
            continue
        for h in range(Hq):
            g = _group_of(h, Hq, Hkv)
            K = dequant_kv(unpack_kv(kc[b, g, :L]), kp[b, g, :L, 0], kp[b, g, :L, 1])
            V = dequant_kv(unpack_kv(vc[b, g, :L]), vp[b, g, :L, 0], vp[b, g, :L, 1])
            s = sc * (K @ q[b, h].astype(np.float64))
            p = np.exp(s - s.max())
            out[b, h] = (p @ V) / p.sum()
    return out


def attention_decode(q, kc, kp, vc, vp, seq_lens, scale) -> np.ndarray:
    """Y fp16 [B, Hq, D] = fp16_rn of the exact decode attention."""
    return attention_decode_exact(q, kc, kp, vc, vp, seq_lens, scale).astype(np.float16)


def attention_error_bound(q, kc, kp, vc, vp, seq_lens, scale) -> np.ndarray:
    """Bound on |o~ - o| per output element, float64 [B, Hq, D], for any
    evaluation in fp32 arithmetic (u = 2^-23 per operation, which covers
    rounding and truncation) in any order and any split of the tokens:

    * score s_j: the D products q[d] K^[j,d] and their sum carry at most
      gamma_{D+1} sum_d |q K^| (gamma_n = n u / (1 - n u)), times `scale`,
      plus 2 u |s_j| for two rounded multiplies (the vector's scale applied
      to the sum of q (code - z), and `scale`): delta_j; delta = max_j delta_j.
    * weight p_j = exp(s_j - max): the computed max is within delta of the
      exact one; the argument carries 2 delta + 2 u delta + 3 u |s_j - m|
      (subtraction, a change of exponent base, a rescale of a partial result
      by exp(m_part - m)), and each of the two exponentials 4 ulps (10 u in
      all, with the products by them): relative weight error
      eps_j = exp(R_j) - 1, R_j = 2 delta (1 + u) + 6 u |s_j - m| + 10 u.
      Perturbing the weights by eps_j moves o by at most
      sum_j p_j eps_j |V^_j - o| / sum_j p_j (1 - eps_j).
    * the sums over the L tokens (numerator sum p V^, denominator sum p)
      and the final division: gamma_{L+4} (sum p |V^| / sum p + |o|) / (1 -
      gamma_{L+4}) + u |o|.
    The sum of the three, plus 10% for the second-order terms left out."""
    q = np.asarray(q, dtype=np.float16)
    B, Hq, D = q.shape
    Hkv = kc.shape[1]
    sc = float(np.float32(scale))
    u = U32
    E = np.zeros((B, Hq, D), dtype=np.float64)
    for b in range(B):
        L = int(seq_lens[b])
        if L == 0:
            continue
        gD = (D + 1) * u / (1 - (D + 1) * u)
        gL = (L + 4) * u / (1 - (L + 4) * u)
        for h in range(Hq):
            g = _group_of(h, Hq, Hkv)
            K = dequant_kv(unpack_kv(kc[b, g, :L]), kp[b, g, :L, 0], kp[b, g, :L, 1])
            V = dequant_kv(unpack_kv(vc[b, g, :L]), vp[b, g, :L, 0], vp[b, g, :L, 1])
            qd = q[b, h].astype(np.float64)
            s = sc * (K @ qd)
            m = s.max()
            delta = np.max(abs(sc) * gD * (np.abs(K) @ np.abs(qd)) + 2 * u * np.abs(s))
            p = np.exp(s - m)
            o = (p @ V) / p.sum()
            R = 2 * delta * (1 + u) + 6 * u * np.abs(s - m) + 10 * u
            eps = np.expm1(R)
            w = (p * eps) @ np.abs(V - o) / np.sum(p * (1 - eps))
            acc = gL * ((p @ np.abs(V)) / p.sum() + np.abs(o)) / (1 - gL) + u * np.abs(o)
            E[b, h] = 1.1 * (w + acc)
    return E
