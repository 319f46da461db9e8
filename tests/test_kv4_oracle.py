"""Pins for the 4-bit KV-cache attention oracle (oracle/kv4_oracle.py).

Each test ties the oracle to something other than itself: values on the
quantization grid that must come back unchanged, the half-step error of a
rounding quantizer, hand-computed packed bytes, closed forms of softmax
attention (one token, uniform weights, two tokens, the hard-max limit),
invariances (token order, grouped-query sharing, padding) and fp32
evaluations in random orders and splits that must stay within the stated
bound, which in turn must be tight enough to see one dropped token.
"""
import math

import numpy as np
import pytest

from oracle import kv4_oracle as KV
from w4a8_quantized_gemm_quantize_b200 import inputs as I


# ------------------------------------------------------------- quantizer
def test_grid_values_come_back_unchanged():
    """x = (c - z) * s with c covering 0 and 15 and s a power of two: the
    range is exactly [-z s, (15 - z) s], so s, z and c are recovered."""
    rng = np.random.default_rng(1)
    for z in range(16):
        for e in (-6, -2, 0, 3):
            s = 2.0 ** e
            c = rng.integers(0, 16, size=(7, 128))
            c[:, 0], c[:, 1] = 0, 15
            if z == 0:
                c[:, 0] = 0
            x = ((c - z) * s).astype(np.float16)
            assert np.array_equal(x.astype(np.float64), (c - z) * s)  # exact in fp16
            codes, sq, zq = KV.quantize_kv(x)
            assert (sq == np.float16(s)).all() and (zq == z).all()
            assert np.array_equal(codes, c)


def test_error_is_at_most_half_a_step():
    """|x - x^| <= s/2, plus the share of the range lost when s is rounded to
    fp16 (at most (hi - lo) 2^-11) for the values clamped at code 15."""
    x = np.concatenate([I.kv_vectors(1, 4, 64, 128, 11)[0].reshape(-1, 128),
                        I.kv_vectors(1, 2, 64, 128, 12, outlier_scale=1.0)[0].reshape(-1, 128),
                        np.abs(I.kv_vectors(1, 1, 16, 128, 13)[0, 0])], axis=0)
    codes, s, z = KV.quantize_kv(x)
    xf = x.astype(np.float64)
    xh = KV.dequant_kv(codes, s, z)
    lo = np.minimum(xf.min(-1), 0)
    hi = np.maximum(xf.max(-1), 0)
    bound = s.astype(np.float64) / 2 + (hi - lo) * 2.0 ** -11
    assert (np.abs(xf - xh) <= bound[:, None]).all()
    # the extremes map to the ends of the code range
    rows = np.arange(x.shape[0])
    pos, neg = xf.max(-1) > 0, xf.min(-1) < 0
    assert (codes[rows, xf.argmax(-1)][pos] == 15).all()
    assert (codes[rows, xf.argmin(-1)][neg] == 0).all()


def test_zero_and_constant_vectors():
    codes, s, z = KV.quantize_kv(np.zeros((2, 128), np.float16))
    assert (s == 0).all() and (z == 0).all() and (codes == 0).all()
    assert (KV.dequant_kv(codes, s, z) == 0).all()
    c = np.float16(3.0)
    codes, s, z = KV.quantize_kv(np.full((1, 128), c))
    assert s[0] == np.float16(np.float32(3.0) / np.float32(15)) and z[0] == 0 and (codes == 15).all()
    assert abs(KV.dequant_kv(codes, s, z)[0, 0] - 3.0) <= 3.0 * 2.0 ** -11
    codes, s, z = KV.quantize_kv(np.full((1, 128), -c))
    assert z[0] == 15 and (codes == 0).all()
    assert abs(KV.dequant_kv(codes, s, z)[0, 0] + 3.0) <= 3.0 * 2.0 ** -11


def test_zero_point_is_stored_as_its_integer():
    """z is an integer 0..15 stored in fp16: a vector without negative
    values (lo = 0) stores z = 0 as +0, not -0."""
    x = np.abs(I.kv_vectors(1, 1, 8, 128, 17)[0, 0])
    _, s, z = KV.quantize_kv(x)
    assert (s > 0).all() and (z.view(np.uint16) == 0).all()
    assert (KV.kv_params(s, z).view(np.uint32)[..., 0] >> 16 == 0).all()


def test_static_parameters_reduce_to_codes():
    """A per-tensor (static) scheme stores one (s, z) for every vector; the
    dequantization only reads the pair, so vectors quantized with a shared
    pair dequantize as (c - z) s with that pair."""
    c = np.random.default_rng(3).integers(0, 16, size=(5, 128)).astype(np.uint8)
    s = np.full(5, np.float16(0.125))
    z = np.full(5, np.float16(6))
    assert np.array_equal(KV.dequant_kv(c, s, z), (c.astype(np.float64) - 6) * 0.125)


def test_pack_hand_bytes_and_round_trip():
    c = np.array([[1, 2, 3, 4, 15, 0, 0, 15]], dtype=np.uint8)
    assert KV.pack_kv(c).tolist() == [[0x21, 0x43, 0x0F, 0xF0]]
    allc = np.arange(256, dtype=np.uint8)
    pairs = np.stack([allc & 15, allc >> 4], axis=-1).reshape(1, -1)
    assert np.array_equal(KV.pack_kv(pairs)[0], allc)
    assert np.array_equal(KV.unpack_kv(KV.pack_kv(pairs)), pairs)
    p = KV.kv_params(np.float16(0.5), np.float16(7))
    assert p.dtype == np.float16 and p.tolist() == [0.5, 7.0]


# ---------------------------------------------------------- attention helpers
def cache_from(K, V):
    """fp16 K, V [B, Hkv, L, D] -> packed codes and (s, z) pairs."""
    kc, ks, kz = KV.quantize_kv(K)
    vc, vs, vz = KV.quantize_kv(V)
    return KV.pack_kv(kc), KV.kv_params(ks, kz), KV.pack_kv(vc), KV.kv_params(vs, vz)


def direct_cache(kcodes, ks, kz, vcodes, vs, vz):
    return (KV.pack_kv(kcodes), KV.kv_params(ks, kz), KV.pack_kv(vcodes), KV.kv_params(vs, vz))


def random_case(B, Hq, Hkv, L, D, seed, lens=None):
    K = I.kv_vectors(B, Hkv, L, D, seed)
    V = I.kv_vectors(B, Hkv, L, D, seed + 1, outlier_scale=1.0)
    q = I.kv_queries(B, Hq, D, seed + 2)
    lens = np.full(B, L, np.int32) if lens is None else np.asarray(lens, np.int32)
    return (q,) + cache_from(K, V) + (lens,)


# ------------------------------------------------------------ attention pins
def test_one_token_returns_its_value():
    q, kc, kp, vc, vp, lens = random_case(2, 4, 2, 1, 128, 21)
    o = KV.attention_decode_exact(q, kc, kp, vc, vp, lens, 0.088)
    for b in range(2):
        for h in range(4):
            Vh = KV.dequant_kv(KV.unpack_kv(vc[b, h // 2, :1]), vp[b, h // 2, :1, 0], vp[b, h // 2, :1, 1])[0]
            assert np.array_equal(o[b, h], Vh)


def test_zero_query_averages_the_values():
    q, kc, kp, vc, vp, lens = random_case(1, 2, 1, 37, 128, 31)
    q[:] = 0
    o = KV.attention_decode_exact(q, kc, kp, vc, vp, lens, 1.0)
    V = KV.dequant_kv(KV.unpack_kv(vc[0, 0]), vp[0, 0, :, 0], vp[0, 0, :, 1])
    assert np.allclose(o[0, 0], V.mean(axis=0), rtol=0, atol=1e-13)
    assert np.allclose(o[0, 1], V.mean(axis=0), rtol=0, atol=1e-13)


def test_two_tokens_closed_form():
    """q = e_0, keys 2 e_0 and 0, scale 1/2: scores 1 and 0, weights
    e/(1+e) and 1/(1+e); values built directly from codes."""
    D = 128
    q = np.zeros((1, 1, D), np.float16)
    q[0, 0, 0] = 1
    kcodes = np.zeros((1, 1, 2, D), np.uint8)
    kcodes[0, 0, 0, 0] = 2
    vcodes = np.zeros((1, 1, 2, D), np.uint8)
    vcodes[0, 0, 0, :] = 3
    vcodes[0, 0, 1, :] = 9
    ones = np.ones((1, 1, 2), np.float16)
    zeros = np.zeros((1, 1, 2), np.float16)
    kc, kp, vc, vp = direct_cache(kcodes, ones, zeros, vcodes, ones * np.float16(0.25), ones * np.float16(1))
    o = KV.attention_decode_exact(q, kc, kp, vc, vp, np.array([2]), 0.5)
    w0 = math.e / (1 + math.e)
    want = w0 * (3 - 1) * 0.25 + (1 - w0) * (9 - 1) * 0.25
    assert np.allclose(o[0, 0], want, rtol=0, atol=1e-14)


def test_hard_max_limit():
    """Scaling the scores up makes softmax select the top-scoring token."""
    q, kc, kp, vc, vp, lens = random_case(1, 1, 1, 50, 128, 41)
    K = KV.dequant_kv(KV.unpack_kv(kc[0, 0]), kp[0, 0, :, 0], kp[0, 0, :, 1])
    V = KV.dequant_kv(KV.unpack_kv(vc[0, 0]), vp[0, 0, :, 0], vp[0, 0, :, 1])
    s = K @ q[0, 0].astype(np.float64)
    top = np.argsort(s)[-2:]
    gap = s[top[1]] - s[top[0]]
    assert gap > 0
    o = KV.attention_decode_exact(q, kc, kp, vc, vp, lens, 800.0 / gap)
    assert np.allclose(o[0, 0], V[top[1]], rtol=0, atol=1e-12 * np.abs(V).max() + 1e-300)


def test_token_order_does_not_matter():
    q, kc, kp, vc, vp, lens = random_case(1, 2, 1, 90, 128, 51)
    perm = np.random.default_rng(5).permutation(90)
    o1 = KV.attention_decode_exact(q, kc, kp, vc, vp, lens, 0.0884)
    o2 = KV.attention_decode_exact(q, kc[:, :, perm], kp[:, :, perm], vc[:, :, perm], vp[:, :, perm], lens, 0.0884)
    assert np.allclose(o1, o2, rtol=1e-13, atol=1e-14)


def test_grouped_queries_share_their_kv_head():
    """Hq = 4 on Hkv = 2 equals Hq = 4 on Hkv = 4 with each kv head repeated."""
    q, kc, kp, vc, vp, lens = random_case(2, 4, 2, 33, 128, 61)
    rep = lambda a: np.repeat(a, 2, axis=1)
    o1 = KV.attention_decode_exact(q, kc, kp, vc, vp, lens, 0.0884)
    o2 = KV.attention_decode_exact(q, rep(kc), rep(kp), rep(vc), rep(vp), lens, 0.0884)
    assert np.array_equal(o1, o2)


def test_padding_beyond_the_length_is_ignored():
    q, kc, kp, vc, vp, _ = random_case(3, 2, 1, 40, 128, 71)
    lens = np.array([40, 17, 0], np.int32)
    o1 = KV.attention_decode_exact(q, kc, kp, vc, vp, lens, 0.0884)
    kc2, kp2, vc2, vp2 = kc.copy(), kp.copy(), vc.copy(), vp.copy()
    for b, L in enumerate(lens):
        kc2[b, :, L:] = 0xFF
        vc2[b, :, L:] = 0x5A
        kp2[b, :, L:] = np.float16(np.inf)
        vp2[b, :, L:] = np.float16(np.nan)
    with np.errstate(invalid="ignore", over="ignore"):
        o2 = KV.attention_decode_exact(q, kc2, kp2, vc2, vp2, lens, 0.0884)
    assert np.array_equal(o1, o2)
    assert (o1[2] == 0).all()
    # and the fp16 output is the rounding of the exact one
    assert np.array_equal(KV.attention_decode(q, kc, kp, vc, vp, lens, 0.0884), o1.astype(np.float16))


# --------------------------------------------------- the fp32 error bound
def chop32(x):
    """float64 -> float32 rounded toward zero (a truncating adder)."""
    x = np.asarray(x, np.float64)
    r = x.astype(np.float32)
    over = np.abs(r.astype(np.float64)) > np.abs(x)
    r = np.where(over, np.nextafter(r, np.float32(0)), r)
    return r.astype(np.float32)


def fp32_attention(q, kc, kp, vc, vp, lens, scale, rng, max_chunk, chop=False):
    """An fp32 evaluation in a random order: scores summed over the head
    dimension in a random order; tokens split at random into chunks of at
    most max_chunk, each with its own max, exponentials and sums (random
    order), the chunks combined with exp(m_c - m) factors. chop: the
    numerator's sums over tokens truncate instead of rounding to nearest
    (the denominator's do not, so the two errors do not cancel)."""
    B, Hq, D = q.shape
    Hkv = kc.shape[1]
    f = np.float32
    add = (lambda a, b: chop32(np.float64(a) + np.asarray(b, np.float64))) if chop else (lambda a, b: (a + b).astype(f))
    out = np.zeros((B, Hq, D), np.float64)
    for b in range(B):
        L = int(lens[b])
        if L == 0:
            continue
        for h in range(Hq):
            g = h // (Hq // Hkv)
            K = KV.dequant_kv(KV.unpack_kv(kc[b, g, :L]), kp[b, g, :L, 0], kp[b, g, :L, 1]).astype(f)
            V = KV.dequant_kv(KV.unpack_kv(vc[b, g, :L]), vp[b, g, :L, 0], vp[b, g, :L, 1]).astype(f)
            qf = q[b, h].astype(f)
            acc = np.zeros(L, f)
            for d in rng.permutation(D):
                acc = (acc + K[:, d] * qf[d]).astype(f)
            s = (acc * f(scale)).astype(f)
            cuts = np.sort(rng.choice(np.arange(1, L), size=min(L - 1, L // max_chunk + rng.integers(0, 3)),
                                      replace=False)) if L > 1 else np.array([], int)
            bounds = np.concatenate([[0], cuts, [L]])
            parts = []
            for c0, c1 in zip(bounds[:-1], bounds[1:]):
                sc = s[c0:c1]
                mc = sc.max()
                p = np.exp((sc - mc).astype(f)).astype(f)
                l = f(0)
                num = np.zeros(D, f)
                for j in rng.permutation(c1 - c0):
                    l = f(l + p[j])
                    num = add(num, (p[j] * V[c0 + j]).astype(f))
                parts.append((mc, l, num))
            m = max(pm for pm, _, _ in parts)
            den = f(0)
            num = np.zeros(D, f)
            for i in rng.permutation(len(parts)):
                mc, l, n = parts[i]
                fac = np.exp(f(mc - m)).astype(f)
                den = f(den + fac * l)
                num = (num + fac * n).astype(f)
            out[b, h] = (num / den).astype(f)
    return out


@pytest.mark.parametrize("L,chunk,seed", [(1, 1, 1), (5, 2, 2), (64, 16, 3), (300, 64, 4), (700, 128, 5)])
def test_fp32_evaluations_stay_within_the_bound(L, chunk, seed):
    q, kc, kp, vc, vp, lens = random_case(2, 4, 2, L, 128, 100 + seed, lens=[L, max(1, L // 3)])
    o = KV.attention_decode_exact(q, kc, kp, vc, vp, lens, 0.08838834764831845)
    E = KV.attention_error_bound(q, kc, kp, vc, vp, lens, 0.08838834764831845)
    rng = np.random.default_rng(seed)
    for _ in range(3):
        of = fp32_attention(q, kc, kp, vc, vp, lens, 0.08838834764831845, rng, chunk)
        assert (np.abs(of - o) <= E).all()


def test_fp32_bound_with_large_scores():
    """Outlier keys and a large scale: scores spread over hundreds."""
    q, kc, kp, vc, vp, lens = random_case(1, 2, 1, 200, 128, 81)
    q = (q.astype(np.float32) * 4).astype(np.float16)
    o = KV.attention_decode_exact(q, kc, kp, vc, vp, lens, 0.5)
    E = KV.attention_error_bound(q, kc, kp, vc, vp, lens, 0.5)
    of = fp32_attention(q, kc, kp, vc, vp, lens, 0.5, np.random.default_rng(9), 32)
    assert (np.abs(of - o) <= E).all()


def test_bound_sees_a_dropped_token():
    """At moderate lengths the bound is far below the effect of leaving one
    token out, so a kernel that skips or repeats a token fails it."""
    L = 256
    q, kc, kp, vc, vp, lens = random_case(1, 2, 1, L, 128, 91)
    o = KV.attention_decode_exact(q, kc, kp, vc, vp, lens, 0.0884)
    E = KV.attention_error_bound(q, kc, kp, vc, vp, lens, 0.0884)
    for j in (0, 100, L - 1):
        keep = np.delete(np.arange(L), j)
        od = KV.attention_decode_exact(q, kc[:, :, keep], kp[:, :, keep], vc[:, :, keep], vp[:, :, keep],
                                       np.array([L - 1]), 0.0884)
        assert (np.abs(od - o) > E).any()


def test_fp32_bound_covers_long_sums():
    """Uniform weights (a zero query): the weights carry almost no error, so
    the accumulation term of the bound has to cover the fp32 rounding of a
    long sum of values with many significant bits."""
    L, D = 3001, 128
    q = np.zeros((1, 1, D), np.float16)
    rng = np.random.default_rng(2)
    kcodes = np.zeros((1, 1, L, D), np.uint8)
    vcodes = rng.integers(0, 16, size=(1, 1, L, D)).astype(np.uint8)
    s = rng.uniform(0.05, 0.2, size=(1, 1, L)).astype(np.float16)
    z = rng.integers(0, 16, size=(1, 1, L)).astype(np.float16)
    kc, kp, vc, vp = direct_cache(kcodes, s, z, vcodes, s, z)
    lens = np.array([L], np.int32)
    o = KV.attention_decode_exact(q, kc, kp, vc, vp, lens, 1.0)
    E = KV.attention_error_bound(q, kc, kp, vc, vp, lens, 1.0)
    of = fp32_attention(q, kc, kp, vc, vp, lens, 1.0, np.random.default_rng(4), L)
    assert (np.abs(of - o) > 0).any()   # the fp32 sums do round here
    assert (np.abs(of - o) <= E).all()


def test_fp32_bound_covers_truncating_sums():
    """Long sums with a truncating adder: every addition errs the same way,
    so the error grows with the length; small scores give weights with full
    fp32 mantissas (every product truncates) while keeping the weight term
    of the bound small, so only its accumulation term covers this."""
    L, D = 3001, 128
    rng = np.random.default_rng(3)
    q = (rng.standard_normal((1, 1, D)) * 0.005).astype(np.float16)
    kcodes = rng.integers(0, 16, size=(1, 1, L, D)).astype(np.uint8)
    vcodes = rng.integers(8, 16, size=(1, 1, L, D)).astype(np.uint8)
    s = rng.uniform(0.05, 0.2, size=(1, 1, L)).astype(np.float16)
    zk = np.full((1, 1, L), np.float16(8))
    zv = np.zeros((1, 1, L), np.float16)
    kc, kp, vc, vp = direct_cache(kcodes, s, zk, vcodes, s, zv)
    lens = np.array([L], np.int32)
    o = KV.attention_decode_exact(q, kc, kp, vc, vp, lens, 1.0)
    E = KV.attention_error_bound(q, kc, kp, vc, vp, lens, 1.0)
    of = fp32_attention(q, kc, kp, vc, vp, lens, 1.0, np.random.default_rng(5), L, chop=True)
    err = np.abs(of - o)
    assert (err <= E).all()
    assert err.max() > 100 * 2.0 ** -23 * np.abs(o).max()  # far above a single rounding
