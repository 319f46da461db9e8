"""Pins for the CPU oracle: checks against what the mathematics fixes, not
against the oracle's own formulas retyped.

Covered: a hand-worked example; closed forms (constant rows, one-hot rows,
all-ones products, exactly representable weight groups); symmetries
(negation, power-of-two scaling, linearity); the exact rational rounding of
every activation code on small inputs; brute-force pure-Python GEMMs; the
full (q, z, s2) domain of the bytewise (SIMD-within-a-register)
dequantization; hand-computed byte positions of the packed layout.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import w4a8_oracle as O
from tests._util import max_ulp_fp16

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------- golden
def _hand_case():
    with open(os.path.join(GOLDEN, "hand_worked_w4a8.json")) as f:
        g = json.load(f)
    K = g["K"]
    A = np.zeros((2, K), dtype=np.float16)
    A[0, :4] = g["A_row0_k0_3"]
    N = 2
    q = np.zeros((N, K), dtype=np.uint8)
    z = np.zeros((N, 1), dtype=np.uint8)
    s2 = np.zeros((N, 1), dtype=np.uint8)
    for n, key in enumerate(("n0", "n1")):
        w = g["weights"][key]
        q[n, :] = w["q_other"]
        q[n, :4] = w["q_k0_3"]
        z[n, 0] = w["z"]
        s2[n, 0] = w["s2"]
    s1 = np.array(g["weights"]["s1"], dtype=np.float16)
    return g, A, q, z, s2, s1


def test_hand_worked_example():
    g, A, q, z, s2, s1 = _hand_case()
    A8, sA, rowsum = O.quantize_act(A)
    assert sA.astype(np.float64).tolist() == g["sA"]
    assert A8[0, :4].tolist() == g["A8_row0_k0_3"]
    assert not A8[0, 4:].any() and not A8[1].any()
    assert rowsum.tolist() == g["rowsum"]
    W8 = O.dequant_weights(q, z, s2)
    assert W8[0, :4].tolist() == g["weights"]["n0"]["W8_k0_3"]
    assert W8[1, :4].tolist() == g["weights"]["n1"]["W8_k0_3"]
    acc = O.gemm_acc(A8, W8)
    assert acc.tolist() == g["acc"]
    Y = O.epilogue(acc, sA, s1)
    assert Y.astype(np.float64).tolist() == g["Y"]


# --------------------------------------------------------- quantize_act
@pytest.mark.parametrize("c", [1.0, -3.5, 0.001, 1000.0, 65504.0, 6.1e-5])
def test_quantize_constant_row(c):
    A = np.full((3, 256), c, dtype=np.float16)
    A8, sA, rowsum = O.quantize_act(A)
    expect_code = 127 if c > 0 else -127
    assert (A8 == expect_code).all()
    # sA is fp16 of |c|/127 computed in fp32
    expect_s = np.float16(np.float32(abs(float(np.float16(c)))) / np.float32(127))
    assert (sA == expect_s).all()
    assert (rowsum == expect_code * 256).all()


def test_quantize_zero_row():
    A = np.zeros((2, 128), dtype=np.float16)
    A[1, 7] = 3.0
    A8, sA, rowsum = O.quantize_act(A)
    assert sA[0] == 0 and not A8[0].any() and rowsum[0] == 0
    assert A8[1, 7] == 127 and A8[1].sum() == 127


def _rand_act(M, K, seed):
    rng = np.random.default_rng(seed)
    a = rng.standard_normal((M, K)).astype(np.float32)
    a[:, rng.choice(K, max(1, K // 100), replace=False)] *= 20
    return a.astype(np.float16)


def test_quantize_odd_symmetry():
    A = _rand_act(8, 512, 1)
    A8, sA, rs = O.quantize_act(A)
    B8, sB, rsB = O.quantize_act(-A)
    assert (B8 == -A8).all() and (sB == sA).all() and (rsB == -rs).all()


@pytest.mark.parametrize("e", [-4, -1, 1, 3])
def test_quantize_power_of_two_scaling(e):
    # keep every value normal in fp16 after scaling: |A| >= 2^-6
    A = _rand_act(8, 384, 2).astype(np.float32)
    A = np.where(np.abs(A) < 2.0 ** -6, np.copysign(2.0 ** -6, A), A).astype(np.float16)
    A8, sA, _ = O.quantize_act(A)
    As = (A.astype(np.float32) * np.float32(2.0 ** e)).astype(np.float16)
    assert (As.astype(np.float32) == A.astype(np.float32) * np.float32(2.0 ** e)).all()
    B8, sB, _ = O.quantize_act(As)
    assert (B8 == A8).all()
    assert (sB.astype(np.float32) == sA.astype(np.float32) * np.float32(2.0 ** e)).all()


def test_quantize_error_bound_and_range():
    A = _rand_act(32, 1024, 3)
    A8, sA, rowsum = O.quantize_act(A)
    sf = sA.astype(np.float64)[:, None]
    Af = A.astype(np.float64)
    assert np.abs(A8).max() <= 127
    clamped = np.abs(Af / sf) > 127
    err = np.abs(Af - A8.astype(np.float64) * sf)
    assert (err[~clamped] <= sf.repeat(A.shape[1], 1)[~clamped] * (0.5 + 1e-6)).all()
    assert (rowsum == A8.astype(np.int64).sum(1)).all()
    # per-row amax reaches the top code (up to the fp16 rounding of the scale)
    assert (np.abs(A8).max(1) >= 126).all()


def _nearest_even(fr: Fraction) -> int:
    fl = fr.numerator // fr.denominator
    rem = fr - fl
    if rem > Fraction(1, 2):
        return fl + 1
    if rem < Fraction(1, 2):
        return fl
    return fl if fl % 2 == 0 else fl + 1


def test_quantize_codes_exact_rational():
    """Each code is the integer nearest to A / sA in exact arithmetic (ties
    to even, clamped), except where A / sA lies so close to a half-integer
    that the fp32 quotient may round across it."""
    A = _rand_act(4, 256, 4)
    A8, sA, _ = O.quantize_act(A)
    n_checked = 0
    for m in range(A.shape[0]):
        amax = max(abs(Fraction(float(v))) for v in A[m])
        assert Fraction(float(np.float16(np.float32(float(amax)) / np.float32(127)))) == Fraction(float(sA[m]))
        s = Fraction(float(sA[m]))
        for k in range(A.shape[1]):
            x = Fraction(float(A[m, k])) / s
            frac = x - (x.numerator // x.denominator)
            if abs(frac - Fraction(1, 2)) < Fraction(1, 10 ** 5):
                continue
            want = max(-127, min(127, _nearest_even(x)))
            assert int(A8[m, k]) == want, (m, k)
            n_checked += 1
    assert n_checked > 1000


# ------------------------------------------------- static activation scale
def test_static_quantize_codes_exact_rational():
    """Static per-tensor codes: the integer nearest to A / s in exact
    arithmetic (ties to even), clamped to [-127, 127] (so tokens with
    |A| > 127.5 s saturate), except where A / s lies so close to a
    half-integer that the fp32 quotient may round across it; sA repeats s
    and rowsum sums the codes."""
    A = _rand_act(5, 256, 14)
    A[2] *= 40  # an outlier token: many codes saturate under the tensor scale
    s = np.float16(0.0123)
    A8, sA, rs = O.quantize_act_static(A, s)
    assert (sA.view(np.uint16) == np.uint16(s.view(np.uint16))).all()
    assert (rs == A8.astype(np.int64).sum(1)).all()
    S = Fraction(float(s))
    n_checked = n_clamped = 0
    for m in range(A.shape[0]):
        for k in range(A.shape[1]):
            x = Fraction(float(A[m, k])) / S
            frac = x - (x.numerator // x.denominator)
            if abs(frac - Fraction(1, 2)) < Fraction(1, 10 ** 5):
                continue
            want = max(-127, min(127, _nearest_even(x)))
            n_clamped += abs(want) == 127 and abs(x) > Fraction(255, 2)
            assert int(A8[m, k]) == want, (m, k)
            n_checked += 1
    assert n_checked > 1200 and n_clamped > 50


def test_static_quantize_reduces_to_dynamic_per_row():
    """With the tensor scale set to a token's own dynamic scale, that
    token's static codes are its dynamic codes (same rounding and range)."""
    A = _rand_act(6, 512, 15)
    A8d, sAd, rsd = O.quantize_act(A)
    for m in range(A.shape[0]):
        A8s, sAs, rss = O.quantize_act_static(A[m:m + 1], sAd[m])
        assert (A8s[0] == A8d[m]).all() and rss[0] == rsd[m]
        assert sAs[0].view(np.uint16) == sAd[m].view(np.uint16)


def test_static_quantize_zero_scale_and_symmetry():
    A = _rand_act(3, 128, 16)
    A8, sA, rs = O.quantize_act_static(A, np.float16(0))
    assert not A8.any() and not rs.any() and not sA.astype(np.float32).any()
    s = np.float16(0.02)
    A8p, _, rsp = O.quantize_act_static(A, s)
    A8n, _, rsn = O.quantize_act_static(-A, s)
    assert (A8n == -A8p).all() and (rsn == -rsp).all()  # rint is odd, the clamp symmetric
    # power-of-two rescaling of both A and s leaves every code unchanged
    s4 = np.float16(np.float32(s) * 4)  # exact: a power-of-two rescaling of an fp16 normal
    A8q, _, _ = O.quantize_act_static((A.astype(np.float32) * 4).astype(np.float16), s4)
    assert (A8q == A8p).all()


# ------------------------------------------------------------- weights
def test_dequant_full_domain_bytewise():
    """All 16*16*8 (q, z, s2): the oracle's W8 lies in [-120, 120] and equals
    the value that the overflow-free bytewise form yields: the byte
    q*s2 + (128 - z*s2) stays in [8, 248] (no carry into the next byte of a
    32-bit word), and flipping its top bit gives W8 as a two's-complement
    int8."""
    q, z, s2 = np.meshgrid(np.arange(16), np.arange(16), np.arange(1, 9), indexing="ij")
    q, z, s2 = q.ravel(), z.ravel(), s2.ravel()
    W8 = O.dequant_weights(q.reshape(-1, 1).astype(np.uint8),
                           z.reshape(-1, 1).astype(np.uint8),
                           s2.reshape(-1, 1).astype(np.uint8), group=1).ravel()
    assert W8.min() == -120 and W8.max() == 120
    for qq, zz, ss, w in zip(q.tolist(), z.tolist(), s2.tolist(), W8.tolist()):
        byte = qq * ss + (128 - zz * ss)
        assert 8 <= byte <= 248
        flipped = byte ^ 0x80
        as_int8 = flipped - 256 if flipped >= 128 else flipped
        assert as_int8 == w
    # four packed lanes at once: no lane disturbs its neighbour
    rng = np.random.default_rng(5)
    for _ in range(2000):
        qs = rng.integers(0, 16, 4)
        zz = int(rng.integers(0, 16))
        ss = int(rng.integers(1, 9))
        word = sum(int(v) << (8 * i) for i, v in enumerate(qs))
        res = (word * ss + (128 - zz * ss) * 0x01010101) ^ 0x80808080
        assert res < 2 ** 32
        lanes = [((res >> (8 * i)) & 0xFF) for i in range(4)]
        lanes = [v - 256 if v >= 128 else v for v in lanes]
        ref = O.dequant_weights(qs.reshape(1, 4).astype(np.uint8), np.array([[zz]], np.uint8),
                                np.array([[ss]], np.uint8), group=4).ravel().tolist()
        assert lanes == ref


def test_unsigned_biased_accumulation_identity():
    """The GEMM may multiply the biased unsigned bytes B = W8 + 128 =
    q*s2 + (128 - z*s2) in [8, 248] against the int8 activations and subtract
    128 * sum_k A8 afterwards: sum_k A8 (W8 + 128) - 128 sum_k A8 equals the
    oracle's accumulator exactly, and the biased sum stays inside int32 for
    every K <= 65536 (|sum| <= 127 * 248 * 65536 < 2^31)."""
    assert 127 * 248 * 65536 < 2 ** 31
    rng = np.random.default_rng(17)
    for K in (128, 384, 1024):
        M, N = 3, 5
        q = rng.integers(0, 16, (N, K)).astype(np.uint8)
        z = rng.integers(0, 16, (N, K // 128)).astype(np.uint8)
        s2 = rng.integers(1, 9, (N, K // 128)).astype(np.uint8)
        A8 = rng.integers(-127, 128, (M, K)).astype(np.int8)
        ref = O.gemm_acc(A8, O.dequant_weights(q, z, s2))
        zz = np.repeat(z.astype(np.int64), 128, axis=1)
        ss = np.repeat(s2.astype(np.int64), 128, axis=1)
        biased = q.astype(np.int64) * ss + (128 - zz * ss)
        assert biased.min() >= 8 and biased.max() <= 248
        for m in range(M):
            rowsum = int(A8[m].astype(np.int64).sum())
            for n in range(N):
                s = sum(int(a) * int(b) for a, b in zip(A8[m].tolist(), biased[n].tolist()))
                assert s - 128 * rowsum == int(ref[m, n])


def test_quantize_weights_exact_group():
    """A row whose groups are exactly representable: s1 = 2^-6 (the largest
    group range is 120 * 2^-6), group 0 holds t in {-56, 0, 64}
    (s2 = 8, z = 7, q = 0, 7, 15) and group 1 holds t in {-3, 0, 12}
    (s2 = 1, z = 3, q = 0, 3, 15)."""
    s1 = 2.0 ** -6
    W = np.zeros((1, 256), dtype=np.float32)
    W[0, 0], W[0, 1], W[0, 2] = -56 * s1, 0.0, 64 * s1
    W[0, 128], W[0, 129], W[0, 130] = -3 * s1, 0.0, 12 * s1
    q, z, s2, s1o = O.quantize_weights(W)
    assert float(s1o[0]) == s1
    assert s2.tolist() == [[8, 1]] and z.tolist() == [[7, 3]]
    assert q[0, :3].tolist() == [0, 7, 15] and q[0, 128:131].tolist() == [0, 3, 15]
    assert (q[0, 3:128] == 7).all() and (q[0, 131:] == 3).all()
    W8 = O.dequant_weights(q, z, s2)
    assert (W8.astype(np.float64) * s1 == W.astype(np.float64)).all()


def test_quantize_weights_bounds_and_error():
    rng = np.random.default_rng(6)
    W = (rng.standard_normal((64, 512)) * 0.02).astype(np.float32)
    W[3] = 0.0
    q, z, s2, s1 = O.quantize_weights(W)
    assert q.max() <= 15 and z.max() <= 15 and s2.min() >= 1 and s2.max() <= 8
    assert float(s1[3]) == 1.0 and not q[3].any() and not z[3].any()
    W8 = O.dequant_weights(q, z, s2).astype(np.float64)
    assert np.abs(W8).max() <= 120
    s1f = s1.astype(np.float64)[:, None]
    s2k = np.repeat(s2.astype(np.float64), 128, axis=1)
    err = np.abs(W.astype(np.float64) - s1f * W8)
    # rounding to the level-2 grid: half a step of s1*s2, plus fp32 slack
    assert (err <= s1f * s2k * (0.5 + 1e-3)).all()
    # the widest group of each row spans nearly the whole int8 range
    g = W8.reshape(64, 4, 128)
    span = (g.max(2) - np.minimum(g.min(2), 0)).max(1)
    assert (span[np.arange(64) != 3] >= 100).all()


# ---------------------------------------------------------------- GEMM
def test_gemm_acc_brute_force():
    rng = np.random.default_rng(7)
    M, N, K = 3, 5, 70
    A8 = rng.integers(-127, 128, (M, K)).astype(np.int8)
    W8 = rng.integers(-120, 121, (N, K)).astype(np.int8)
    acc = O.gemm_acc(A8, W8)
    for m in range(M):
        for n in range(N):
            s = 0
            for k in range(K):
                s += int(A8[m, k]) * int(W8[n, k])
            assert int(acc[m, n]) == s


def test_gemm_closed_forms():
    K = 512
    ones_a = np.ones((4, K), np.int8)
    q = np.ones((8, K), np.uint8)
    z = np.zeros((8, K // 128), np.uint8)
    s2 = np.ones((8, K // 128), np.uint8)
    W8 = O.dequant_weights(q, z, s2)
    assert (O.gemm_acc(ones_a, W8) == K).all()
    # one-hot rows select a column of W8
    rng = np.random.default_rng(8)
    q = rng.integers(0, 16, (8, K)).astype(np.uint8)
    z = rng.integers(0, 16, (8, K // 128)).astype(np.uint8)
    s2 = rng.integers(1, 9, (8, K // 128)).astype(np.uint8)
    W8 = O.dequant_weights(q, z, s2)
    js = [0, 1, 127, 128, 300, 511]
    E = np.zeros((len(js), K), np.int8)
    for i, j in enumerate(js):
        E[i, j] = 1
    acc = O.gemm_acc(E, W8)
    for i, j in enumerate(js):
        assert (acc[i] == W8[:, j].astype(np.int32)).all()
    # linearity and sign flip
    A1 = rng.integers(-60, 61, (4, K)).astype(np.int8)
    A2 = rng.integers(-60, 61, (4, K)).astype(np.int8)
    assert (O.gemm_acc((A1 + A2).astype(np.int8), W8) == O.gemm_acc(A1, W8) + O.gemm_acc(A2, W8)).all()
    assert (O.gemm_acc((-A1).astype(np.int8), W8) == -O.gemm_acc(A1, W8)).all()
    # extreme magnitudes stay exact: 127 * 120 * K
    big_a = np.full((1, 14336), 127, np.int8)
    big_w = np.full((1, 14336), 120, np.int8)
    assert int(O.gemm_acc(big_a, big_w)[0, 0]) == 127 * 120 * 14336


def test_epilogue_within_one_ulp_of_fp64():
    rng = np.random.default_rng(9)
    acc = rng.integers(-(2 ** 24), 2 ** 24, (16, 64)).astype(np.int32)
    sA = rng.uniform(1e-3, 0.25, 16).astype(np.float16)
    s1 = rng.uniform(1e-4, 1e-2, 64).astype(np.float16)
    Y = O.epilogue(acc, sA, s1)
    ref = (acc.astype(np.float64) * sA.astype(np.float64)[:, None] * s1.astype(np.float64)[None, :])
    ref16 = ref.astype(np.float16)
    assert max_ulp_fp16(Y, ref16) <= 1
    # exact cases: powers of two
    acc = np.array([[1, -4, 1024]], np.int32)
    Y = O.epilogue(acc, np.array([0.5], np.float16), np.array([1.0, 0.25, 2.0 ** -10], np.float16))
    assert Y.astype(np.float64).tolist() == [[0.5, -0.5, 0.5]]


def test_w4a8_gemm_matches_fp64_dequantize_then_matmul():
    """Brute force in fp64: dequantize each weight by hand as
    s1 * (q - z) * s2, multiply by A8 * sA and sum; the oracle's fp16 output
    is within 1 ulp of that value rounded to fp16, and its int32 accumulator
    equals the exact sum."""
    rng = np.random.default_rng(10)
    M, N, K = 5, 6, 256
    A = _rand_act(M, K, 11)
    A8, sA, _ = O.quantize_act(A)
    q = rng.integers(0, 16, (N, K)).astype(np.uint8)
    z = rng.integers(0, 16, (N, 2)).astype(np.uint8)
    s2 = rng.integers(1, 9, (N, 2)).astype(np.uint8)
    s1 = rng.uniform(1e-3, 1e-2, N).astype(np.float16)
    Y = O.w4a8_gemm(A8, sA, q, z, s2, s1)
    ref = np.zeros((M, N))
    acc_ref = np.zeros((M, N), dtype=np.int64)
    for n in range(N):
        for k in range(K):
            g = k // 128
            w8 = (int(q[n, k]) - int(z[n, g])) * int(s2[n, g])
            acc_ref[:, n] += A8[:, k].astype(np.int64) * w8
    ref = acc_ref * sA.astype(np.float64)[:, None] * s1.astype(np.float64)[None, :]
    acc = O.gemm_acc(A8, O.dequant_weights(q, z, s2))
    assert (acc == acc_ref).all()
    assert max_ulp_fp16(Y, ref.astype(np.float16)) <= 1


# ---------------------------------------------------------------- pack
def test_pack_hand_positions():
    """Byte positions worked out by hand for N=256, K=384 (3 k-tiles)."""
    N, K = 256, 384
    q = np.zeros((N, K), np.uint8)
    z = np.zeros((N, 3), np.uint8)
    s2 = np.ones((N, 3), np.uint8)
    s1 = np.zeros(N, np.float16)
    # (n=130, k=300): tile (1, 2) -> tile index 5 -> 64 + 5*8320 = 41664;
    # row 2, in-tile k 44 = 8*5 + 4 -> word 5, high nibble of byte 0;
    # word 5 -> ((5//4)*128 + 2)*4 + 5%4 = 521 -> byte 2084.
    q[130, 300] = 0xB
    # (n=1, k=2): tile 0 at 64; row 1, word 0, low nibble of byte 2 -> 64 + 4*4 + 2
    q[1, 2] = 0x6
    # meta of (n=130, group 2): byte 41664 + 8192 + 2; z=3, s2=5 -> 0x43
    z[130, 2], s2[130, 2] = 3, 5
    s1[0], s1[255] = 1.5, -2.0
    blob = O.pack_weights(q, z, s2, s1)
    assert blob.size == 64 + 6 * 8320 + 512
    assert blob[43748] == 0xB0
    assert blob[82] == 0x06
    assert blob[41664 + 8192 + 2] == 0x43
    # every other meta byte is z=0, s2=1 -> 0
    s1_off = 64 + 6 * 8320
    assert int.from_bytes(bytes(blob[32:40]), "little") == s1_off
    assert np.frombuffer(bytes(blob[s1_off:s1_off + 2]), np.float16)[0] == 1.5
    assert np.frombuffer(bytes(blob[s1_off + 510:s1_off + 512]), np.float16)[0] == -2.0
    nz = np.flatnonzero(blob[64:s1_off]) + 64
    assert sorted(nz.tolist()) == [82, 43748, 41664 + 8192 + 2]
    assert bytes(blob[0:4]) == b"W4A8"
    assert O.code_byte_offset(2, 44) == (2084, True)
    assert O.code_byte_offset(1, 2) == (18, False)


def test_pack_roundtrip():
    rng = np.random.default_rng(12)
    N, K = 384, 512
    q = rng.integers(0, 16, (N, K)).astype(np.uint8)
    z = rng.integers(0, 16, (N, K // 128)).astype(np.uint8)
    s2 = rng.integers(1, 9, (N, K // 128)).astype(np.uint8)
    s1 = rng.uniform(1e-3, 1e-2, N).astype(np.float16)
    blob = O.pack_weights(q, z, s2, s1)
    q2, z2, s22, s12, N2, K2 = O.unpack_weights(blob)
    assert (N2, K2) == (N, K)
    assert (q2 == q).all() and (z2 == z).all() and (s22 == s2).all()
    assert (s12.view(np.uint16) == s1.view(np.uint16)).all()
    # a 16-byte vector of a row holds k = 32c .. 32c+31 of that row
    r, c = 77, 2
    off = 64 + (c * 128 + r) * 16
    vec = blob[off:off + 16]
    lo = [int(v) & 0xF for v in vec]
    hi = [int(v) >> 4 for v in vec]
    ks = []
    for jj in range(4):
        ks += [32 * c + 8 * jj + b for b in range(4)] + [32 * c + 8 * jj + 4 + b for b in range(4)]
    vals = []
    for jj in range(4):
        vals += lo[4 * jj:4 * jj + 4] + hi[4 * jj:4 * jj + 4]
    assert vals == q[r, ks].tolist()


# ------------------------------------------------------- 4-bit activations
def test_act4_codes_exact_rational():
    """Dynamic 4-bit codes: sA = fp16(fp32(amax) / 7) and each code is the
    integer nearest to A / sA in exact arithmetic (ties to even), clamped to
    [-7, 7], except where A / sA lies so close to a half-integer that the fp32
    quotient may round across it; rowsum sums the codes."""
    A = _rand_act(5, 256, 21)
    A4, sA, rs = O.quantize_act4(A)
    assert A4.min() >= -7 and A4.max() <= 7 and (rs == A4.astype(np.int64).sum(1)).all()
    n_checked = 0
    for m in range(A.shape[0]):
        amax = max(abs(Fraction(float(v))) for v in A[m])
        assert Fraction(float(np.float16(np.float32(float(amax)) / np.float32(7)))) == Fraction(float(sA[m]))
        s = Fraction(float(sA[m]))
        for k in range(A.shape[1]):
            x = Fraction(float(A[m, k])) / s
            frac = x - (x.numerator // x.denominator)
            if abs(frac - Fraction(1, 2)) < Fraction(1, 10 ** 5):
                continue
            assert int(A4[m, k]) == max(-7, min(7, _nearest_even(x))), (m, k)
            n_checked += 1
    assert n_checked > 1200
    # the outlier channels reach the range ends (the scale is fixed by them)
    assert (np.abs(A4).max(1) == 7).all()


def test_act4_static_codes_exact_rational_with_saturation():
    A = _rand_act(4, 256, 22)
    A[1] *= 30  # an outlier token: many codes saturate under the tensor scale
    s = np.float16(0.5)
    A4, sA, rs = O.quantize_act4_static(A, s)
    assert (sA.view(np.uint16) == np.uint16(s.view(np.uint16))).all()
    assert (rs == A4.astype(np.int64).sum(1)).all()
    S = Fraction(float(s))
    n_checked = n_clamped = 0
    for m in range(A.shape[0]):
        for k in range(A.shape[1]):
            x = Fraction(float(A[m, k])) / S
            frac = x - (x.numerator // x.denominator)
            if abs(frac - Fraction(1, 2)) < Fraction(1, 10 ** 5):
                continue
            want = max(-7, min(7, _nearest_even(x)))
            n_clamped += abs(want) == 7 and abs(x) > Fraction(15, 2)
            assert int(A4[m, k]) == want, (m, k)
            n_checked += 1
    assert n_checked > 900 and n_clamped > 50


def test_act4_constant_zero_rows_and_symmetries():
    c = np.float16(3.5)
    A = np.full((2, 128), c, dtype=np.float16)
    A[1] = 0
    A4, sA, rs = O.quantize_act4(A)
    assert (A4[0] == 7).all() and rs[0] == 7 * 128
    assert sA[0] == np.float16(np.float32(c) / np.float32(7)) and not A4[1].any() and sA[1] == 0
    B = _rand_act(6, 384, 23)
    P4, Ps, _ = O.quantize_act4(B)
    N4, Ns, _ = O.quantize_act4(-B)
    assert (N4 == -P4).all() and (Ns == Ps).all()  # rint is odd, amax even
    Q4, Qs, _ = O.quantize_act4((B.astype(np.float32) * 8).astype(np.float16))
    assert (Q4 == P4).all() and (Qs.astype(np.float32) == Ps.astype(np.float32) * 8).all()


def test_act4_static_reduces_to_dynamic_per_row():
    A = _rand_act(5, 512, 24)
    A4d, sAd, rsd = O.quantize_act4(A)
    for m in range(A.shape[0]):
        A4s, sAs, rss = O.quantize_act4_static(A[m:m + 1], sAd[m])
        assert (A4s[0] == A4d[m]).all() and rss[0] == rsd[m]


def test_act4_pack_hand_bytes_and_full_domain():
    codes = np.array([[1, -1, 7, -7, 0, -8, 3, 4]], dtype=np.int8)
    # byte j: code 2j in bits 0-3, code 2j+1 in bits 4-7 (two's complement)
    assert O.pack_act4(codes).tolist() == [[0xF1, 0x97, 0x80, 0x43]]
    lo, hi = np.meshgrid(np.arange(-8, 8), np.arange(-8, 8), indexing="ij")
    pairs = np.stack([lo.ravel(), hi.ravel()], axis=1).reshape(1, -1).astype(np.int8)
    P = O.pack_act4(pairs)
    assert sorted(P[0].tolist()) == list(range(256))  # a bijection on bytes
    assert (O.unpack_act4(P) == pairs).all()


def test_w4a4_gemm_brute_force():
    """Pure-Python loops on the 4-bit codes and the element-wise dequantized
    weights, epilogue in fp64: the oracle is within 1 fp16 ulp."""
    rng = np.random.default_rng(25)
    M, N, K = 3, 4, 256
    A4, sA, _ = O.quantize_act4(_rand_act(M, K, 26))
    q = rng.integers(0, 16, (N, K)).astype(np.uint8)
    z = rng.integers(0, 16, (N, K // 128)).astype(np.uint8)
    s2 = rng.integers(1, 9, (N, K // 128)).astype(np.uint8)
    s1 = rng.uniform(0.001, 0.01, N).astype(np.float16)
    Y = O.w4a4_gemm(O.pack_act4(A4), sA, q, z, s2, s1)
    for m in range(M):
        for n in range(N):
            acc = sum(int(A4[m, k]) * (int(q[n, k]) - int(z[n, k // 128])) * int(s2[n, k // 128]) for k in range(K))
            ref = np.float16(float(sA[m]) * float(s1[n]) * acc)
            assert max_ulp_fp16(Y[m:m + 1, n:n + 1], np.array([[ref]])) <= 1, (m, n)
    # 4-bit codes are a subset of the 8-bit codes: the 8-bit GEMM fed with them agrees exactly
    assert (Y.view(np.uint16) == O.w4a8_gemm(A4, sA, q, z, s2, s1).view(np.uint16)).all()


# ---------------------------------------------- lookup-table weights (FLUTE)
def _fp16_is_nearest(c: np.float16, exact: Fraction) -> bool:
    """c is an fp16 value nearest to `exact` (ties: even mantissa)."""
    d = abs(Fraction(float(c)) - exact)
    for nb in (np.nextafter(c, np.float16(np.inf)), np.nextafter(c, np.float16(-np.inf))):
        dn = abs(Fraction(float(nb)) - exact)
        if dn < d or (dn == d and int(np.float16(nb).view(np.uint16)) % 2 == 0 and int(c.view(np.uint16)) % 2 == 1):
            return False
    return True


def test_lut_dequant_rounds_the_exact_product_once():
    from w4a8_quantized_gemm_quantize_b200 import inputs as I
    T = I.lut_table()
    q, s = I.lut_codes(4, 256, 31)
    W = O.lut_dequant(q, s, T)
    for n in range(4):
        for k in range(0, 256, 3):
            exact = Fraction(float(T[q[n, k]])) * Fraction(float(s[n, k // 128]))
            assert _fp16_is_nearest(W[n, k], exact), (n, k)
    # a power-of-two scale is exact: W = T[q] * 2^-3
    s8 = np.full((4, 2), np.float16(0.125))
    assert (O.lut_dequant(q, s8, T).astype(np.float64) == T.astype(np.float64)[q] / 8).all()


def test_lut_gemm_brute_force_and_one_hot():
    from w4a8_quantized_gemm_quantize_b200 import inputs as I
    T = I.lut_table()
    M, N, K = 3, 5, 256
    q, s = I.lut_codes(N, K, 32)
    A = _rand_act(M, K, 33)
    W = O.lut_dequant(q, s, T)
    ex = O.lut_gemm_exact(A, q, s, T)
    Y = O.lut_gemm(A, q, s, T)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(A[m, k])) * Fraction(float(W[n, k])) for k in range(K))
            assert abs(Fraction(ex[m, n]) - exact) <= abs(exact) * Fraction(1, 2 ** 40) + Fraction(1, 2 ** 60)
            assert _fp16_is_nearest(Y[m, n], Fraction(ex[m, n]))
    # one-hot rows select a weight column: exact, and exact again in fp16
    A1 = np.zeros((4, K), dtype=np.float16)
    cols = [0, 77, 128, 255]
    for m, j in enumerate(cols):
        A1[m, j] = 1.0
    Y1 = O.lut_gemm(A1, q, s, T)
    assert (Y1.view(np.uint16) == W[:, cols].T.view(np.uint16)).all()


def test_lut_error_bound_covers_fp32_accumulation_orders():
    from w4a8_quantized_gemm_quantize_b200 import inputs as I
    T = I.lut_table()
    M, N, K = 2, 3, 1024
    q, s = I.lut_codes(N, K, 34)
    A = _rand_act(M, K, 35)
    W = O.lut_dequant(q, s, T)
    ex = O.lut_gemm_exact(A, q, s, T)
    bound = O.lut_error_bound(A, W)
    rng = np.random.default_rng(36)
    for m in range(M):
        for n in range(N):
            prods = A[m].astype(np.float32) * W[n].astype(np.float32)  # exact in fp32
            for _ in range(4):
                acc = np.float32(0)
                for p in prods[rng.permutation(K)]:
                    acc = np.float32(acc + p)
                assert abs(float(acc) - ex[m, n]) <= bound[m, n]
    assert (bound > 0).all()


def test_lut_pack_hand_positions_and_roundtrip():
    from w4a8_quantized_gemm_quantize_b200 import inputs as I
    T = I.lut_table()
    N, K = 128, 256
    q = np.zeros((N, K), dtype=np.uint8)
    q[3, 5] = 9    # row 3, k 5: byte j = 2 of vector 0 -> offset (0*128 + 3)*16 + 2 = 50, high nibble
    q[3, 4] = 6    # same byte, low nibble
    q[7, 128 + 37] = 12  # tile kt = 1, k 37: j = 18 -> vector 1, byte 2 -> (128 + 7)*16 + 2 = 2162, high
    s = np.full((N, 2), np.float16(0.25))
    s[3, 1] = np.float16(-1.5)
    blob = O.lut_pack_weights(q, s, T)
    assert O.lut_code_byte_offset(3, 5) == (50, True)
    assert O.lut_code_byte_offset(7, 37) == (2162, True)
    tile1 = 64 + 8448
    assert blob[64 + 50] == (9 << 4) | 6
    assert blob[tile1 + 2162] == 12 << 4
    assert blob[tile1 + 8192 + 2 * 3:tile1 + 8192 + 2 * 3 + 2].view(np.float16)[0] == np.float16(-1.5)
    assert int.from_bytes(bytes(blob[0:4]), "little") == 0x544C3457
    t_off = int.from_bytes(bytes(blob[32:40]), "little")
    assert t_off == 64 + 2 * 8448 and (blob[t_off:t_off + 32].view(np.float16) == T).all()
    q2, s2, T2, N2, K2 = O.lut_unpack_weights(blob)
    assert (q2 == q).all() and (s2 == s).all() and (N2, K2) == (N, K)
    qr, sr = I.lut_codes(256, 384, 37)
    q3, s3, _, _, _ = O.lut_unpack_weights(O.lut_pack_weights(qr, sr, T))
    assert (q3 == qr).all() and (s3.view(np.uint16) == sr.view(np.uint16)).all()


def test_lut_quantize_picks_the_nearest_entry():
    from w4a8_quantized_gemm_quantize_b200 import inputs as I
    T = I.lut_table()
    W = np.random.default_rng(38).standard_normal((3, 256)).astype(np.float32) * np.float32(0.02)
    W[1, :128] = 0  # an all-zero group: scale 1, index of the zero entry
    q, s = O.lut_quantize_weights(W, T)
    tmax = max(abs(Fraction(float(t))) for t in T)
    for n in range(3):
        for g in range(2):
            grp = W[n, 128 * g:128 * (g + 1)]
            am = max(abs(Fraction(float(v))) for v in grp)
            if am == 0:
                assert s[n, g] == np.float16(1)
                assert (T[q[n, 128 * g:128 * (g + 1)]] == 0).all()
                continue
            want = np.float16(np.float32(float(am)) / np.float32(float(tmax)))
            assert s[n, g].view(np.uint16) == want.view(np.uint16)
            for k in range(128 * g, 128 * (g + 1), 5):
                x = Fraction(float(np.float32(W[n, k]) / np.float32(s[n, g])))
                d = [abs(x - Fraction(float(t))) for t in T]
                assert d[q[n, k]] == min(d) and q[n, k] == d.index(min(d)), (n, k)


# ------------------------------------------------ 3-bit lookup-table storage
from w4a8_quantized_gemm_quantize_b200 import inputs as I  # noqa: E402  (seeded generators only)

def test_lut3_planes_hand_computed():
    """Indices q[kk] = kk % 8 on every row: bit c of kk % 8 repeats with
    period 8, so every byte of plane 0 is 0b10101010, of plane 1 0b11001100,
    of plane 2 0b11110000; the scales follow the planes."""
    N, K = 128, 256
    q = np.tile((np.arange(K) % 8).astype(np.uint8), (N, 1))
    s = np.full((N, K // 128), np.float16(0.5))
    T = I.lut3_table()
    blob = O.lut3_pack_weights(q, s, T)
    assert blob.size == O.lut3_packed_bytes(N, K) == 64 + 2 * 6400 + 64
    for kt in range(2):
        base = 64 + kt * 6400
        for c, want in enumerate((0xAA, 0xCC, 0xF0)):
            assert (blob[base + c * 2048:base + (c + 1) * 2048] == want).all()
        assert (blob[base + 6144:base + 6400].view(np.float16) == np.float16(0.5)).all()
    assert int.from_bytes(bytes(blob[0:4]), "little") == O.LUT3_MAGIC
    assert bytes(blob[0:4]) == b"W3LT"
    t_off = int.from_bytes(bytes(blob[32:40]), "little")
    assert t_off == 64 + 2 * 6400
    assert (blob[t_off:t_off + 16].view(np.float16) == T).all() and not blob[t_off + 16:].any()


def test_lut3_single_index_sets_its_bits():
    """One nonzero index (7 = all three bits) at (n, k) sets exactly bit
    k % 128 % 8 of byte k % 128 // 8 in each plane of row n % 128 of tile
    (n // 128, k // 128), and nothing else in the index area."""
    N, K = 256, 384
    for n, k in [(0, 0), (5, 127), (130, 200), (255, 383)]:
        q = np.zeros((N, K), np.uint8)
        q[n, k] = 7
        blob = O.lut3_pack_weights(q, np.zeros((N, K // 128), np.float16), I.lut3_table())
        tile = 64 + ((n // 128) * (K // 128) + k // 128) * 6400
        expect = set()
        for c in range(3):
            off, bit = O.lut3_bit_position(n % 128, k % 128, c)
            assert off == (c * 128 + n % 128) * 16 + (k % 128) // 8 and bit == k % 8
            expect.add((tile + off, bit))
        t_off = int.from_bytes(bytes(blob[32:40]), "little")
        nz = np.flatnonzero(blob[64:t_off]) + 64
        got = {(int(i), b) for i in nz for b in range(8) if (blob[i] >> b) & 1}
        assert got == expect


def test_lut3_round_trip_and_dequant():
    N, K = 256, 640
    q, s = I.lut3_codes(N, K, 3)
    T = I.lut3_table()
    q2, s2, T2, N2, K2 = O.lut3_unpack_weights(O.lut3_pack_weights(q, s, T))
    assert (N2, K2) == (N, K) and np.array_equal(q2, q)
    assert np.array_equal(s2.view(np.uint16), s.view(np.uint16)) and np.array_equal(T2.view(np.uint16), T.view(np.uint16))
    # the 3-bit weights dequantize exactly as the 4-bit path does with an 8-entry table
    W = O.lut_dequant(q, s, T)
    assert np.array_equal(W.astype(np.float64), (T.astype(np.float32)[q] * np.repeat(s.astype(np.float32), 128, axis=1)).astype(np.float16).astype(np.float64))
    # and the nearest-entry quantizer returns 3-bit indices for an 8-entry table
    qq, ss = O.lut_quantize_weights(O.lut_dequant(q, s, T).astype(np.float32), T)
    assert qq.max() < 8
