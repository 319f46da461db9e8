"""GPU parity of the 4-bit KV cache and decode attention over it against the
CPU oracle (oracle/kv4_oracle.py), through the C ABI.

Bars: codes and parameter words bit-exact (the quantizer's integer
decisions are taken in fp32 with IEEE divides on both sides); attention
output within half an fp16 ulp of the exact result plus the oracle's fp32
evaluation bound; repeated launches bit-identical (the chunk merge runs in
a fixed order), whatever the workspace held before.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import w4a8_quantized_gemm_quantize_b200 as w4a8
from w4a8_quantized_gemm_quantize_b200 import inputs as I
from oracle import kv4_oracle as KV

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

DEV = torch.device("cuda:0")
SCALE = float(np.float32(1.0 / np.sqrt(128.0)))


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def host(t):
    return t.cpu().numpy()


@pytest.fixture(autouse=True)
def _no_device_error():
    w4a8.clear_device_error(DEV)
    yield
    assert w4a8.get_device_error(DEV) == 0


def words(s, z):
    return KV.kv_params(s, z).view(np.uint32)[..., 0]


def special_vectors():
    rows = [np.zeros(128), np.full(128, 3.0), np.full(128, -3.0), np.full(128, 65504.0),
            np.full(128, 6e-8), np.linspace(-1, 1, 128), np.linspace(0.5, 2, 128), -np.linspace(0.5, 2, 128)]
    return np.stack(rows).astype(np.float16)


@pytest.mark.parametrize("n", [1, 7, 1000, 40000])
def test_kv4_quantize_bit_exact(n):
    X = np.concatenate([I.kv_vectors(1, 1, n, 128, I.seed_of("t-kvq", n))[0, 0], special_vectors()])
    codes, params = w4a8.kv4_quantize(dev(X))
    torch.cuda.synchronize()
    oc, os_, oz = KV.quantize_kv(X)
    assert (host(codes) == KV.pack_kv(oc)).all()
    assert (host(params).view(np.uint32) == words(os_, oz)).all()


def test_kv4_append_places_the_new_token():
    B, Hkv, Lmax = 5, 4, 64
    kc = torch.zeros((B, Hkv, Lmax, 64), dtype=torch.uint8, device=DEV)
    kp = torch.zeros((B, Hkv, Lmax), dtype=torch.int32, device=DEV)
    vc, vp = torch.zeros_like(kc), torch.zeros_like(kp)
    K = I.kv_vectors(B, Hkv, 1, 128, 5)[:, :, 0]
    V = I.kv_vectors(B, Hkv, 1, 128, 6, outlier_scale=1.0)[:, :, 0]
    pos = np.array([0, 3, 63, 17, 1], np.int32)
    w4a8.kv4_append(dev(K), dev(V), dev(pos), kc, kp, vc, vp)
    torch.cuda.synchronize()
    hkc, hkp, hvc, hvp = host(kc), host(kp).view(np.uint32), host(vc), host(vp).view(np.uint32)
    okc, oks, okz = KV.quantize_kv(K)
    ovc, ovs, ovz = KV.quantize_kv(V)
    mask = np.zeros((B, Hkv, Lmax), bool)
    for b in range(B):
        mask[b, :, pos[b]] = True
        assert (hkc[b, :, pos[b]] == KV.pack_kv(okc[b])).all() and (hvc[b, :, pos[b]] == KV.pack_kv(ovc[b])).all()
        assert (hkp[b, :, pos[b]] == words(oks[b], okz[b])).all()
        assert (hvp[b, :, pos[b]] == words(ovs[b], ovz[b])).all()
    assert not hkc[~mask].any() and not hkp[~mask].any() and not hvc[~mask].any() and not hvp[~mask].any()


def make_cache(B, Hq, Hkv, Lmax, seed):
    K = I.kv_vectors(B, Hkv, Lmax, 128, seed)
    V = I.kv_vectors(B, Hkv, Lmax, 128, seed + 1, outlier_scale=1.0)
    q = I.kv_queries(B, Hq, 128, seed + 2)
    kc, ks, kz = KV.quantize_kv(K)
    vc, vs, vz = KV.quantize_kv(V)
    return q, KV.pack_kv(kc), KV.kv_params(ks, kz), KV.pack_kv(vc), KV.kv_params(vs, vz)


def run(q, kc, kp, vc, vp, lens, ws=None):
    B, Hq, _ = q.shape
    Hkv, Lmax = kc.shape[1], kc.shape[2]
    if ws is None:
        ws = torch.zeros(w4a8.kv4_workspace_bytes(B, Hq, Hkv, Lmax), dtype=torch.uint8, device=DEV)
    Y = w4a8.kv4_attention_decode(dev(q), dev(kc), dev(kp.view(np.int32)[..., 0]), dev(vc),
                                  dev(vp.view(np.int32)[..., 0]), dev(lens), SCALE, workspace=ws)
    torch.cuda.synchronize()
    return host(Y), ws


def check(Y, q, kc, kp, vc, vp, lens, heads=None):
    o = KV.attention_decode_exact(q, kc, kp, vc, vp, lens, SCALE)
    E = KV.attention_error_bound(q, kc, kp, vc, vp, lens, SCALE)
    mag = np.abs(o) + E
    ulp = np.spacing(np.maximum(mag, 6.1e-05).astype(np.float16)).astype(np.float64)
    err = np.abs(Y.astype(np.float64) - o)
    assert (err <= 0.5 * ulp + E).all(), float((err / (0.5 * ulp + E)).max())


@pytest.mark.parametrize("Hq,Hkv", [(4, 2), (4, 4), (8, 2), (12, 4), (16, 2), (32, 8)])
@pytest.mark.parametrize("lens", [[300, 77, 1], [1, 256, 257], [0, 299, 300]])
def test_kv4_attention_within_the_bound(Hq, Hkv, lens):
    lens = np.array(lens, np.int32)
    q, kc, kp, vc, vp = make_cache(3, Hq, Hkv, 300, I.seed_of("t-kva", Hq, Hkv))
    Y, ws = run(q, kc, kp, vc, vp, lens)
    check(Y, q, kc, kp, vc, vp, lens)
    # a workspace full of garbage gives the same bits
    ws.fill_(0xA7)
    Y2, _ = run(q, kc, kp, vc, vp, lens, ws)
    assert np.array_equal(Y.view(np.uint16), Y2.view(np.uint16))


def test_kv4_attention_padding_is_not_read():
    q, kc, kp, vc, vp = make_cache(2, 8, 2, 520, 77)
    lens = np.array([300, 513], np.int32)
    Y1, _ = run(q, kc, kp, vc, vp, lens)
    for b, L in enumerate(lens):
        kc[b, :, L:] = 0xFF
        vc[b, :, L:] = 0xA5
        kp[b, :, L:] = np.float16(np.inf)
        vp[b, :, L:] = np.float16(np.nan)
    Y2, _ = run(q, kc, kp, vc, vp, lens)
    assert np.array_equal(Y1.view(np.uint16), Y2.view(np.uint16))


def test_kv4_attention_full_size_decode():
    """Llama-3-8B attention (32 query heads on 8 kv heads), 16 sequences of
    2048..4096 cached tokens, in full on sampled heads."""
    wl = I.KV_WORKLOADS["kv-decode"]
    Hq, Hkv, _ = wl.heads
    q, kc, kp, vc, vp = make_cache(wl.batch, Hq, Hkv, wl.max_len, I.seed_of("t-kvfull"))
    lens = I.kv_seq_lens(wl, I.seed_of("t-kvlens"))
    Y, _ = run(q, kc, kp, vc, vp, lens)
    rng = np.random.default_rng(3)
    for b in rng.choice(wl.batch, 4, replace=False):
        sl = slice(b, b + 1)
        check(Y[sl], q[sl], kc[sl], kp[sl], vc[sl], vp[sl], lens[sl])


def test_kv4_repeated_launches_bit_identical():
    q, kc, kp, vc, vp = make_cache(4, 32, 8, 1500, 99)
    lens = np.array([1500, 1, 700, 1024], np.int32)
    Y0, ws = run(q, kc, kp, vc, vp, lens)
    args = (dev(q), dev(kc), dev(kp.view(np.int32)[..., 0]), dev(vc), dev(vp.view(np.int32)[..., 0]), dev(lens))
    ref = dev(Y0).view(torch.int16)
    bad = torch.zeros((), dtype=torch.int64, device=DEV)
    outs = [torch.empty_like(ref).view(torch.float16) for _ in range(2)]
    for _ in range(500):
        for o in outs:
            w4a8.kv4_attention_decode(*args, SCALE, out=o, workspace=ws)
        for o in outs:
            bad += (o.view(torch.int16) != ref).any()
    torch.cuda.synchronize()
    assert int(bad) == 0


def test_kv4_length_out_of_range_is_clamped_and_reported():
    q, kc, kp, vc, vp = make_cache(2, 4, 2, 64, 55)
    Y_ok, _ = run(q, kc, kp, vc, vp, np.array([64, 10], np.int32))
    Y, _ = run(q, kc, kp, vc, vp, np.array([1000, 10], np.int32))
    assert w4a8.get_device_error(DEV) == 7
    w4a8.clear_device_error(DEV)
    assert np.array_equal(Y.view(np.uint16), Y_ok.view(np.uint16))


def test_kv4_decode_flow_quantize_append_attend():
    """The decode flow through the public calls: the cache of L tokens
    quantized on the GPU, the new token appended at position L, attention
    over L + 1 tokens; the oracle quantizes the same fp16 vectors itself."""
    B, Hq, Hkv, Lmax = 3, 8, 2, 400
    K = I.kv_vectors(B, Hkv, Lmax, 128, 301)
    V = I.kv_vectors(B, Hkv, Lmax, 128, 302, outlier_scale=1.0)
    q = I.kv_queries(B, Hq, 128, 303)
    L = np.array([399, 256, 1], np.int32)       # tokens already cached
    kc, kp = w4a8.kv4_quantize(dev(K))
    vc, vp = w4a8.kv4_quantize(dev(V))
    newK = np.ascontiguousarray(K[np.arange(B), :, L])   # the token at position L of each sequence
    newV = np.ascontiguousarray(V[np.arange(B), :, L])
    # positions >= L hold stale vectors until appended: overwrite position L with garbage first
    bi = torch.arange(B, device=DEV)
    li = torch.from_numpy(L).to(DEV).long()
    kc[bi, :, li] = 0xFF
    vp[bi, :, li] = -1
    w4a8.kv4_append(dev(newK), dev(newV), dev(L), kc, kp, vc, vp)
    lens = L + 1
    ws = torch.zeros(w4a8.kv4_workspace_bytes(B, Hq, Hkv, Lmax), dtype=torch.uint8, device=DEV)
    Y = w4a8.kv4_attention_decode(dev(q), kc, kp, vc, vp, dev(lens), SCALE, workspace=ws)
    torch.cuda.synchronize()
    okc, oks, okz = KV.quantize_kv(K)
    ovc, ovs, ovz = KV.quantize_kv(V)
    okc, okp, ovc, ovp = KV.pack_kv(okc), KV.kv_params(oks, okz), KV.pack_kv(ovc), KV.kv_params(ovs, ovz)
    for b in range(B):  # the cached prefix and the appended token, byte for byte
        n = lens[b]
        assert (host(kc)[b, :, :n] == okc[b, :, :n]).all() and (host(vc)[b, :, :n] == ovc[b, :, :n]).all()
        assert (host(kp).view(np.uint32)[b, :, :n] == okp.view(np.uint32)[b, :, :n, 0]).all()
        assert (host(vp).view(np.uint32)[b, :, :n] == ovp.view(np.uint32)[b, :, :n, 0]).all()
    check(host(Y), q, okc, okp, ovc, ovp, lens)
