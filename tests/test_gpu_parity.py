"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on
the same seeded inputs.

Bars: int8 activation codes, fp16 scales, rowsums, weight codes and the
packed blob are bit/byte-exact; the int32 accumulators are bit-exact; the
fp16 output is within 1 fp16 ulp of the oracle (both sides round the same
fp32 epilogue, so it is expected to be exact; the test allows the 1-ulp
tolerance that the specification grants).

The oracle always derives its own codes from the seeded fp32 / fp16 inputs;
nothing it consumes comes from the GPU.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import w4a8_quantized_gemm_quantize_b200 as w4a8
from w4a8_quantized_gemm_quantize_b200 import inputs as I
from oracle import w4a8_oracle as O
from tests._util import max_ulp_fp16

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

DEV = torch.device("cuda:0")


def dev(a: np.ndarray):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def host(t):
    return t.cpu().numpy()


@pytest.fixture(autouse=True)
def _no_device_error():
    w4a8.clear_device_error(DEV)
    yield
    assert w4a8.get_device_error(DEV) == 0


# -------------------------------------------------------- quantize_act
def special_rows(K):
    rows = [np.zeros(K), np.full(K, 3.0), np.full(K, -65504.0), np.full(K, 6e-8)]
    r = np.zeros(K)
    r[K // 3] = 1e-3
    rows.append(r)
    r = np.linspace(-1, 1, K)
    rows.append(r)
    return np.stack(rows).astype(np.float16)


@pytest.mark.parametrize("M,K", [(1, 512), (3, 4096), (17, 14336), (64, 24576), (5, 65536), (300, 1024), (2, 8)])
def test_quantize_act_bit_exact(M, K):
    A = I.activations(M, K, I.seed_of("t-qa", M, K))
    if K >= 8:
        S = special_rows(K)
        A = np.concatenate([A, S], axis=0)
    A8, sA, rs = w4a8.quantize_act(dev(A))
    torch.cuda.synchronize()
    oA8, osA, ors = O.quantize_act(A)
    assert (host(A8) == oA8).all()
    assert (host(sA).view(np.uint16) == osA.view(np.uint16)).all()
    assert (host(rs) == ors).all()


@pytest.mark.parametrize("M,K", [(1, 512), (3, 4096), (17, 14336), (5, 65536), (300, 1024), (2, 8)])
@pytest.mark.parametrize("s", [0.0123, 1e-4, 0.0])
def test_quantize_act_static_bit_exact(M, K, s):
    """Per-tensor static quantization (outlier tokens saturate at +-127)."""
    A = I.activations(M, K, I.seed_of("t-qas", M, K))
    if K >= 8:
        A = np.concatenate([A, special_rows(K)], axis=0)
    sd = torch.tensor([s], dtype=torch.float16, device=DEV)
    A8, sA, rs = w4a8.quantize_act_static(dev(A), sd)
    torch.cuda.synchronize()
    oA8, osA, ors = O.quantize_act_static(A, np.float16(s))
    assert (host(A8) == oA8).all()
    assert (host(sA).view(np.uint16) == osA.view(np.uint16)).all()
    assert (host(rs) == ors).all()


def half_integer_rows(K, scale_exp):
    """Rows whose values over the scale 2^scale_exp are half-integers n + 1/2
    (ties) or one fp16 step above or below one; one element 127 * 2^e sets
    amax, so the dynamic scale is exactly 2^e."""
    n = np.arange(-127, 127, dtype=np.float64)
    ties = ((n + 0.5) * 2.0 ** scale_exp).astype(np.float16)
    up = np.nextafter(ties, np.float16(np.inf))
    down = np.nextafter(ties, np.float16(-np.inf))
    vals = np.concatenate([ties, up, down])
    rows = []
    for shift in range(3):
        r = np.zeros(K, np.float16)
        r[:vals.size] = np.roll(vals, 37 * shift)
        r[K - 1] = np.float16(127 * 2.0 ** scale_exp)
        rows.append(r)
    return np.stack(rows)


@pytest.mark.parametrize("scale_exp", [-4, -9, 3])
def test_quantize_act_half_integer_quotients(scale_exp):
    """Quotients exactly at and one fp16 step beside half-integers: the codes
    follow the IEEE divide and ties-to-even exactly."""
    A = half_integer_rows(4096, scale_exp)
    A8, sA, rs = w4a8.quantize_act(dev(A))
    oA8, osA, ors = O.quantize_act(A)
    torch.cuda.synchronize()
    assert (host(sA).view(np.uint16) == osA.view(np.uint16)).all()
    assert (host(A8) == oA8).all() and (host(rs) == ors).all()
    s = np.array([2.0 ** scale_exp], np.float16)
    sA8, _, srs = w4a8.quantize_act_static(dev(A), dev(s))
    oS8, _, osrs = O.quantize_act_static(A, s[0])
    A4, sA4, rs4 = w4a8.w4a4_quantize_act(dev(A))
    oA4, osA4, ors4 = O.quantize_act4(A)
    torch.cuda.synchronize()
    assert (host(sA8) == oS8).all() and (host(srs) == osrs).all()
    assert (host(A4) == O.pack_act4(oA4)).all() and (host(rs4) == ors4).all()


def test_static_quantization_through_the_gemm():
    """Static activation codes feed the unchanged GEMM: bit-exact int32
    accumulators and Y within 1 ulp of the oracle's static path."""
    M, N, K = 20, 512, 1024
    q, z, s2, s1 = I.uniform_codes(N, K, I.seed_of("t-sg", N, K))
    A = I.activations(M, K, I.seed_of("t-sga", M, K))
    s = np.float16(float(np.abs(A.astype(np.float32)).max()) / 127 / 4)  # a quarter of the tensor range: saturation
    blob = gpu_path_from_codes(q, z, s2, s1)
    A8, sA, rs = w4a8.quantize_act_static(dev(A), torch.tensor([float(s)], dtype=torch.float16, device=DEV))
    acc = w4a8.gemm_debug_acc(A8, rs, blob, N, K)
    Y = w4a8.gemm(A8, sA, rs, blob, N, K)
    torch.cuda.synchronize()
    oA8, osA, _ = O.quantize_act_static(A, s)
    oacc = O.gemm_acc(oA8, O.dequant_weights(q, z, s2))
    assert (host(acc) == oacc).all()
    assert max_ulp_fp16(host(Y), O.epilogue(oacc, osA, s1)) <= 1


def test_quantize_act_empty():
    A = torch.empty((0, 256), dtype=torch.float16, device=DEV)
    A8, sA, rs = w4a8.quantize_act(A)
    assert A8.shape == (0, 256)


# ----------------------------------------------------- quantize_weights
@pytest.mark.parametrize("N,K,std", [(256, 512, 0.02), (384, 4096, 0.015), (128, 14336, 0.02), (130, 128, 1.0)])
def test_quantize_weights_bit_exact(N, K, std):
    W = I.dense_weights(N, K, std, I.seed_of("t-qw", N, K))
    W[0] = 0.0                       # all-zero row: s1 = 1, zero codes
    W[1, :128] = 0.0                 # an all-zero group
    W[2] = np.abs(W[2])              # one-signed rows
    W[3] = -np.abs(W[3])
    q, z, s2, s1 = w4a8.quantize_weights(dev(W))
    torch.cuda.synchronize()
    oq, oz, os2, os1 = O.quantize_weights(W)
    assert (host(q) == oq).all()
    assert (host(z) == oz).all()
    assert (host(s2) == os2).all()
    assert (host(s1).view(np.uint16) == os1.view(np.uint16)).all()


# ----------------------------------------------------------------- pack
@pytest.mark.parametrize("N,K", [(128, 128), (256, 512), (384, 1152)])
def test_pack_byte_exact(N, K):
    q, z, s2, s1 = I.uniform_codes(N, K, I.seed_of("t-pack", N, K))
    blob = w4a8.pack_weights(dev(q), dev(z), dev(s2), dev(s1))
    torch.cuda.synchronize()
    ob = O.pack_weights(q, z, s2, s1)
    assert (host(blob) == ob).all()


def test_pack_reports_codes_out_of_range():
    """A code, zero point or scale outside its range is reported through the
    device error word (the packers keep only the field's low bits)."""
    N, K = 128, 256
    q, z, s2, s1 = I.uniform_codes(N, K, I.seed_of("t-pack-range", N, K))
    for field, bad in (("q", 16), ("z", 16), ("s2", 0), ("s2", 9)):
        qq, zz, ss = q.copy(), z.copy(), s2.copy()
        {"q": qq, "z": zz, "s2": ss}[field][3, 1] = bad
        w4a8.clear_device_error(DEV)
        w4a8.pack_weights(dev(qq), dev(zz), dev(ss), dev(s1))
        assert w4a8.get_device_error(DEV) == w4a8.DEVERR_PACK_RANGE, (field, bad)
    w4a8.clear_device_error(DEV)
    w4a8.pack_weights(dev(q), dev(z), dev(s2), dev(s1))
    assert w4a8.get_device_error(DEV) == 0


# ----------------------------------------------------------------- GEMM
def gpu_path_from_codes(q, z, s2, s1):
    return w4a8.pack_weights(dev(q), dev(z), dev(s2), dev(s1))


GUARD = 4096  # bytes of canary before and after every output buffer
CANARY = 0xA5


class Guarded:
    """A contiguous tensor with canary bytes on both sides (stand-in for a
    memory checker): a write past its first or last element changes them."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((GUARD + n + GUARD,), CANARY, dtype=torch.uint8, device=DEV)
        self.t = self.raw[GUARD:GUARD + n].view(dtype).view(shape)

    def intact(self):
        r = self.raw.cpu().numpy()
        return bool((r[:GUARD] == CANARY).all() and (r[len(r) - GUARD:] == CANARY).all())


def check_gemm(A, q, z, s2, s1, schedules=((0, 0, 0),)):
    """A fp16 host, codes host; runs the GPU path from the same inputs. Every
    buffer the library writes (codes, scales, rowsums, accumulators, Y, the
    workspace) sits between canary regions that must survive each call."""
    M, K = A.shape
    N = q.shape[0]
    blob = gpu_path_from_codes(q, z, s2, s1)
    gA8, gsA, grs = Guarded((M, K), torch.int8), Guarded((M,), torch.float16), Guarded((M,), torch.int32)
    A8, sA, rs = w4a8.quantize_act(dev(A), out=(gA8.t, gsA.t, grs.t))
    oA8, osA, _ = O.quantize_act(A)
    oacc = O.gemm_acc(oA8, O.dequant_weights(q, z, s2))
    oY = O.epilogue(oacc, osA, s1)
    gws = Guarded((w4a8.workspace_bytes(M, N, K),), torch.uint8)
    gws.t.zero_()
    ws = gws.t
    for sched, bm, ctas in schedules:
        gacc, gY = Guarded((M, N), torch.int32), Guarded((M, N), torch.float16)
        acc = w4a8.gemm_ex(A8, None, rs, blob, N, K, acc=gacc.t, workspace=ws, schedule=sched, block_m=bm,
                           max_ctas=ctas)
        Y = w4a8.gemm_ex(A8, sA, rs, blob, N, K, Y=gY.t, workspace=ws, schedule=sched, block_m=bm,
                         max_ctas=ctas)
        torch.cuda.synchronize()
        ha = host(acc)
        bad = np.argwhere(ha != oacc)
        assert bad.size == 0, (sched, bm, ctas, bad[:5], ha[tuple(bad[0])], oacc[tuple(bad[0])])
        assert max_ulp_fp16(host(Y), oY) <= 1, (sched, bm, ctas)
        assert not host(ws).any(), "workspace must be left zero-filled"
        assert gacc.intact() and gY.intact() and gws.intact(), ("write outside a buffer", sched, bm, ctas)
    assert gA8.intact() and gsA.intact() and grs.intact(), "quantizer wrote outside its buffers"
    return oY


def test_guard_regions_see_a_stray_write():
    """The canary check itself: one byte written just past a buffer is seen."""
    g = Guarded((3, 5), torch.float16)
    assert g.intact()
    g.raw[GUARD + 3 * 5 * 2] = 0
    assert not g.intact()


# (schedule, block_m, max_ctas); auto with a small grid mixes stream-K
# remainder tiles with whole tiles
ALL_SCHEDULES = ([(0, 0, 0), (0, 16, 4), (0, 16, 5), (0, 32, 3)] +
                 [(s, bm, c) for s in (1, 2) for bm in (16, 32, 64, 128) for c in (0, 7)] +
                 [(3, 16, 0), (3, 32, 0)])
CLUSTER = [(3, 16, 0), (3, 32, 0)]  # cluster split-K: needs few enough tiles


@pytest.mark.parametrize("M", [1, 16, 33])
def test_gemm_tiny_config_all_schedules(M):
    """The tiny case (K=512, N=256, codes drawn directly) through every
    schedule, token-tile size and a small grid (more work per CTA)."""
    N, K = 256, 512
    q, z, s2, s1 = I.uniform_codes(N, K, I.weight_seed("tiny", N, K))
    A = I.activations(M, K, I.activation_seed("tiny", M, K))
    check_gemm(A, q, z, s2, s1, ALL_SCHEDULES)


@pytest.mark.parametrize("M,N,K", [(3, 384, 1024), (17, 512, 640), (65, 256, 2048), (129, 384, 512),
                                   (200, 128, 384), (1, 1024, 4096), (300, 640, 256), (100, 384, 1024),
                                   (128, 4096, 512)])
def test_gemm_ragged_shapes(M, N, K):
    q, z, s2, s1 = I.uniform_codes(N, K, I.seed_of("t-g", N, K))
    A = I.activations(M, K, I.seed_of("t-a", M, K))
    scheds = [(0, 0, 0), (1, 0, 0), (2, 0, 0), (2, 16, 5), (1, 128, 3), (0, 16, 5), (0, 64, 3)]
    if (N // 128) * -(-M // 16) <= 32:  # one cluster per tile fits
        scheds += CLUSTER
    check_gemm(A, q, z, s2, s1, scheds)


@pytest.mark.parametrize("K", [256, 384, 512, 4096])
def test_gemm_cluster_split_sizes(K):
    """Cluster split-K with every split size the k-block count allows
    (2, 3, 4 CTAs per tile), through the automatic choice and forced."""
    N, M = 512, 5
    q, z, s2, s1 = I.uniform_codes(N, K, I.seed_of("t-cl", N, K))
    A = I.activations(M, K, I.seed_of("t-cla", M, K))
    check_gemm(A, q, z, s2, s1, [(0, 0, 0)] + CLUSTER)


@pytest.mark.parametrize("M,N", [(2500, 384), (3000, 128), (2432, 256)])
def test_gemm_banded_tile_order_ragged_bands(M, N):
    """Activation codes above 32 MiB (K = 14336) switch whole tiles to bands
    of 16 token tiles; 20, 24 and 19 token tiles leave a last band of 4, 8
    and 3. Whole tiles (the automatic choice at 128-token tiles) and a
    reduced grid, so that every CTA walks several bands."""
    K = 14336
    q, z, s2, s1 = I.uniform_codes(N, K, I.seed_of("t-band-w", M, N))
    A = I.activations(M, K, I.seed_of("t-band-a", M, N))
    check_gemm(A, q, z, s2, s1, [(0, 0, 0), (1, 128, 7)])


def test_gemm_cluster_split_needs_two_k_blocks():
    N, K, M = 256, 128, 4
    q, z, s2, s1 = I.uniform_codes(N, K, 12)
    blob = gpu_path_from_codes(q, z, s2, s1)
    A8 = torch.zeros((M, K), dtype=torch.int8, device=DEV)
    rs = torch.zeros((M,), dtype=torch.int32, device=DEV)
    with pytest.raises(w4a8.W4A8Error, match="UNSUPPORTED"):
        w4a8.gemm_ex(A8, None, rs, blob, N, K, acc=torch.empty((M, N), dtype=torch.int32, device=DEV),
                     schedule=3)


def test_gemm_extreme_codes():
    """Largest |W8| = 120 with largest |A8| = 127 over K = 65536: |acc| reaches
    127 * 120 * 65536 = 998,768,640 (no int32 overflow)."""
    N, K, M = 128, 65536, 2
    q = np.zeros((N, K), np.uint8)
    q[::2] = 15
    z = np.zeros((N, K // 128), np.uint8)
    z[1::2] = 15
    s2 = np.full((N, K // 128), 8, np.uint8)
    s1 = np.full(N, 1e-3, np.float16)
    A = np.full((M, K), 1.0, np.float16)
    A[1] = -1.0
    check_gemm(A, q, z, s2, s1, [(0, 0, 0), (2, 0, 0), (3, 16, 0)])


def test_gemm_zero_rows_and_columns():
    N, K, M = 256, 512, 20
    q, z, s2, s1 = I.uniform_codes(N, K, 77)
    q[5] = np.repeat(z[5], 128)      # a weight row that dequantizes to 0
    A = I.activations(M, K, 78)
    A[4] = 0                         # a zero token: sA = 0
    check_gemm(A, q, z, s2, s1, [(0, 0, 0), (2, 16, 0), (3, 32, 0)])


def test_gemm_empty_m():
    N, K = 256, 512
    q, z, s2, s1 = I.uniform_codes(N, K, 5)
    blob = gpu_path_from_codes(q, z, s2, s1)
    A8 = torch.empty((0, K), dtype=torch.int8, device=DEV)
    sA = torch.empty((0,), dtype=torch.float16, device=DEV)
    rs = torch.empty((0,), dtype=torch.int32, device=DEV)
    Y = w4a8.gemm(A8, sA, rs, blob, N, K)
    assert Y.shape == (0, N)


def test_gemm_without_workspace_uses_whole_tiles():
    N, K, M = 512, 1024, 8
    q, z, s2, s1 = I.uniform_codes(N, K, 9)
    A = I.activations(M, K, 10)
    blob = gpu_path_from_codes(q, z, s2, s1)
    A8, sA, rs = w4a8.quantize_act(dev(A))
    empty_ws = torch.zeros(16, dtype=torch.uint8, device=DEV)
    Y = w4a8.gemm(A8, sA, rs, blob, N, K, workspace=empty_ws)
    oA8, osA, _ = O.quantize_act(A)
    oY = O.w4a8_gemm(oA8, osA, q, z, s2, s1)
    torch.cuda.synchronize()
    assert max_ulp_fp16(host(Y), oY) <= 1


def test_gemm_split_k_requires_workspace():
    N, K, M = 256, 512, 4
    q, z, s2, s1 = I.uniform_codes(N, K, 11)
    blob = gpu_path_from_codes(q, z, s2, s1)
    A8 = torch.zeros((M, K), dtype=torch.int8, device=DEV)
    rs = torch.zeros((M,), dtype=torch.int32, device=DEV)
    with pytest.raises(w4a8.W4A8Error, match="WORKSPACE"):
        w4a8.gemm_ex(A8, None, rs, blob, N, K, acc=torch.empty((M, N), dtype=torch.int32, device=DEV),
                     workspace=torch.zeros(16, dtype=torch.uint8, device=DEV), schedule=2)


# ------------------------------------------- full-size workload checks
_W_CACHE = {}


def _weights(workload, N, K):
    """The seeded fp32 weights of one layer and their GPU blob (and codes),
    kept for the next case of the same layer (cases are ordered by layer)."""
    key = (workload, N, K)
    if key not in _W_CACHE:
        _W_CACHE.clear()
        torch.cuda.empty_cache()
        wl = I.WORKLOADS[workload]
        W = I.dense_weights(N, K, wl.weight_std, I.weight_seed(workload, N, K))
        Wd = dev(W)
        q, z, s2, s1 = w4a8.quantize_weights(Wd)
        del Wd
        blob = w4a8.pack_weights(q, z, s2, s1)
        _W_CACHE[key] = (W, q, z, s2, s1, blob)
    return _W_CACHE[key]


def _full_size_case(workload, lin, M, n_random_cols=64):
    """Runs the GPU path end to end from the seeded fp32 weights and fp16
    activations at full size (the launch configuration the benchmark uses)
    and compares every token against the oracle on sampled output channels:
    two whole 128-channel tiles plus random channels. The oracle quantizes
    only the weight rows it needs (rows are independent)."""
    name, N, K = lin
    W, q, z, s2, s1, blob = _weights(workload, N, K)
    A = I.activations(M, K, I.activation_seed(workload, M, K))
    A8, sA, rs = w4a8.quantize_act(dev(A))
    ws = torch.zeros(w4a8.workspace_bytes(M, N, K), dtype=torch.uint8, device=DEV)
    Y = w4a8.gemm(A8, sA, rs, blob, N, K, workspace=ws)
    acc = w4a8.gemm_debug_acc(A8, rs, blob, N, K, workspace=ws)
    torch.cuda.synchronize()
    # activations: full comparison
    oA8, osA, ors = O.quantize_act(A)
    assert (host(A8) == oA8).all() and (host(sA).view(np.uint16) == osA.view(np.uint16)).all()
    assert (host(rs) == ors).all()
    # sampled output channels
    rng = np.random.default_rng(I.seed_of("cols", workload, N, K, M))
    nt = N // 128
    tiles = [0, int(rng.integers(1, nt))]
    cols = np.unique(np.concatenate([np.arange(t * 128, t * 128 + 128) for t in tiles] +
                                    [rng.choice(N, n_random_cols, replace=False)]))
    ct = torch.from_numpy(cols).to(DEV)
    oq, oz, os2, os1 = O.quantize_weights(W[cols])
    assert (host(q[ct]) == oq).all() and (host(z[ct]) == oz).all()
    assert (host(s2[ct]) == os2).all() and (host(s1[ct]).view(np.uint16) == os1.view(np.uint16)).all()
    oacc = O.gemm_acc(oA8, O.dequant_weights(oq, oz, os2))
    oY = O.epilogue(oacc, osA, os1)
    assert (host(acc[:, ct]) == oacc).all()
    assert max_ulp_fp16(host(Y[:, ct]), oY) <= 1
    # the packed tiles of one whole n-tile, byte for byte
    t = tiles[0]
    KT = K // 128
    sub = O.pack_weights(*O.quantize_weights(W[t * 128:(t + 1) * 128]))
    hb = host(blob[64 + t * KT * 8320:64 + (t + 1) * KT * 8320])
    assert (hb == sub[64:64 + KT * 8320]).all()
    assert not ws.any().item()


# Every (M, layer) case of the four dense-weight workloads (56 GEMMs; the tiny
# case is compared in full above), ordered by layer so that each layer's
# weights are generated once.
FULL_SIZE_CASES = [(wl, lin, M) for wl in ("decode", "serving", "prefill", "qwen72b")
                   for lin in I.WORKLOADS[wl].linears for M in I.WORKLOADS[wl].ms]


@pytest.mark.parametrize("workload,lin,M", FULL_SIZE_CASES, ids=lambda v: v[0] if isinstance(v, tuple) else str(v))
def test_full_size(workload, lin, M):
    _full_size_case(workload, lin, M)
