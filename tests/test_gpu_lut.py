"""GPU parity of the lookup-table weight-only GEMM ("Fast Matrix
Multiplications for Lookup Table-Quantized LLMs", FLUTE reading) against the
CPU oracle, through the C ABI.

Bars: the packed blob byte-exact; one-hot activation rows reproduce the
dequantized weights bit for bit (a single exact product per output, so any
wrong table entry, scale or index shows); for general activations the fp32
sums within the fp32 accumulation bound of the exact sum, and the fp16
output within half an fp16 ulp plus that bound. Every schedule and both
token-tile sizes run.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import w4a8_quantized_gemm_quantize_b200 as w4a8
from w4a8_quantized_gemm_quantize_b200 import inputs as I
from oracle import w4a8_oracle as O

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

DEV = torch.device("cuda:0")
T = I.lut_table()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def host(t):
    return t.cpu().numpy()


@pytest.fixture(autouse=True)
def _no_device_error():
    w4a8.clear_device_error(DEV)
    yield
    assert w4a8.get_device_error(DEV) == 0


def blob_of(q, s):
    return w4a8.lut_pack_weights(dev(q), dev(s), dev(T))


@pytest.mark.parametrize("N,K", [(128, 128), (256, 640), (384, 4096)])
def test_lut_pack_byte_exact(N, K):
    q, s = I.lut_codes(N, K, I.seed_of("t-lp", N, K))
    b = blob_of(q, s)
    torch.cuda.synchronize()
    assert (host(b) == O.lut_pack_weights(q, s, T)).all()


def test_lut_pack_reports_indices_above_15():
    N, K = 128, 256
    q, s = I.lut_codes(N, K, I.seed_of("t-lr", N, K))
    bad = q.copy()
    bad[9, 17] = 16
    w4a8.clear_device_error(DEV)
    blob_of(bad, s)
    assert w4a8.get_device_error(DEV) == w4a8.DEVERR_PACK_RANGE
    w4a8.clear_device_error(DEV)
    blob_of(q, s)
    assert w4a8.get_device_error(DEV) == 0


SCHEDULES = ([(0, 0, 0), (0, 16, 5), (0, 32, 3)] + [(s, bm, c) for s in (1, 2) for bm in (16, 32) for c in (0, 7)] +
             [(3, 16, 0), (3, 32, 0)])


def run(A, blob, N, K, sched, bm, ctas, ws):
    M = A.shape[0]
    acc = w4a8.lut_gemm_ex(dev(A), blob, N, K, acc=torch.empty((M, N), dtype=torch.float32, device=DEV),
                           workspace=ws, schedule=sched, block_m=bm, max_ctas=ctas)
    Y = w4a8.lut_gemm_ex(dev(A), blob, N, K, Y=torch.empty((M, N), dtype=torch.float16, device=DEV),
                         workspace=ws, schedule=sched, block_m=bm, max_ctas=ctas)
    torch.cuda.synchronize()
    return host(acc), host(Y)


@pytest.mark.parametrize("M", [1, 16, 32, 48])
def test_lut_one_hot_rows_select_weights_bit_exactly(M):
    """A[m] = e_{j_m}: every output is one exact product W[n, j_m], in fp32
    and again after rounding to fp16 (W is fp16)."""
    N, K = 256, 512
    q, s = I.lut_codes(N, K, I.seed_of("t-l1", N, K))
    W = O.lut_dequant(q, s, T)
    rng = np.random.default_rng(I.seed_of("t-l1c", M))
    cols = rng.choice(K, size=M, replace=False)
    A = np.zeros((M, K), dtype=np.float16)
    A[np.arange(M), cols] = 1.0
    blob = blob_of(q, s)
    ws = torch.zeros(w4a8.workspace_bytes(M, N, K), dtype=torch.uint8, device=DEV)
    want = W[:, cols].T
    for sched, bm, ctas in SCHEDULES:
        acc, Y = run(A, blob, N, K, sched, bm, ctas, ws)
        assert (acc == want.astype(np.float32)).all(), (sched, bm, ctas)
        assert (Y.view(np.uint16) == want.view(np.uint16)).all(), (sched, bm, ctas)
        assert not host(ws).any()


def check_bound(A, q, s, acc, Y):
    W = O.lut_dequant(q, s, T)
    ex = O.lut_gemm_exact(A, q, s, T)
    E = O.lut_error_bound(A, W)
    assert (np.abs(acc.astype(np.float64) - ex) <= E).all()
    # |Y - exact| <= |Y - acc| + |acc - exact|: half an fp16 ulp of a value
    # no larger than |exact| + E, plus E
    mag = np.abs(ex) + E
    ulp = np.spacing(np.maximum(mag, 6.1e-05).astype(np.float16)).astype(np.float64)
    assert (np.abs(Y.astype(np.float64) - ex) <= 0.5 * ulp + E).all()


@pytest.mark.parametrize("M,N,K", [(1, 256, 512), (16, 384, 1024), (33, 256, 640), (100, 512, 256)])
def test_lut_gemm_within_the_fp32_bound_all_schedules(M, N, K):
    q, s = I.lut_codes(N, K, I.seed_of("t-lg", N, K))
    A = I.activations(M, K, I.seed_of("t-lga", M, K))
    blob = blob_of(q, s)
    ws = torch.zeros(w4a8.workspace_bytes(M, N, K), dtype=torch.uint8, device=DEV)
    for sched, bm, ctas in SCHEDULES:
        acc, Y = run(A, blob, N, K, sched, bm, ctas, ws)
        check_bound(A, q, s, acc, Y)
        assert not host(ws).any(), (sched, bm, ctas)
    Yd = w4a8.lut_gemm(dev(A), blob, N, K)  # the default entry point
    torch.cuda.synchronize()
    check_bound(A, q, s, acc, host(Yd))


@pytest.mark.parametrize("M,lin", [(16, ("gate_up", 28672, 4096)), (1, ("down", 4096, 14336)),
                                   (32, ("qkv", 6144, 4096))])
def test_lut_full_size_decode(M, lin):
    """Llama-3-8B-shaped linears at decode token counts in the benchmark's
    launch configuration, compared in full."""
    name, N, K = lin
    q, s = I.lut_codes(N, K, I.weight_seed("decode-lut", N, K))
    A = I.activations(M, K, I.activation_seed("decode", M, K))
    blob = blob_of(q, s)
    ws = torch.zeros(w4a8.workspace_bytes(M, N, K), dtype=torch.uint8, device=DEV)
    acc, Y = run(A, blob, N, K, 0, 0, 0, ws)
    check_bound(A, q, s, acc, Y)
