"""GPU parity of the 3-bit lookup-table GEMM ("Fast Matrix Multiplications
for Lookup Table-Quantized LLMs", widths that do not divide a byte) against
the CPU oracle, through the C ABI.

Bars as for the 4-bit table: the blob byte-exact; one-hot activation rows
reproduce the dequantized weights bit for bit; general activations within
the fp32 accumulation bound, Y within half an fp16 ulp plus it; every
schedule and both token-tile sizes.
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
T = I.lut3_table()


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
    return w4a8.lut3_pack_weights(dev(q), dev(s), dev(T))


@pytest.mark.parametrize("N,K", [(128, 128), (256, 640), (384, 4096)])
def test_lut3_pack_byte_exact(N, K):
    q, s = I.lut3_codes(N, K, I.seed_of("t-l3p", N, K))
    b = blob_of(q, s)
    torch.cuda.synchronize()
    assert (host(b) == O.lut3_pack_weights(q, s, T)).all()


def test_lut3_pack_reports_indices_above_7():
    """Only bits 0-2 of an index are packed: an index of 8..15 (a 4-bit index
    given to the 3-bit packer) is reported through the device error word."""
    N, K = 128, 256
    q, s = I.lut3_codes(N, K, I.seed_of("t-l3r", N, K))
    bad = q.copy()
    bad[7, 100] = 8
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
    acc = w4a8.lut3_gemm_ex(dev(A), blob, N, K, acc=torch.empty((M, N), dtype=torch.float32, device=DEV),
                            workspace=ws, schedule=sched, block_m=bm, max_ctas=ctas)
    Y = w4a8.lut3_gemm_ex(dev(A), blob, N, K, Y=torch.empty((M, N), dtype=torch.float16, device=DEV),
                          workspace=ws, schedule=sched, block_m=bm, max_ctas=ctas)
    torch.cuda.synchronize()
    return host(acc), host(Y)


@pytest.mark.parametrize("M", [1, 16, 32, 48])
def test_lut3_one_hot_rows_select_weights_bit_exactly(M):
    N, K = 256, 512
    q, s = I.lut3_codes(N, K, I.seed_of("t-l31", N, K))
    W = O.lut_dequant(q, s, T)
    cols = np.random.default_rng(I.seed_of("t-l31c", M)).choice(K, size=M, replace=False)
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
    mag = np.abs(ex) + E
    ulp = np.spacing(np.maximum(mag, 6.1e-05).astype(np.float16)).astype(np.float64)
    assert (np.abs(Y.astype(np.float64) - ex) <= 0.5 * ulp + E).all()


@pytest.mark.parametrize("M,N,K", [(1, 256, 512), (16, 384, 1024), (33, 256, 640), (100, 512, 256)])
def test_lut3_gemm_within_the_fp32_bound_all_schedules(M, N, K):
    q, s = I.lut3_codes(N, K, I.seed_of("t-l3g", N, K))
    A = I.activations(M, K, I.seed_of("t-l3ga", M, K))
    blob = blob_of(q, s)
    ws = torch.zeros(w4a8.workspace_bytes(M, N, K), dtype=torch.uint8, device=DEV)
    for sched, bm, ctas in SCHEDULES:
        acc, Y = run(A, blob, N, K, sched, bm, ctas, ws)
        check_bound(A, q, s, acc, Y)
        assert not host(ws).any(), (sched, bm, ctas)
    Yd = w4a8.lut3_gemm(dev(A), blob, N, K)
    torch.cuda.synchronize()
    check_bound(A, q, s, acc, host(Yd))


@pytest.mark.parametrize("M,lin", [(16, ("gate_up", 28672, 4096)), (1, ("down", 4096, 14336))])
def test_lut3_full_size_decode(M, lin):
    name, N, K = lin
    q, s = I.lut3_codes(N, K, I.weight_seed("decode-lut3", N, K))
    A = I.activations(M, K, I.activation_seed("decode", M, K))
    blob = blob_of(q, s)
    ws = torch.zeros(w4a8.workspace_bytes(M, N, K), dtype=torch.uint8, device=DEV)
    acc, Y = run(A, blob, N, K, 0, 0, 0, ws)
    check_bound(A, q, s, acc, Y)
