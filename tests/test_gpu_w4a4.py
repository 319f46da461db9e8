"""GPU parity of the W4A4 path (4-bit activations, "PrefixQuant ..." W4A4KV4
reading) against the CPU oracle, through the C ABI.

Bars: packed 4-bit codes, scales and rowsums bit/byte-exact; int32
accumulators bit-exact; fp16 output within 1 ulp of the oracle's epilogue.
Every token-tile size (16, 32, 64, 128 tokens) and schedule runs, since the
kernel expands the packed activation tile in shared memory per tile size.
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


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def host(t):
    return t.cpu().numpy()


@pytest.fixture(autouse=True)
def _no_device_error():
    w4a8.clear_device_error(DEV)
    yield
    assert w4a8.get_device_error(DEV) == 0


def special_rows(K):
    rows = [np.zeros(K), np.full(K, 3.0), np.full(K, -65504.0), np.full(K, 6e-8), np.linspace(-1, 1, K)]
    return np.stack(rows).astype(np.float16)


# ------------------------------------------------------------ quantizers
@pytest.mark.parametrize("M,K", [(1, 512), (3, 4096), (17, 14336), (5, 65536), (300, 1024), (2, 8)])
def test_w4a4_quantize_bit_exact(M, K):
    A = I.activations(M, K, I.seed_of("t-q4", M, K))
    A = np.concatenate([A, special_rows(K)], axis=0)
    A4, sA, rs = w4a8.w4a4_quantize_act(dev(A))
    torch.cuda.synchronize()
    o4, osA, ors = O.quantize_act4(A)
    assert (host(A4) == O.pack_act4(o4)).all()
    assert (host(sA).view(np.uint16) == osA.view(np.uint16)).all()
    assert (host(rs) == ors).all()


@pytest.mark.parametrize("M,K", [(1, 512), (7, 4096), (3, 14336), (260, 1024)])
@pytest.mark.parametrize("s", [0.25, 2e-3, 0.0])
def test_w4a4_quantize_static_bit_exact(M, K, s):
    """Per-tensor static 4-bit codes (outlier tokens saturate at +-7)."""
    A = np.concatenate([I.activations(M, K, I.seed_of("t-q4s", M, K)), special_rows(K)], axis=0)
    A4, sA, rs = w4a8.w4a4_quantize_act_static(dev(A), torch.tensor([s], dtype=torch.float16, device=DEV))
    torch.cuda.synchronize()
    o4, osA, ors = O.quantize_act4_static(A, np.float16(s))
    assert (host(A4) == O.pack_act4(o4)).all()
    assert (host(sA).view(np.uint16) == osA.view(np.uint16)).all()
    assert (host(rs) == ors).all()


# ------------------------------------------------------------------ GEMM
def check_w4a4(A, q, z, s2, s1, schedules, static_s=None, ws_tail=True):
    """ws_tail: workspace with the scratch tail (large token tiles expand the
    codes once, then the int8 GEMM runs) or without it (the GEMM expands them
    in shared memory for every tile size)."""
    M, K = A.shape
    N = q.shape[0]
    blob = w4a8.pack_weights(dev(q), dev(z), dev(s2), dev(s1))
    if static_s is None:
        A4, sA, rs = w4a8.w4a4_quantize_act(dev(A))
        o4, osA, _ = O.quantize_act4(A)
    else:
        A4, sA, rs = w4a8.w4a4_quantize_act_static(dev(A), torch.tensor([static_s], dtype=torch.float16, device=DEV))
        o4, osA, _ = O.quantize_act4_static(A, np.float16(static_s))
    oacc = O.gemm_acc(o4, O.dequant_weights(q, z, s2))
    # the oracle's W4A4 GEMM is this epilogue of these accumulators; it is
    # called once on a small case to tie the two together
    oY = O.epilogue(oacc, osA, s1)
    if M * N * K <= 1 << 24:
        assert (O.w4a4_gemm(O.pack_act4(o4), osA, q, z, s2, s1).view(np.uint16) == oY.view(np.uint16)).all()
    base = w4a8.workspace_bytes(M, N, K)
    size = w4a8.w4a4_workspace_bytes(M, N, K) if ws_tail else base
    ws = torch.zeros(max(size, 1), dtype=torch.uint8, device=DEV)
    for sched, bm, ctas in schedules:
        acc = w4a8.w4a4_gemm_ex(A4, sA, rs, blob, N, K, acc=torch.empty((M, N), dtype=torch.int32, device=DEV),
                                workspace=ws, schedule=sched, block_m=bm, max_ctas=ctas)
        Y = w4a8.w4a4_gemm_ex(A4, sA, rs, blob, N, K, Y=torch.empty((M, N), dtype=torch.float16, device=DEV),
                              workspace=ws, schedule=sched, block_m=bm, max_ctas=ctas)
        torch.cuda.synchronize()
        ha = host(acc)
        bad = np.argwhere(ha != oacc)
        assert bad.size == 0, (sched, bm, ctas, bad[:5])
        assert max_ulp_fp16(host(Y), oY) <= 1, (sched, bm, ctas)
        assert not host(ws)[:base].any(), "workspace must be left zero-filled (all but the scratch tail)"
    Yd = w4a8.w4a4_gemm(A4, sA, rs, blob, N, K)  # the default entry point
    torch.cuda.synchronize()
    assert max_ulp_fp16(host(Yd), oY) <= 1


SCHEDULES = ([(0, 0, 0), (0, 16, 5), (0, 32, 3)] +
             [(s, bm, c) for s in (1, 2) for bm in (16, 32, 64, 128) for c in (0, 7)] +
             [(3, 16, 0), (3, 32, 0)])


@pytest.mark.parametrize("ws_tail", [True, False], ids=["expand-once", "expand-in-gemm"])
@pytest.mark.parametrize("M", [1, 4, 16, 33, 70, 130])
def test_w4a4_gemm_all_schedules(M, ws_tail):
    N, K = 256, 512
    q, z, s2, s1 = I.uniform_codes(N, K, I.weight_seed("tiny", N, K))
    A = I.activations(M, K, I.seed_of("t-w4a4", M, K))
    check_w4a4(A, q, z, s2, s1, SCHEDULES, ws_tail=ws_tail)


@pytest.mark.parametrize("M,N,K", [(3, 384, 1024), (17, 512, 640), (65, 256, 2048), (129, 384, 512),
                                   (300, 640, 256), (1, 1024, 4096)])
def test_w4a4_gemm_ragged_shapes(M, N, K):
    q, z, s2, s1 = I.uniform_codes(N, K, I.seed_of("t-w4a4g", N, K))
    A = I.activations(M, K, I.seed_of("t-w4a4a", M, K))
    check_w4a4(A, q, z, s2, s1, [(0, 0, 0), (1, 0, 0), (2, 16, 5), (1, 128, 3), (0, 64, 3)])


def test_w4a4_static_scale_through_the_gemm():
    M, N, K = 20, 512, 1024
    q, z, s2, s1 = I.uniform_codes(N, K, I.seed_of("t-w4a4s", N, K))
    A = I.activations(M, K, I.seed_of("t-w4a4sa", M, K))
    s = float(np.float16(float(np.abs(A.astype(np.float32)).max()) / 7 / 4))  # a quarter of the range: saturation
    check_w4a4(A, q, z, s2, s1, [(0, 0, 0), (1, 32, 0)], static_s=s)


@pytest.mark.parametrize("M,lin", [(16, ("gate_up", 28672, 4096)), (1, ("down", 4096, 14336)),
                                   (2048, ("o", 4096, 4096))])
def test_w4a4_full_size(M, lin):
    """Llama-3-8B-shaped linears at decode and prefill token counts, in the
    launch configuration the benchmark uses, compared in full (the prefill
    case both with and without the scratch tail)."""
    name, N, K = lin
    q, z, s2, s1 = O.quantize_weights(I.dense_weights(N, K, 0.02, I.weight_seed("decode", N, K)))
    A = I.activations(M, K, I.activation_seed("decode", M, K))
    check_w4a4(A, q, z, s2, s1, [(0, 0, 0)])
    if M > 32:
        check_w4a4(A, q, z, s2, s1, [(0, 0, 0)], ws_tail=False)
