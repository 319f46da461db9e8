"""Repeated launches stay exact.

The GEMM kernel hands its ring slots (weight and activation tiles in shared
memory, dequantized weights in tensor memory, accumulators) from warp to warp
through mbarrier phase parity. A slot handed over at the wrong phase shows up
as one wrong chunk of the sum in a few launches out of thousands, not in any
single launch. So each case checks one launch against the oracle on sampled
output channels, then repeats the launch thousands of times, back to back on
one stream as the benchmark issues them (consecutive launches overlap through
programmatic dependent launch), and requires every repeat to agree: bit for
bit with the first on the int32 paths (W4A8, W4A4), and within the fp32
accumulation bound of the oracle's exact sum on the sampled channels for the
lookup-table GEMM, whose fp32 sums depend on the order in which the tensor
pipe runs the two MMA issuers' chunks.
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
REPEATS = 2500  # x 4 launches per case


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def host(t):
    return t.cpu().numpy()


@pytest.fixture(autouse=True)
def _no_device_error():
    w4a8.clear_device_error(DEV)
    yield
    assert w4a8.get_device_error(DEV) == 0


def sampled_cols(N, seed):
    rng = np.random.default_rng(seed)
    tiles = [0, int(rng.integers(1, N // 128))] if N > 128 else [0]
    return np.unique(np.concatenate([np.arange(t * 128, t * 128 + 128) for t in tiles] +
                                    [rng.choice(N, min(64, N), replace=False)]))


def repeat_exact(launch_y, launch_acc, Y0, acc0):
    """Launches Y, acc, Y, acc back to back REPEATS times; counts the launches
    whose output differs from the first launch's in any bit."""
    Ys = [torch.empty_like(Y0) for _ in range(2)]
    accs = [torch.empty_like(acc0) for _ in range(2)]
    y_ref, a_ref = Y0.view(torch.int16), acc0
    bad = torch.zeros(2, dtype=torch.int64, device=DEV)
    for _ in range(REPEATS):
        for i in range(2):
            launch_y(Ys[i])
            launch_acc(accs[i])
        for i in range(2):
            bad[0] += (Ys[i].view(torch.int16) != y_ref).any()
            bad[1] += (accs[i] != a_ref).any()
    torch.cuda.synchronize()
    return host(bad).tolist()


W4A8_CASES = [
    ("gate_up", 16, 28672, 4096),   # 16-token tiles, stream-K split plus whole tiles per CTA
    ("qkv", 8, 6144, 4096),         # 16-token tiles, cluster split-K
    ("o-72b", 1, 8192, 8192),       # cluster split-K, one tile per cluster
    ("down", 32, 4096, 14336),      # 32-token tiles
    ("o", 64, 4096, 4096),          # 64-token tiles
    ("o", 256, 4096, 4096),         # 128-token tiles
]


@pytest.mark.parametrize("name,M,N,K", W4A8_CASES, ids=[f"{c[0]}-M{c[1]}" for c in W4A8_CASES])
def test_w4a8_repeated_launches_bit_identical(name, M, N, K):
    q, z, s2, s1 = I.uniform_codes(N, K, I.seed_of("t-rep-w", N, K))
    A = I.activations(M, K, I.seed_of("t-rep-a", M, K))
    blob = w4a8.pack_weights(dev(q), dev(z), dev(s2), dev(s1))
    A8, sA, rs = w4a8.quantize_act(dev(A))
    ws = torch.zeros(w4a8.workspace_bytes(M, N, K), dtype=torch.uint8, device=DEV)
    Y0 = w4a8.gemm(A8, sA, rs, blob, N, K, workspace=ws)
    acc0 = w4a8.gemm_debug_acc(A8, rs, blob, N, K, workspace=ws)
    torch.cuda.synchronize()
    oA8, osA, _ = O.quantize_act(A)
    assert (host(A8) == oA8).all()
    cols = sampled_cols(N, I.seed_of("t-rep-c", N, K, M))
    oacc = O.gemm_acc(oA8, O.dequant_weights(q[cols], z[cols], s2[cols]))
    assert (host(acc0)[:, cols] == oacc).all()
    assert max_ulp_fp16(host(Y0)[:, cols], O.epilogue(oacc, osA, s1[cols])) <= 1
    bad = repeat_exact(lambda Y: w4a8.gemm(A8, sA, rs, blob, N, K, out=Y, workspace=ws),
                       lambda acc: w4a8.gemm_debug_acc(A8, rs, blob, N, K, out=acc, workspace=ws), Y0, acc0)
    assert bad == [0, 0], f"launches differing from the first: Y {bad[0]}, acc {bad[1]} of {2 * REPEATS} each"
    assert not host(ws).any()


@pytest.mark.parametrize("ws_tail", [True, False], ids=["expand-once", "expand-in-gemm"])
def test_w4a4_repeated_launches_bit_identical(ws_tail):
    M, N, K = 16, 28672, 4096
    q, z, s2, s1 = I.uniform_codes(N, K, I.seed_of("t-rep-w", N, K))
    A = I.activations(M, K, I.seed_of("t-rep-a4", M, K))
    blob = w4a8.pack_weights(dev(q), dev(z), dev(s2), dev(s1))
    A4, sA, rs = w4a8.w4a4_quantize_act(dev(A))
    base = w4a8.workspace_bytes(M, N, K)
    ws = torch.zeros(w4a8.w4a4_workspace_bytes(M, N, K) if ws_tail else base, dtype=torch.uint8, device=DEV)

    def launch(Y=None, acc=None):
        return w4a8.w4a4_gemm_ex(A4, sA, rs, blob, N, K, Y=Y, acc=acc, workspace=ws)

    Y0 = launch(Y=torch.empty((M, N), dtype=torch.float16, device=DEV))
    acc0 = launch(acc=torch.empty((M, N), dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    o4, osA, _ = O.quantize_act4(A)
    cols = sampled_cols(N, I.seed_of("t-rep-c4", N, K, M))
    oacc = O.gemm_acc(o4, O.dequant_weights(q[cols], z[cols], s2[cols]))
    assert (host(acc0)[:, cols] == oacc).all()
    assert max_ulp_fp16(host(Y0)[:, cols], O.epilogue(oacc, osA, s1[cols])) <= 1
    bad = repeat_exact(lambda Y: launch(Y=Y), lambda acc: launch(acc=acc), Y0, acc0)
    assert bad == [0, 0], f"launches differing from the first: Y {bad[0]}, acc {bad[1]} of {2 * REPEATS} each"
    assert not host(ws)[:base].any()


LUT_CASES = [("gate_up", 16, 28672, 4096), ("down", 1, 4096, 14336), ("qkv", 32, 6144, 4096)]


@pytest.mark.parametrize("name,M,N,K", LUT_CASES, ids=[f"{c[0]}-M{c[1]}" for c in LUT_CASES])
def test_lut_repeated_launches_within_the_bound(name, M, N, K):
    T = I.lut_table()
    q, s = I.lut_codes(N, K, I.seed_of("t-rep-lw", N, K))
    A = I.activations(M, K, I.seed_of("t-rep-la", M, K))
    blob = w4a8.lut_pack_weights(dev(q), dev(s), dev(T))
    Ad = dev(A)
    ws = torch.zeros(w4a8.workspace_bytes(M, N, K), dtype=torch.uint8, device=DEV)
    cols = sampled_cols(N, I.seed_of("t-rep-lc", N, K, M))
    W = O.lut_dequant(q[cols], s[cols], T)
    ex = O.lut_gemm_exact(A, q[cols], s[cols], T)
    E = O.lut_error_bound(A, W)
    ulp = np.spacing(np.maximum(np.abs(ex) + E, 6.1e-05).astype(np.float16)).astype(np.float64)
    tol_acc, tol_y = dev(E), dev(0.5 * ulp + E)
    ex_d, cols_d = dev(ex), dev(cols)
    bad = torch.zeros(2, dtype=torch.int64, device=DEV)
    Ys = [torch.empty((M, N), dtype=torch.float16, device=DEV) for _ in range(2)]
    accs = [torch.empty((M, N), dtype=torch.float32, device=DEV) for _ in range(2)]
    for _ in range(REPEATS):
        for i in range(2):
            w4a8.lut_gemm_ex(Ad, blob, N, K, Y=Ys[i], workspace=ws)
            w4a8.lut_gemm_ex(Ad, blob, N, K, acc=accs[i], workspace=ws)
        for i in range(2):
            bad[0] += ((Ys[i][:, cols_d].double() - ex_d).abs() > tol_y).any()
            bad[1] += ((accs[i][:, cols_d].double() - ex_d).abs() > tol_acc).any()
    torch.cuda.synchronize()
    bad = host(bad).tolist()
    assert bad == [0, 0], f"launches outside the bound: Y {bad[0]}, acc {bad[1]} of {2 * REPEATS} each"
    assert not host(ws).any()
