"""GPU parity of the GEMM chain (w4a8_chain: several W4A8 GEMMs in one
persistent launch) against the CPU oracle, through the C ABI.

Bars, per link: the int8 codes, fp16 scales and rowsums bit-exact with the
oracle's per-token quantization of that link's activations; Y within 1 fp16
ulp of the oracle and bit-identical to the per-GEMM path (w4a8_quantize_act +
w4a8_gemm) on the same inputs; the workspace zero-filled again after every
call. Links that consume the previous link's output (A_j = Y_{j-1}) check the
ordering between links: the oracle runs the same chain on its own outputs.
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


def make_link(M, N, K, seed, A=None, s1_scale=1.0):
    q, z, s2, s1 = I.uniform_codes(N, K, I.seed_of("t-chain-w", seed, N, K))
    codes = (q, z, s2, (s1.astype(np.float32) * np.float32(s1_scale)).astype(np.float16))
    blob = w4a8.pack_weights(*(dev(x) for x in codes))
    A_host = I.activations(M, K, I.seed_of("t-chain-a", seed, M, K)) if A is None else A
    return dict(codes=codes, blob=blob, A_host=A_host, M=M, N=N, K=K)


def gpu_links(links, A_dev=None):
    out = []
    for i, L in enumerate(links):
        M, N, K = L["M"], L["N"], L["K"]
        A = dev(L["A_host"]) if (A_dev is None or A_dev[i] is None) else A_dev[i]
        out.append(dict(A=A, blob=L["blob"], N=N, K=K,
                        Y=torch.full((M, N), float("nan"), dtype=torch.float16, device=DEV),
                        A8=torch.empty((M, K), dtype=torch.int8, device=DEV),
                        sA=torch.empty((M,), dtype=torch.float16, device=DEV),
                        rowsum=torch.empty((M,), dtype=torch.int32, device=DEV)))
    return out


def run_chain(g):
    arr = w4a8.chain_links(g)
    ws = torch.zeros(w4a8.chain_workspace_bytes(arr), dtype=torch.uint8, device=DEV)
    w4a8.chain(arr, ws)
    torch.cuda.synchronize()
    return ws


def oracle_link(A, codes):
    q, z, s2, s1 = codes
    A8, sA, rs = O.quantize_act(A)
    Y = O.epilogue(O.gemm_acc(A8, O.dequant_weights(q, z, s2)), sA, s1)
    return A8, sA, rs, Y


def check_link(g, A_oracle, codes):
    oA8, osA, ors, oY = oracle_link(A_oracle, codes)
    assert (host(g["A8"]) == oA8).all()
    assert (host(g["sA"]).view(np.uint16) == osA.view(np.uint16)).all()
    assert (host(g["rowsum"]) == ors).all()
    assert max_ulp_fp16(host(g["Y"]), oY) <= 1
    # the per-GEMM path on the same device codes gives the same bits
    Yp = w4a8.gemm(g["A8"], g["sA"], g["rowsum"], g["blob"], g["N"], g["K"])
    torch.cuda.synchronize()
    assert torch.equal(Yp, g["Y"])
    return oY


# (M, N, K): tile counts from 1 to above the SM count (one k-range per tile),
# k-block counts from 1 (no split) to many, M from 1 to 32
SHAPES = [(1, 1024, 512), (8, 256, 4096), (32, 20480, 256), (17, 384, 1280), (5, 128, 128), (32, 4096, 2048),
          (3, 6144, 384)]


def test_chain_independent_links_match_the_oracle():
    links = [make_link(M, N, K, i) for i, (M, N, K) in enumerate(SHAPES)]
    g = gpu_links(links)
    ws = run_chain(g)
    for L, gl in zip(links, g):
        check_link(gl, L["A_host"], L["codes"])
    assert not ws.any().item(), "workspace must be left zero-filled"


@pytest.mark.parametrize("dims", [[512, 1024, 512, 4096, 256], [128, 128, 128], [4096, 1024, 14336 // 128 * 128]])
@pytest.mark.parametrize("M", [1, 16, 32])
def test_chain_links_consume_the_previous_output(dims, M):
    """Link j reads Y_{j-1}: the chain must quantize it only once it is
    complete. The oracle runs the same chain on its own outputs."""
    n = len(dims) - 1
    links = []
    for j in range(n):
        K, N = dims[j], dims[j + 1]
        # s1 scaled down so that the outputs stay O(1) from link to link (no
        # fp16 overflow in the activations the next link quantizes)
        links.append(make_link(M, N, K, 100 + j, A=I.activations(M, K, I.seed_of("t-chain-d", j, M)) if j == 0
                               else np.zeros((M, K), np.float16), s1_scale=0.05))
    # GPU: link j's A is link j-1's Y tensor
    g = gpu_links(links)
    for j in range(1, n):
        g[j]["A"] = g[j - 1]["Y"]
    ws = run_chain(g)
    A = links[0]["A_host"]
    for j in range(n):
        oA8, osA, ors, oY = oracle_link(A, links[j]["codes"])
        assert (host(g[j]["A8"]) == oA8).all(), j
        assert (host(g[j]["sA"]).view(np.uint16) == osA.view(np.uint16)).all(), j
        assert (host(g[j]["rowsum"]) == ors).all(), j
        # same fp32 epilogue on both sides: the bits agree, so the next link
        # quantizes the same values on both sides
        assert (host(g[j]["Y"]).view(np.uint16) == oY.view(np.uint16)).all(), j
        A = oY
    assert not ws.any().item()


def test_chain_repeated_calls_and_shared_code_buffers():
    """Three calls in a row on one workspace (the counters and tickets are
    reset by each call), with every link writing its scales and rowsums into
    one shared pair of buffers (allowed: a link's are consumed before the next
    link's are written)."""
    shapes = [(4, 2048, 1024), (4, 512, 2048), (4, 8192, 512)]
    links = [make_link(M, N, K, 200 + i) for i, (M, N, K) in enumerate(shapes)]
    g = gpu_links(links)
    Kmax = max(K for (_, _, K) in shapes)
    A8s = torch.empty((4, Kmax), dtype=torch.int8, device=DEV)
    for gl in g:
        gl["A8"] = A8s[:, :gl["K"]] if gl["K"] == Kmax else torch.empty((4, gl["K"]), dtype=torch.int8, device=DEV)
        gl["sA"] = g[0]["sA"]
        gl["rowsum"] = g[0]["rowsum"]
    arr = w4a8.chain_links(g)
    ws = torch.zeros(w4a8.chain_workspace_bytes(arr), dtype=torch.uint8, device=DEV)
    ref = None
    for _ in range(3):
        w4a8.chain(arr, ws)
        torch.cuda.synchronize()
        ys = [gl["Y"].clone() for gl in g]
        if ref is None:
            ref = ys
        assert all(torch.equal(a, b) for a, b in zip(ref, ys))
        assert not ws.any().item()
    for L, gl, y in zip(links, g, ref):
        _, _, _, oY = oracle_link(L["A_host"], L["codes"])
        assert max_ulp_fp16(host(y), oY) <= 1


def test_chain_sixteen_links_and_one_link():
    shapes = [((j % 4) * 10 + 1, 128 * (1 + j % 3), 128 * (1 + (j * 5) % 7)) for j in range(16)]
    links = [make_link(M, N, K, 300 + i) for i, (M, N, K) in enumerate(shapes)]
    g = gpu_links(links)
    ws = run_chain(g)
    for L, gl in zip(links, g):
        check_link(gl, L["A_host"], L["codes"])
    assert not ws.any().item()
    one = gpu_links(links[:1])
    run_chain(one)
    check_link(one[0], links[0]["A_host"], links[0]["codes"])


def test_chain_full_size_decode_step():
    """The benchmark's decode step as one chain: Llama-3-8B qkv, o, gate_up,
    down at M = 1, 8, 16, 32 (16 links, full size). Codes, scales and rowsums
    in full; Y bit-identical to the per-GEMM path and, on sampled output
    channels (two whole tiles and 64 random channels), within 1 ulp of the
    oracle."""
    wl = I.WORKLOADS["decode"]
    blobs, Ws = {}, {}
    for (name, N, K) in wl.linears:
        W = I.dense_weights(N, K, wl.weight_std, I.weight_seed("decode", N, K))
        q, z, s2, s1 = w4a8.quantize_weights(dev(W))
        blobs[name] = w4a8.pack_weights(q, z, s2, s1)
        Ws[name] = W
    cases = [(M, name, N, K) for M in wl.ms for (name, N, K) in wl.linears]
    g = []
    for (M, name, N, K) in cases:
        g.append(dict(A=dev(I.activations(M, K, I.activation_seed("decode", M, K))), blob=blobs[name], N=N, K=K,
                      Y=torch.empty((M, N), dtype=torch.float16, device=DEV),
                      A8=torch.empty((M, K), dtype=torch.int8, device=DEV),
                      sA=torch.empty((M,), dtype=torch.float16, device=DEV),
                      rowsum=torch.empty((M,), dtype=torch.int32, device=DEV)))
    ws = run_chain(g)
    assert not ws.any().item()
    rng = np.random.default_rng(I.seed_of("t-chain-cols"))
    for (M, name, N, K), gl in zip(cases, g):
        A = I.activations(M, K, I.activation_seed("decode", M, K))
        oA8, osA, ors = O.quantize_act(A)
        assert (host(gl["A8"]) == oA8).all() and (host(gl["rowsum"]) == ors).all()
        assert (host(gl["sA"]).view(np.uint16) == osA.view(np.uint16)).all()
        Yp = w4a8.gemm(gl["A8"], gl["sA"], gl["rowsum"], blobs[name], N, K)
        torch.cuda.synchronize()
        assert torch.equal(Yp, gl["Y"]), (M, name)
        t = int(rng.integers(1, N // 128))
        cols = np.unique(np.concatenate([np.arange(0, 128), np.arange(t * 128, t * 128 + 128),
                                         rng.choice(N, 64, replace=False)]))
        oq, oz, os2, os1 = O.quantize_weights(Ws[name][cols])
        oY = O.epilogue(O.gemm_acc(oA8, O.dequant_weights(oq, oz, os2)), osA, os1)
        assert max_ulp_fp16(host(gl["Y"][:, torch.from_numpy(cols).to(DEV)]), oY) <= 1, (M, name)


def test_chain_rejects_bad_links():
    L = make_link(4, 256, 512, 400)
    g = gpu_links([L])
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device=DEV)
    bad = dict(g[0])
    bad["A"] = torch.zeros((40, 512), dtype=torch.float16, device=DEV)
    bad["Y"] = torch.zeros((40, 256), dtype=torch.float16, device=DEV)
    with pytest.raises(w4a8.W4A8Error, match="UNSUPPORTED"):  # M > 32
        w4a8.chain([bad], ws)
    with pytest.raises(w4a8.W4A8Error, match="WORKSPACE"):
        w4a8.chain(g, torch.zeros(16, dtype=torch.uint8, device=DEV))
    with pytest.raises(w4a8.W4A8Error, match="MISALIGNED"):
        w4a8.chain(g, ws[8:])
