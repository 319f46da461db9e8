"""Benchmark of the W4A8 hot path on B200: activation quantization + W4A8 GEMM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode]
                    [--impl w4a8|reference]

One step = one pass of the hot path over the workload's cases: for every
(M, layer) pair, `w4a8_quantize_act` of that layer's fp16 activations, then
`w4a8_gemm` against the layer's packed 4-bit weights. Weight quantization and
packing are offline (done once before timing). Default workload: Llama-3-8B
decode linears (qkv 6144x4096, o 4096x4096, gate_up 28672x4096,
down 4096x14336) at M in {1, 8, 16, 32}, group 128; 16 GEMMs per step.

Each M value streams its own copy of the packed weights, so a step touches
436 MB of distinct weights (> the 126 MB L2) and no GEMM finds its weights in
L2. The W warm-up steps run eagerly. The K timed steps are one CUDA graph
(K steps unrolled) replayed once between two events; `value` comes from it.
A second graph of the same K steps with an event pair around every GEMM
launch is replayed right after it (events between kernels stop consecutive
kernels from overlapping, so it is not used for `value`): the GEMM's
roofline comes from its per-launch durations.

`value` is the weight-stream rate: packed weight bytes streamed per second
over the whole step (quantization included), summed over ranks.

`e2e` is the same step through the same public calls, with this step's fp16
activations copied in from pinned host memory (one copy of all of them) and
its outputs copied back (one copy), double-buffered on two copy streams so
that the copies of one step overlap the kernels of the next; K steps in one
CUDA graph.

`configs` (default run, one GPU): every GEMM case of the five workloads
(tiny, decode, serving, prefill, Qwen1.5-72B; 57 cases) timed alone: a CUDA
graph of back-to-back launches of that case, rotating over enough copies of
its packed weights that their bytes exceed 3x the L2 cache, mean time per
launch. Per case and per workload: int8 TOPS, weight GB/s and the fraction
of the roofline min(int8 peak, AI x HBM), with the int8 peak taken as 2 x the
measured burst bf16 GEMM rate (the nominal int8/bf16 ratio) and, beside it,
the fraction of a measured `torch._int_mm` 8192^3 int8 ceiling.

`--impl reference` times the CPU oracle on the host cores instead (bounded
sample of the same workload), printing the same kind of line.

`--workload kv-decode` (and the other kv-* workloads) measures the 4-bit
KV-cache decode attention instead: one step = for each of LAYERS layer
caches, `w4kv_append` of the new token's K and V (written at position
L_b - 1) and `w4kv_attention_decode` over the L_b cached tokens of every
sequence; `value` is cache bytes read per second (codes + parameter words
of K and V).

Multi-GPU: the path does not shard across GPUs here (replicas only): every
rank runs the whole workload on its own GPU; the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from w4a8_quantized_gemm_quantize_b200 import inputs as I  # noqa: E402

METRIC = "W4A8 GEMM TOPS & weight GB/s vs M on 1 B200, as % of INT8/HBM roofline"
TILE_BYTES = 8320
HBM_FALLBACK_GBS = 6650.0
BF16_FALLBACK_TFLOPS = 1590.0
INT8_OVER_BF16 = 2.0  # nominal dense ratio (4.5 POPS int8 vs 2.25 PFLOP/s bf16)
INT8_NOMINAL_TOPS = 4500.0  # B200 dense int8, nominal
CONFIG_ORDER = ("tiny", "decode", "serving", "prefill", "qwen72b")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "w4a8_gemm_dram_traffic.json")
KERNEL_SOURCES = ("gemm.cuh", "ptx.cuh", "pack.cuh", "w4a8_api.cu")


# ------------------------------------------------------------ workload facts
LUT_TILE_BYTES = 8448   # 4-bit indices (1/2 byte per weight) + fp16 row scales per 128 x 128 tile
LUT3_TILE_BYTES = 6400  # 3-bit indices (3/8 byte per weight) + fp16 row scales per 128 x 128 tile


def weight_bytes(N, K, lut=False):
    """Packed weight bytes a GEMM must stream: codes + meta + s1, or (lookup-
    table weights, lut = 4 or 3 index bits) indices + row scales + the table."""
    if lut:
        return (N // 128) * (K // 128) * (LUT3_TILE_BYTES if lut == 3 else LUT_TILE_BYTES) + 64
    return (N // 128) * (K // 128) * TILE_BYTES + 2 * N


def algorithmic_bytes(M, N, K, act_bits=8, lut=False):
    """Bytes a W4A8 (W4A4: act_bits=4) GEMM must move at least: packed
    weights, the activation codes, the activation scales, the fp16 output;
    the lookup-table GEMM reads fp16 activations and no scales."""
    if lut:
        return weight_bytes(N, K, lut) + 2 * M * K + 2 * M * N
    return weight_bytes(N, K) + M * K * act_bits // 8 + 2 * M + 2 * M * N


def lut_bits(weights):
    """Index bits of a lookup-table weight format (0: two-level W4A8)."""
    return {"lut": 4, "lut3": 3}.get(weights, 0)


ACT_BITS = {"dynamic": 8, "static": 8, "dynamic4": 4, "static4": 4}


def gemm_ops(M, N, K):
    return 2 * M * N * K


def cases_of(workload, only=None):
    """The workload's (M, layer, N, K) cases; `only` ("16:gate_up,1:o")
    keeps a subset (for profiling single shapes)."""
    wl = I.WORKLOADS[workload]
    cases = [(M, name, N, K) for M in wl.ms for (name, N, K) in wl.linears]
    if only:
        keep = {(int(x.split(":")[0]), x.split(":")[1]) for x in only.split(",")}
        cases = [c for c in cases if (c[0], c[1]) in keep]
        if not cases:
            raise SystemExit(f"--cases {only!r} selects nothing from workload {workload!r}")
    return cases


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": HBM_FALLBACK_GBS, "bf16_tflops": BF16_FALLBACK_TFLOPS,
                "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def kernel_source_hash():
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "w4a8_quantized_gemm_quantize_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload):
    """DRAM bytes per GEMM launch from a committed ncu summary, if it was taken
    on the current kernel sources (else None)."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    if t.get("kernel_source_hash") != kernel_source_hash():
        return None
    return t.get("per_launch_bytes", {}).get(workload)


# ------------------------------------------------------------------- ranks
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(value: float, world: int) -> float:
    """Max of a per-rank scalar over all ranks (identity with one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, torch_device, period_s=0.002):
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            handle = None
            try:
                import torch
                uuid = str(torch.cuda.get_device_properties(torch_device).uuid)
                handle = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
            except Exception:
                handle = None
            if handle is None:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
                idx = torch_device.index or 0
                if vis and vis.split(",")[idx].strip().isdigit():
                    idx = int(vis.split(",")[idx])
                handle = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.h = handle
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _reasons(self):
        try:
            return self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            return self.nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self._reasons())
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# -------------------------------------------------------------- CPU oracle
_ORACLE_WEIGHTS = {}


def cpu_oracle_run(workload, budget_s, reps=1, act_bits=8, lut=False):
    """Times the CPU oracle (activation quantization + GEMM with the fp32
    epilogue; 4-bit activations with act_bits=4) on this host over a bounded
    sample of the workload's cases; returns (weight GB/s, description of the
    sample, threads used)."""
    from oracle import w4a8_oracle as O
    cases = cases_of(workload)
    prepared = _ORACLE_WEIGHTS
    done_bytes, done_time, done = 0, 0.0, []
    t_start = time.perf_counter()
    for (M, name, N, K) in cases:
        if time.perf_counter() - t_start > budget_s and done:
            break
        wl = I.WORKLOADS[workload]
        key = (workload, N, K, lut)
        if key not in prepared and lut == 3:
            prepared[key] = I.lut3_codes(N, K, I.weight_seed(workload + "-lut3", N, K))
        elif key not in prepared and lut:
            prepared[key] = I.lut_codes(N, K, I.weight_seed(workload + "-lut", N, K))
        elif key not in prepared:
            if wl.weight_std == 0.0:
                prepared[key] = I.uniform_codes(N, K, I.weight_seed(workload, N, K))
            else:
                W = I.dense_weights(N, K, wl.weight_std, I.weight_seed(workload, N, K))
                prepared[key] = O.quantize_weights(W)
        A = I.activations(M, K, I.activation_seed(workload, M, K))
        for _ in range(reps):
            t0 = time.perf_counter()
            if lut:
                q, s = prepared[key]
                O.lut_gemm(A, q, s, I.lut3_table() if lut == 3 else I.lut_table())
                done_time += time.perf_counter() - t0
                done_bytes += weight_bytes(N, K, lut)
                continue
            q, z, s2, s1 = prepared[key]
            if act_bits == 4:
                A4, sA, _ = O.quantize_act4(A)
                O.w4a4_gemm(O.pack_act4(A4), sA, q, z, s2, s1)
            else:
                A8, sA, _ = O.quantize_act(A)
                O.w4a8_gemm(A8, sA, q, z, s2, s1)
            done_time += time.perf_counter() - t0
            done_bytes += weight_bytes(N, K)
        done.append(f"M={M} {name} {N}x{K}")
    threads = cpu_threads()
    return done_bytes / done_time / 1e9, done, threads, done_time


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = max((int(p.get("num_threads", 1)) for p in threadpool_info()), default=1)
        return n
    except Exception:
        return os.cpu_count() or 1


# ----------------------------------------------------------------- GPU arm
def run_gpu(args, world, rank, local):
    import torch
    import w4a8_quantized_gemm_quantize_b200 as w4a8

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wl = I.WORKLOADS[args.workload]
    cases = cases_of(args.workload, args.cases)
    n_copies = len(wl.ms)  # one weight copy per M value: no GEMM reuses L2-resident weights

    # ---- offline: quantize + pack the weights (untimed), one copy per M
    blobs = {}
    lut = lut_bits(args.weights)
    table = torch.from_numpy(I.lut3_table() if lut == 3 else I.lut_table()).to(dev) if lut else None
    for (name, N, K) in wl.linears:
        if lut:
            gen = I.lut3_codes if lut == 3 else I.lut_codes
            q, s = (torch.from_numpy(x).to(dev) for x in gen(N, K, I.weight_seed(f"{args.workload}-{args.weights}", N, K)))
            blobs[(name, 0)] = (w4a8.lut3_pack_weights if lut == 3 else w4a8.lut_pack_weights)(q, s, table)
            del q, s
            for c in range(1, n_copies):
                blobs[(name, c)] = blobs[(name, 0)].clone()
            continue
        if wl.weight_std == 0.0:
            q, z, s2, s1 = (torch.from_numpy(x).to(dev) for x in I.uniform_codes(N, K, I.weight_seed(args.workload, N, K)))
        else:
            W = torch.from_numpy(I.dense_weights(N, K, wl.weight_std, I.weight_seed(args.workload, N, K))).to(dev)
            q, z, s2, s1 = w4a8.quantize_weights(W)
            del W
        blob = w4a8.pack_weights(q, z, s2, s1)
        del q, z, s2
        blobs[(name, 0)] = blob
        for c in range(1, n_copies):
            blobs[(name, c)] = blob.clone()
    torch.cuda.synchronize()

    # ---- activations and outputs, resident in HBM. Each kind lives in one
    # buffer (per-case views at 256-byte aligned offsets), so that the
    # end-to-end run moves a step's inputs and outputs with one copy each.
    def packed_views(shapes, dtype, n_buffers=1):
        esize = torch.empty((), dtype=dtype).element_size()
        offs, total = [], 0
        for shp in shapes:
            offs.append(total)
            total += (int(np.prod(shp)) * esize + 255) // 256 * 256
        bufs = [torch.zeros((max(total, 256),), dtype=torch.uint8, device=dev) for _ in range(n_buffers)]
        views = [[b[o:o + int(np.prod(shp)) * esize].view(dtype).view(shp) for o, shp in zip(offs, shapes)]
                 for b in bufs]
        return bufs, views

    acts, outs = {}, {}
    ws_size = w4a8.w4a4_workspace_bytes if ACT_BITS[args.act] == 4 else w4a8.workspace_bytes
    ws = torch.zeros(max(ws_size(M, N, K) for (M, _, N, K) in cases), dtype=torch.uint8, device=dev)
    a_bufs, a_views = packed_views([(M, K) for (M, _, N, K) in cases], torch.float16, 3)
    y_bufs, y_views = packed_views([(M, N) for (M, _, N, K) in cases], torch.float16, 3)
    host_acts = [I.activations(M, K, I.activation_seed(args.workload, M, K)) for (M, name, N, K) in cases]
    for i, (M, name, N, K) in enumerate(cases):
        for b in range(3):
            a_views[b][i].copy_(torch.from_numpy(host_acts[i]))
        acts[(M, name)] = a_views[0][i]
        codes = (torch.empty((M, K), dtype=torch.int8, device=dev) if ACT_BITS[args.act] == 8 else
                 torch.empty((M, K // 2), dtype=torch.uint8, device=dev))
        outs[(M, name)] = (codes,
                           torch.empty((M,), dtype=torch.float16, device=dev),
                           torch.empty((M,), dtype=torch.int32, device=dev),
                           y_views[0][i])
    copy_of = {M: i for i, M in enumerate(wl.ms)}
    static_scales = None
    if args.act in ("static", "static4"):
        # offline calibration: one scale per activation tensor, from its range
        qmax = 127 if args.act == "static" else 7
        static_scales = {key: (A.float().abs().max() / qmax).to(torch.float16).reshape(1)
                         for key, A in acts.items()}
    if lut:
        quantize = None

        lut_gemm = w4a8.lut3_gemm if lut == 3 else w4a8.lut_gemm

        def gemm(A8, sA, rs, blob, N, K, out, workspace):  # weight-only: the fp16 activations feed the GEMM
            return lut_gemm(A8, blob, N, K, out=out, workspace=workspace)
    elif ACT_BITS[args.act] == 4:
        quantize = (w4a8.w4a4_quantize_act_static if static_scales is not None else w4a8.w4a4_quantize_act)
        gemm = w4a8.w4a4_gemm
    else:
        quantize = (w4a8.quantize_act_static if static_scales is not None else w4a8.quantize_act)
        gemm = w4a8.gemm

    chain = bool(getattr(args, "chain_mode", False))
    if chain:
        # the step as one chain launch (w4a8_chain): the same quantize + GEMM
        # per case, in the same order, each link after the previous one
        chain_arrs = [w4a8.chain_links([dict(A=a_views[b][i], blob=blobs[(name, copy_of[M])], N=N, K=K,
                                             Y=y_views[b][i], A8=outs[(M, name)][0], sA=outs[(M, name)][1],
                                             rowsum=outs[(M, name)][2])
                                        for i, (M, name, N, K) in enumerate(cases)]) for b in range(3)]
        chain_ws = torch.zeros(w4a8.chain_workspace_bytes(chain_arrs[0]), dtype=torch.uint8, device=dev)

    def step(events=None, gemm_only=False, buf=0, quant_only=False):
        """One pass over the cases; `buf` selects the activation and output
        buffers (the end-to-end run alternates between two); `quant_only`
        runs the activation quantizers alone (their roofline)."""
        if chain:
            w4a8.chain(chain_arrs[buf], chain_ws)
            return
        for i, (M, name, N, K) in enumerate(cases):
            A = a_views[buf][i]
            A8, sA, rs, _ = outs[(M, name)]
            Y = y_views[buf][i]
            if lut:
                A8 = A
            elif not gemm_only:
                if static_scales is not None:
                    quantize(A, static_scales[(M, name)], out=(A8, sA, rs))
                else:
                    quantize(A, out=(A8, sA, rs))
            if quant_only:
                continue
            if events is not None:
                events[i][0].record()
            gemm(A8, sA, rs, blobs[(name, copy_of[M])], N, K, out=Y, workspace=ws)
            if events is not None:
                events[i][1].record()

    if args.profile:
        # for an external profiler: eager steps only, no timing, no JSON line
        for _ in range(args.profile):
            step()
        torch.cuda.synchronize()
        assert w4a8.get_device_error(dev) == 0
        print(f"profile: {args.profile} eager steps of {len(cases)} cases done")
        return None

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert w4a8.get_device_error(dev) == 0

    # ---- timed region 1: K steps (unrolled) in one CUDA graph, no events
    # inside, so consecutive kernels overlap through programmatic launch
    def capture(events_per_step, gemm_only=False, quant_only=False):
        g = torch.cuda.CUDAGraph()
        cap_stream = torch.cuda.Stream(dev)
        cap_stream.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(cap_stream):
            with torch.cuda.graph(g, stream=cap_stream):
                for s in range(args.steps):
                    step(events=None if events_per_step is None else events_per_step[s], gemm_only=gemm_only,
                         quant_only=quant_only)
        torch.cuda.current_stream(dev).wait_stream(cap_stream)
        return g

    K_steps = args.steps
    g_plain = capture(None)
    # ---- timed region 2: the GEMM launches of the same K steps alone (same
    # inputs, same launch configuration, same weight rotation), events only at
    # the ends: the GEMM kernel's average duration for the roofline (a chain
    # step is one launch: this graph is the same K chain launches)
    g_gemm = capture(None, gemm_only=True)
    # ---- timed region 3: the full steps with an external event pair around
    # every GEMM (a per-case breakdown; these events add a few microseconds
    # to each launch and stop consecutive kernels from overlapping); a chain
    # step has no per-case launches, so it is timed as a whole
    ev = [[[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)] for _ in cases]
          for _ in range(K_steps)]
    g_ev = capture(None if chain else ev)
    # ---- timed region 4: the activation quantizers of the same K steps alone
    g_quant = None if (chain or lut) else capture(None, quant_only=True)
    for g in (g_plain, g_gemm, g_ev, g_quant):  # untimed replays: settle clocks and caches
        if g is not None:
            g.replay()
    torch.cuda.synchronize()

    stream = torch.cuda.current_stream(dev)
    t0, t1, t2, t3, t4, t5 = (torch.cuda.Event(enable_timing=True) for _ in range(6))
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        t0.record(stream)
        g_plain.replay()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        t2.record(stream)
        g_gemm.replay()
        t3.record(stream)
        torch.cuda.synchronize()
        g_ev.replay()
        torch.cuda.synchronize()
        if g_quant is not None:
            barrier(world)
            t4.record(stream)
            g_quant.replay()
            t5.record(stream)
            torch.cuda.synchronize()
    barrier(world)
    elapsed_ms = t0.elapsed_time(t1)
    max_ms = max_over_ranks(elapsed_ms, world)
    gemm_ms = max_over_ranks(t2.elapsed_time(t3), world)
    quant_ms = max_over_ranks(t4.elapsed_time(t5), world) if g_quant is not None else None
    assert w4a8.get_device_error(dev) == 0

    per_case_ms = np.zeros(len(cases))
    if not chain:
        for s in range(K_steps):
            for i in range(len(cases)):
                per_case_ms[i] += ev[s][i][0].elapsed_time(ev[s][i][1])
        per_case_ms /= K_steps
    del g_plain, g_gemm, g_ev, g_quant

    # ---- end to end through the public API: each step copies its fp16
    # activations in from pinned host memory (one copy) and its outputs back
    # (one copy). Double-buffered on two copy streams: step s computes on
    # buffer 1 + s % 2 while step s + 1's inputs arrive and step s - 1's
    # outputs leave.
    a_host = torch.empty((a_bufs[0].numel(),), dtype=torch.uint8).pin_memory()
    a_host.copy_(a_bufs[0].cpu())
    y_host = [torch.empty((y_bufs[0].numel(),), dtype=torch.uint8).pin_memory() for _ in range(2)]
    h2d_bytes, d2h_bytes = a_host.numel(), y_host[0].numel()

    def capture_e2e(nsteps):
        g = torch.cuda.CUDAGraph()
        cs = torch.cuda.Stream(dev)
        hs, ds = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = [[torch.cuda.Event() for _ in range(3)] for _ in range(nsteps)]  # inputs in, computed, outputs out
        cs.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(cs):
            with torch.cuda.graph(g, stream=cs):
                hs.wait_stream(cs)
                ds.wait_stream(cs)
                for s_ in range(nsteps):
                    b = 1 + s_ % 2
                    with torch.cuda.stream(hs):
                        if s_ >= 2:
                            hs.wait_event(ev[s_ - 2][1])  # buffer b's previous inputs consumed
                        a_bufs[b].copy_(a_host, non_blocking=True)
                        ev[s_][0].record(hs)
                    cs.wait_event(ev[s_][0])
                    if s_ >= 2:
                        cs.wait_event(ev[s_ - 2][2])  # buffer b's previous outputs copied out
                    step(buf=b)
                    ev[s_][1].record(cs)
                    with torch.cuda.stream(ds):
                        ds.wait_event(ev[s_][1])
                        y_host[s_ % 2].copy_(y_bufs[b], non_blocking=True)
                        ev[s_][2].record(ds)
                cs.wait_stream(hs)
                cs.wait_stream(ds)
        torch.cuda.current_stream(dev).wait_stream(cs)
        return g

    g_e2e = capture_e2e(K_steps)
    g_e2e.replay()  # untimed
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g_e2e.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    del g_e2e
    # the outputs that came back equal the device-resident run's (bit for bit
    # with integer sums; the lookup-table GEMM's fp32 sums may add in another
    # order under split k-ranges)
    y_back, y_dev = y_host[(K_steps - 1) % 2].view(torch.float16), y_bufs[0].cpu().view(torch.float16)
    if lut:
        assert torch.allclose(y_back.float(), y_dev.float(), rtol=1e-2, atol=1e-3)
    else:
        assert torch.equal(y_back, y_dev)
    assert w4a8.get_device_error(dev) == 0

    return dict(elapsed_ms=elapsed_ms, max_ms=max_ms, gemm_ms=gemm_ms, quant_ms=quant_ms, per_case_ms=per_case_ms,
                clocks=clk.summary(),
                e2e_ms=e2e_ms, cases=cases, n_copies=n_copies, h2d_bytes=h2d_bytes, d2h_bytes=d2h_bytes,
                gpu_name=torch.cuda.get_device_name(dev))


# ------------------------------------------------ per-case sweep of configs
def int8_ceiling_tops(dev, n=8192, reps=10):
    """Best-of-`reps` int8 throughput of torch._int_mm (cuBLAS) on n^3:
    a measured int8 tensor ceiling for this box (None if unavailable)."""
    import torch
    try:
        a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev)
        b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev).t()  # column-major operand
        torch._int_mm(a, b)
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._int_mm(a, b)
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        del a, b
        return 2.0 * n ** 3 / (best * 1e-3) / 1e12
    except Exception as e:  # noqa: BLE001 - reported, not fatal
        return f"unavailable: {type(e).__name__}: {str(e)[:120]}"


def run_configs(dev, peaks, int8_meas):
    """Times every GEMM case of the five workloads alone (see the module
    docstring); returns the `configs` block of the JSON line."""
    import torch
    import w4a8_quantized_gemm_quantize_b200 as w4a8
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    hbm = peaks["hbm_gbs"]
    int8_peak = peaks["bf16_tflops"] * INT8_OVER_BF16
    block, launches = {}, 0
    for wname in CONFIG_ORDER:
        wl = I.WORKLOADS[wname]
        rows = []
        for (lname, N, K) in wl.linears:
            if wl.weight_std == 0.0:
                q, z, s2, s1 = (torch.from_numpy(x).to(dev) for x in I.uniform_codes(N, K, I.weight_seed(wname, N, K)))
            else:
                W = torch.from_numpy(I.dense_weights(N, K, wl.weight_std, I.weight_seed(wname, N, K))).to(dev)
                q, z, s2, s1 = w4a8.quantize_weights(W)
                del W
            blob = w4a8.pack_weights(q, z, s2, s1)
            del q, z, s2, s1
            wb = weight_bytes(N, K)
            n_copies = min(max(2, -(-3 * l2 // wb)), 512)  # > 3x L2 of distinct weights per rotation
            l2_resident = n_copies * wb < 3 * l2  # only the tiny case: its copies cannot outgrow L2
            blobs = [blob] + [blob.clone() for _ in range(n_copies - 1)]
            for M in wl.ms:
                A = torch.from_numpy(I.activations(M, K, I.activation_seed(wname, M, K))).to(dev)
                A8, sA, rs = w4a8.quantize_act(A)
                Y = torch.empty((M, N), dtype=torch.float16, device=dev)
                ws = torch.zeros(w4a8.workspace_bytes(M, N, K), dtype=torch.uint8, device=dev)
                ops, ab = gemm_ops(M, N, K), algorithmic_bytes(M, N, K)
                est_ms = max(ab / (hbm * 1e9), ops / (int8_peak * 1e12)) * 1e3 + 0.006
                reps = max(1, -(-int(np.ceil(3.0 / est_ms)) // n_copies))  # ~3 ms per replay
                R = min(max(n_copies * reps, 4), 512)
                for i in range(2):
                    w4a8.gemm(A8, sA, rs, blobs[i % n_copies], N, K, out=Y, workspace=ws)
                g = torch.cuda.CUDAGraph()
                cs = torch.cuda.Stream(dev)
                cs.wait_stream(torch.cuda.current_stream(dev))
                with torch.cuda.stream(cs):
                    with torch.cuda.graph(g, stream=cs):
                        for i in range(R):
                            w4a8.gemm(A8, sA, rs, blobs[i % n_copies], N, K, out=Y, workspace=ws)
                torch.cuda.current_stream(dev).wait_stream(cs)
                g.replay()
                torch.cuda.synchronize()
                ts = []
                for _ in range(3):
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record()
                    g.replay()
                    e1.record()
                    torch.cuda.synchronize()
                    ts.append(e0.elapsed_time(e1) / R)
                launches += 4 * R + 2
                del g
                t = sorted(ts)[1] * 1e-3  # median, seconds per launch
                t_hbm, t_tc = ab / (hbm * 1e9), ops / (int8_peak * 1e12)
                row = {"M": M, "layer": lname, "N": N, "K": K, "us": round(t * 1e6, 2),
                       "tops": round(ops / t / 1e12, 2), "weight_GBs": round(wb / t / 1e9, 1),
                       "bound": "hbm" if t_hbm >= t_tc else "tensor",
                       "roofline_frac": round(max(t_hbm, t_tc) / t, 4), "launches_per_graph": R}
                if l2_resident:
                    row["weights_in_l2"] = True
                if isinstance(int8_meas, float) and t_tc > t_hbm:
                    row["frac_of_int_mm"] = round(ops / t / 1e12 / int8_meas, 4)
                rows.append(row)
                del A, A8, sA, rs, Y, ws
            del blobs, blob
            torch.cuda.empty_cache()
        assert w4a8.get_device_error(dev) == 0
        tot_t = sum(r["us"] for r in rows) * 1e-6
        tot_ops = sum(gemm_ops(r["M"], r["N"], r["K"]) for r in rows)
        tot_w = sum(weight_bytes(r["N"], r["K"]) for r in rows)
        roof = sum(r["roofline_frac"] * r["us"] for r in rows) * 1e-6
        block[wname] = {"cases": rows, "tops": round(tot_ops / tot_t / 1e12, 2),
                        "weight_GBs": round(tot_w / tot_t / 1e9, 1), "roofline_frac": round(roof / tot_t, 4)}

    def frac_over(pred):
        rs = [r for w in block.values() for r in w["cases"] if pred(r)]
        t = sum(r["us"] for r in rs)
        return round(sum(r["roofline_frac"] * r["us"] for r in rs) / t, 4) if t else None

    summary = {
        "hbm_frac_M_le_32": frac_over(lambda r: r["M"] <= 32 and r["bound"] == "hbm"),
        "tensor_frac_M_ge_2048": frac_over(lambda r: r["M"] >= 2048),
        "int8_peak_tops": int8_peak,
        "int8_peak_source": f"{peaks['source']} burst bf16 x {INT8_OVER_BF16:g} (nominal int8/bf16 ratio)",
        "int8_int_mm_tops": round(int8_meas, 1) if isinstance(int8_meas, float) else int8_meas,
        "int8_nominal_tops": INT8_NOMINAL_TOPS,
        "hbm_peak_gbs": hbm,
        "timing": "per case: CUDA graph of back-to-back launches rotating over > 3x L2 of weight copies; "
                  "median of 3 replays / launches",
    }
    rs_big = [r for w in block.values() for r in w["cases"] if r["M"] >= 2048]
    if rs_big and isinstance(int8_meas, float):
        t = sum(r["us"] for r in rs_big) * 1e-6
        summary["tensor_M_ge_2048_frac_of_int_mm"] = round(
            sum(gemm_ops(r["M"], r["N"], r["K"]) for r in rs_big) / t / 1e12 / int8_meas, 4)
        summary["tensor_M_ge_2048_frac_of_nominal"] = round(
            sum(gemm_ops(r["M"], r["N"], r["K"]) for r in rs_big) / t / 1e12 / INT8_NOMINAL_TOPS, 4)
    return {"summary": summary, **block}, launches


# ------------------------------------------------------ 4-bit KV attention
KV_METRIC = "KV4 decode attention: 4-bit KV-cache bytes read per second on 1 B200, as % of HBM roofline"
KV_LAYERS = 4  # distinct layer caches per step: the step's cache bytes exceed L2


def kv_cache_bytes(lens, Hkv):
    """Bytes of the cached K and V a decode step must read: per token and kv
    head 64 code bytes + one 4-byte parameter word, for K and for V."""
    return int(np.sum(lens)) * Hkv * 2 * (64 + 4)


def kv_algorithmic_bytes(lens, Hq, Hkv):
    """The attention launch's bytes: the cache it reads, the queries, the output."""
    B = len(lens)
    return kv_cache_bytes(lens, Hkv) + 2 * B * Hq * 128 * 2


def kv_case(wl, seed_tag):
    Hq, Hkv, D = wl.heads
    K = I.kv_vectors(wl.batch, Hkv, wl.max_len, D, I.seed_of(seed_tag, "k", wl.name))
    V = I.kv_vectors(wl.batch, Hkv, wl.max_len, D, I.seed_of(seed_tag, "v", wl.name), outlier_scale=1.0)
    q = I.kv_queries(wl.batch, Hq, D, I.seed_of(seed_tag, "q", wl.name))
    lens = I.kv_seq_lens(wl, I.seed_of(seed_tag, "lens", wl.name))
    return K, V, q, lens


def cpu_oracle_run_kv(workload, budget_s):
    """Times the CPU oracle's decode attention on sequences of the workload
    until the budget is spent; returns (cache GB/s, sample, threads, seconds)."""
    from oracle import kv4_oracle as KV
    wl = I.KV_WORKLOADS[workload]
    Hq, Hkv, D = wl.heads
    key = ("kv", workload)
    if key not in _ORACLE_WEIGHTS:  # the cache, quantized once (untimed), as on the GPU
        K, V, q, lens = kv_case(wl, "bench")
        kc, ks, kz = KV.quantize_kv(K)
        vc, vs, vz = KV.quantize_kv(V)
        _ORACLE_WEIGHTS[key] = (K, V, q, lens, KV.pack_kv(kc), KV.kv_params(ks, kz), KV.pack_kv(vc),
                                KV.kv_params(vs, vz))
    K, V, q, lens, kc, kp, vc, vp = _ORACLE_WEIGHTS[key]
    done_t, done_b, seqs = 0.0, 0, []
    for b in range(wl.batch):
        if done_t > budget_s and seqs:
            break
        L = int(lens[b])
        sl = slice(b, b + 1)
        t0 = time.perf_counter()
        # the step of one sequence: quantize the new token's K and V, attend
        KV.quantize_kv(K[b, :, L - 1])
        KV.quantize_kv(V[b, :, L - 1])
        KV.attention_decode(q[sl], kc[sl], kp[sl], vc[sl], vp[sl], lens[sl], 1.0 / np.sqrt(D))
        done_t += time.perf_counter() - t0
        done_b += kv_cache_bytes(lens[sl], Hkv)
        seqs.append(f"seq {b} ({L} tokens)")
    return done_b / done_t / 1e9, seqs, cpu_threads(), done_t


def run_gpu_kv(args, world, rank, local):
    import torch
    import w4a8_quantized_gemm_quantize_b200 as w4a8

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wl = I.KV_WORKLOADS[args.workload]
    Hq, Hkv, D = wl.heads
    K, V, q, lens = kv_case(wl, "bench")
    scale = float(np.float32(1.0 / np.sqrt(D)))
    # ---- offline: the caches of KV_LAYERS layers (untimed)
    caches = []
    for _ in range(KV_LAYERS):
        kc, kp = w4a8.kv4_quantize(torch.from_numpy(K).to(dev))
        vc, vp = w4a8.kv4_quantize(torch.from_numpy(V).to(dev))
        caches.append((kc, kp, vc, vp))
    qd = torch.from_numpy(q).to(dev)
    lens_d = torch.from_numpy(lens).to(dev)
    pos_d = torch.from_numpy(np.maximum(lens - 1, 0).astype(np.int32)).to(dev)
    k_new = torch.from_numpy(np.ascontiguousarray(K[np.arange(wl.batch), :, np.maximum(lens - 1, 0)])).to(dev)
    v_new = torch.from_numpy(np.ascontiguousarray(V[np.arange(wl.batch), :, np.maximum(lens - 1, 0)])).to(dev)
    outs = [torch.empty((wl.batch, Hq, D), dtype=torch.float16, device=dev) for _ in range(KV_LAYERS)]
    ws = torch.zeros(w4a8.kv4_workspace_bytes(wl.batch, Hq, Hkv, wl.max_len), dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()

    def step(attn_only=False, h2d=None, d2h=None):
        for i, (kc, kp, vc, vp) in enumerate(caches):
            if h2d is not None:
                qd.copy_(h2d[0], non_blocking=True)
                k_new.copy_(h2d[1], non_blocking=True)
                v_new.copy_(h2d[2], non_blocking=True)
            if not attn_only:
                w4a8.kv4_append(k_new, v_new, pos_d, kc, kp, vc, vp)
            w4a8.kv4_attention_decode(qd, kc, kp, vc, vp, lens_d, scale, out=outs[i], workspace=ws)
            if d2h is not None:
                d2h[i].copy_(outs[i], non_blocking=True)

    if args.profile:
        # for an external profiler: eager steps only, no timing, no JSON line
        for _ in range(args.profile):
            step()
        torch.cuda.synchronize()
        assert w4a8.get_device_error(dev) == 0
        print(f"profile: {args.profile} eager steps of {KV_LAYERS} layer caches done")
        return None

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert w4a8.get_device_error(dev) == 0

    def capture(attn_only):
        g = torch.cuda.CUDAGraph()
        cs = torch.cuda.Stream(dev)
        cs.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(cs):
            with torch.cuda.graph(g, stream=cs):
                for _ in range(args.steps):
                    step(attn_only)
        torch.cuda.current_stream(dev).wait_stream(cs)
        return g

    g_plain, g_attn = capture(False), capture(True)
    for g in (g_plain, g_attn):
        g.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    t0, t1, t2, t3 = (torch.cuda.Event(enable_timing=True) for _ in range(4))
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        t0.record(stream)
        g_plain.replay()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        t2.record(stream)
        g_attn.replay()
        t3.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    max_ms = max_over_ranks(t0.elapsed_time(t1), world)
    attn_ms = max_over_ranks(t2.elapsed_time(t3), world)
    assert w4a8.get_device_error(dev) == 0
    del g_plain, g_attn

    # ---- end to end through the public API: pinned q and new K/V in, Y out
    h2d = tuple(t.cpu().pin_memory() for t in (qd, k_new, v_new))
    d2h = [torch.empty((wl.batch, Hq, D), dtype=torch.float16).pin_memory() for _ in range(KV_LAYERS)]
    step(h2d=h2d, d2h=d2h)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step(h2d=h2d, d2h=d2h)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    for i in range(KV_LAYERS):
        assert torch.equal(d2h[i], outs[i].cpu())
    return dict(max_ms=max_ms, attn_ms=attn_ms, e2e_ms=e2e_ms, clocks=clk.summary(), lens=lens,
                h2d_bytes=KV_LAYERS * sum(t.numel() * t.element_size() for t in h2d),
                d2h_bytes=KV_LAYERS * wl.batch * Hq * D * 2, gpu_name=torch.cuda.get_device_name(dev))


def main_kv(args, world, rank, local):
    wl = I.KV_WORKLOADS[args.workload]
    Hq, Hkv, D = wl.heads
    if args.impl == "reference":
        if rank != 0:
            return
        cpu_oracle_run_kv(args.workload, 0.0)  # untimed warm-up (one sequence)
        tot_b, tot_t, sample, threads = 0.0, 0.0, [], 1
        for _ in range(args.steps):
            v, sample, threads, t = cpu_oracle_run_kv(args.workload, args.cpu_seconds / max(args.steps, 1))
            tot_b += v * t * 1e9
            tot_t += t
        value = tot_b / tot_t / 1e9
        print(json.dumps({
            "metric": KV_METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(tot_t / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": args.workload, "heads": list(wl.heads), "batch": wl.batch,
                       "max_len": wl.max_len},
            "impl": "reference",
            "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": f"per step: {len(sample)} sequences ({'; '.join(sample)})"},
            "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
            flush=True)
        return
    if world > 1:
        import torch
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    r = run_gpu_kv(args, world, rank, local)
    if r is None:  # --profile
        return 0
    peaks = load_peaks()
    lens = r["lens"]
    cache_b = KV_LAYERS * kv_cache_bytes(lens, Hkv)
    ms_step = r["max_ms"] / args.steps
    attn_launch_ms = r["attn_ms"] / (args.steps * KV_LAYERS)
    achieved = kv_algorithmic_bytes(lens, Hq, Hkv) / (attn_launch_ms * 1e-3) / 1e9
    line = {
        "metric": KV_METRIC, "value": round(world * cache_b / (ms_step * 1e-3) / 1e9, 1), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": args.workload, "heads": list(wl.heads), "batch": wl.batch, "max_len": wl.max_len,
                   "tokens": int(np.sum(lens)), "layers_per_step": KV_LAYERS,
                   "l2": f"inputs larger than L2: {KV_LAYERS} layer caches, {cache_b / 1e6:.0f} MB per step",
                   "parallelism": f"replicas x{world}"},
        # per layer: the append's two quantizer launches, the attention's two
        # (partial results per chunk, then the merge)
        "gpu_launches": 4 * KV_LAYERS * args.steps,
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": None,
                     "peak_source": f"{peaks['source']} HBM copy",
                     "kernel": "kv4_decode_kernel + kv4_merge_kernel (one attention call)",
                     "avg_launch_us": round(attn_launch_ms * 1e3, 3)},
        "e2e": {"value": round(world * cache_b / (r["e2e_ms"] / args.steps * 1e-3) / 1e9, 1), "unit": "GB/s",
                "h2d_bytes_per_step": r["h2d_bytes"], "d2h_bytes_per_step": r["d2h_bytes"]},
        "clocks": r["clocks"], "gpu": r["gpu_name"],
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, sample, threads, t = cpu_oracle_run_kv(args.workload, args.cpu_seconds)
        line["cpu_baseline"] = {"value": round(v, 3), "unit": "GB/s", "cores": threads, "kind": "oracle",
                                "sample": f"{len(sample)} of {wl.batch} sequences, {t:.1f} s of oracle time"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="decode", choices=sorted(I.WORKLOADS) + sorted(I.KV_WORKLOADS))
    ap.add_argument("--impl", default="w4a8", choices=["w4a8", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="budget of the CPU-oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--chain", default="off", choices=["off", "on"],
                    help="on: run the step as one w4a8_chain launch (8-bit dynamic activations, every M <= 32, at "
                         "most 16 cases; measured slower than separate launches on the decode workload); the "
                         "per-launch figures are reported beside it")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-case sweep of all five workloads (the `configs` block)")
    ap.add_argument("--cases", default=None,
                    help="subset of the workload's cases, e.g. 16:gate_up,1:o (profiling)")
    ap.add_argument("--act", default="dynamic", choices=["dynamic", "static", "dynamic4", "static4"],
                    help="activation codes and scales: 8-bit per-token dynamic (w4a8_quantize_act) or per-tensor "
                         "static calibrated once before timing (w4a8_quantize_act_static); 4-bit (W4A4: "
                         "w4a4_quantize_act / w4a4_quantize_act_static + w4a4_gemm)")
    ap.add_argument("--weights", default="w4a8", choices=["w4a8", "lut", "lut3"],
                    help="w4a8: two-level 4-bit weights against quantized activations; lut: 4-bit indices into a "
                         "16-entry fp16 table with group scales against fp16 activations (weight-only, "
                         "w4lut_gemm); lut3: 3-bit indices into an 8-entry table (w4lut3_gemm)")
    ap.add_argument("--profile", type=int, default=0,
                    help="run this many eager steps for an external profiler and exit (no timing)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world, rank, local = dist_env()
    if args.workload in I.KV_WORKLOADS:
        return main_kv(args, world, rank, local)
    if args.impl == "reference":
        return main_reference(args, world, rank)

    if world > 1:
        import torch
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))

    r = run_gpu(args, world, rank, local)
    if r is None:  # --profile
        return 0
    cases = r["cases"]
    peaks = load_peaks()
    lut = lut_bits(args.weights)
    wbytes = sum(weight_bytes(N, K, lut) for (M, _, N, K) in cases)
    abytes = [algorithmic_bytes(M, N, K, ACT_BITS[args.act], lut) for (M, _, N, K) in cases]
    ops = [gemm_ops(M, N, K) for (M, _, N, K) in cases]
    ms_step = r["max_ms"] / args.steps
    value = world * wbytes / (ms_step * 1e-3) / 1e9
    tops = world * sum(ops) / (ms_step * 1e-3) / 1e12

    # roofline of the dominant kernel (the GEMM): its launches timed alone
    per = r["per_case_ms"]
    gemm_ms = r["gemm_ms"] / args.steps  # all GEMM launches of one step
    # the GEMM launches are timed back to back for a few milliseconds, not a
    # seconds-long power-capped loop: the burst figure (the sustained one is
    # reported beside it)
    int8_peak_tops = peaks["bf16_tflops"] * INT8_OVER_BF16
    int8_sustained_tops = peaks["bf16_tflops_sustained"] * INT8_OVER_BF16
    hbm = peaks["hbm_gbs"]
    roof_t = [max(b / (hbm * 1e9), o / (int8_peak_tops * 1e12)) * 1e3 for b, o in zip(abytes, ops)]
    hbm_bound = sum(b / (hbm * 1e9) >= o / (int8_peak_tops * 1e12) for b, o in zip(abytes, ops)) * 2 >= len(cases)
    if hbm_bound:
        achieved = sum(abytes) / (gemm_ms * 1e-3) / 1e9
        roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                    "frac": round(achieved / hbm, 4)}
    else:
        achieved = sum(ops) / (gemm_ms * 1e-3) / 1e12
        roofline = {"bound": "tensor", "achieved": round(achieved, 1), "peak": int8_peak_tops,
                    "unit": "TOPS", "frac": round(achieved / int8_peak_tops, 4),
                    "frac_of_sustained": round(achieved / int8_sustained_tops, 4)}
    traffic = (recorded_traffic(f"{args.workload}-{args.weights}") if lut else
               recorded_traffic(args.workload) if ACT_BITS[args.act] == 8 else None)
    roofline["traffic"] = traffic
    roofline["peak_source"] = (f"{peaks['source']} HBM copy" if hbm_bound else
                               f"{peaks['source']} burst bf16 x {INT8_OVER_BF16:g} (nominal int8/bf16 ratio)")
    roofline["kernel"] = "w4a8_gemm_kernel"
    roofline["roofline_time_frac"] = round(sum(roof_t) / gemm_ms, 4)
    roofline["launches"] = len(cases) * args.steps
    roofline["avg_launch_us"] = round(gemm_ms * 1e3 / len(cases), 3)

    # the activation quantizers' launches timed alone: fp16 activations in,
    # codes (8- or 4-bit), per-token scale (2 B) and rowsum (4 B) out
    quantizer = None
    if r.get("quant_ms") is not None:
        qbytes = sum(M * K * 2 + M * K * ACT_BITS[args.act] // 8 + 6 * M for (M, _, N, K) in cases)
        q_ms = r["quant_ms"] / args.steps
        q_ach = qbytes / (q_ms * 1e-3) / 1e9
        quantizer = {"kernel": ("quantize_act_static_kernel" if args.act.startswith("static") else "quantize_act_kernel")
                               + ("" if ACT_BITS[args.act] == 8 else " (4-bit codes)"),
                     "bound": "hbm", "achieved": round(q_ach, 1), "peak": hbm, "unit": "GB/s",
                     "frac": round(q_ach / hbm, 4), "bytes_per_step": qbytes,
                     "avg_launch_us": round(q_ms * 1e3 / len(cases), 3),
                     "note": "latency-bound at these sizes (at most 32 x 14336 activations per launch)"}

    per_case = []
    for (M, name, N, K), t, b, o, rt in zip(cases, per, abytes, ops, roof_t):
        per_case.append({"M": M, "layer": name, "N": N, "K": K, "us_with_events": round(t * 1e3, 2),
                         "weight_GBs": round(weight_bytes(N, K, lut) / (t * 1e-3) / 1e9, 1),
                         "tops": round(o / (t * 1e-3) / 1e12, 2), "roofline_frac": round(rt / t, 3)})

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp16" if lut else "int8", "data": "synthetic",
        "config": {"workload": args.workload, "weights": args.weights,
                   "activation_scales": "none (fp16 activations)" if lut else args.act, "cases": len(cases),
                   "gemm_call": ("w4a4_gemm" if ACT_BITS[args.act] == 4 and not lut
                                 else "w4lut3_gemm" if lut == 3 else "w4lut_gemm" if lut else "w4a8_gemm"),
                   "shapes": [f"M={M} {n} {N}x{K}" for (M, n, N, K) in cases][:: max(1, len(cases) // 16)],
                   "group": 128, "weights_per_step_MB": round(wbytes / 1e6, 1),
                   "l2": f"inputs larger than L2: {r['n_copies']} weight copies, {wbytes / 1e6:.0f} MB per step",
                   "parallelism": f"replicas x{world}",
                   "timing": "value: one CUDA graph of K unrolled steps; roofline: a second graph of the same "
                             "K steps' GEMM launches alone; cases: a third with events around each GEMM; e2e: "
                             "K steps in one graph, one host-to-device and one device-to-host copy per step, "
                             "double-buffered on two copy streams"},
        "tops": round(tops, 2),
        # timed region of `value`, per case: the activation quantizer (none for
        # the weight-only GEMM), the 4-bit expansion pre-pass (W4A4), the GEMM
        "gpu_launches": (1 + (0 if lut else 1) + (1 if ACT_BITS[args.act] == 4 and not lut else 0))
                        * len(cases) * args.steps,
        "roofline": roofline,
        "quantizer": quantizer,
        "e2e": {"value": round(world * wbytes / (r["e2e_ms"] / args.steps * 1e-3) / 1e9, 1), "unit": "GB/s",
                "h2d_bytes_per_step": r["h2d_bytes"], "d2h_bytes_per_step": r["d2h_bytes"]},
        "clocks": r["clocks"],
        "cases": per_case,
        "gpu": r["gpu_name"],
    }
    use_chain = args.chain == "on" and not lut and args.act == "dynamic" and \
        max(M for (M, _, _, _) in cases) <= 32 and len(cases) <= 16
    if use_chain:
        # The step as one w4a8_chain launch (the same quantize + GEMM per case,
        # each case after the previous one): value, roofline and e2e come from
        # it; the per-launch figures above move to `per_launch`.
        args.chain_mode = True
        rc = run_gpu(args, world, rank, local)
        args.chain_mode = False
        ms_c = rc["max_ms"] / args.steps
        launch_c = rc["gemm_ms"] / args.steps  # one chain launch per step
        # bytes the chain must move: weights, fp16 activations in, their codes,
        # scales and rowsums out, Y out
        cbytes = [weight_bytes(N, K) + 2 * M * K + M * K + 6 * M + 2 * M * N for (M, _, N, K) in cases]
        achieved_c = sum(cbytes) / (launch_c * 1e-3) / 1e9
        line["per_launch"] = {"value": line["value"], "ms_per_step": line["ms_per_step"], "tops": line["tops"],
                              "roofline": roofline, "e2e": line["e2e"], "gpu_launches": line["gpu_launches"],
                              "note": "the same step as separate w4a8_quantize_act + w4a8_gemm launches per case"}
        line["value"] = round(world * wbytes / (ms_c * 1e-3) / 1e9, 1)
        line["ms_per_step"] = round(ms_c, 5)
        line["tops"] = round(world * sum(ops) / (ms_c * 1e-3) / 1e12, 2)
        line["gpu_launches"] = args.steps
        line["roofline"] = {"bound": "hbm", "achieved": round(achieved_c, 1), "peak": hbm, "unit": "GB/s",
                            "frac": round(achieved_c / hbm, 4), "traffic": recorded_traffic(args.workload + "-chain"),
                            "peak_source": f"{peaks['source']} HBM copy", "kernel": "w4a8_chain_kernel",
                            "launches": args.steps, "avg_launch_us": round(launch_c * 1e3, 3),
                            "bytes_per_launch": int(sum(cbytes))}
        line["e2e"] = {"value": round(world * wbytes / (rc["e2e_ms"] / args.steps * 1e-3) / 1e9, 1), "unit": "GB/s",
                       "h2d_bytes_per_step": rc["h2d_bytes"], "d2h_bytes_per_step": rc["d2h_bytes"]}
        line["clocks"] = rc["clocks"]
        line["config"]["timing"] = ("value: one CUDA graph of K unrolled steps, each step one w4a8_chain launch over "
                                    "the cases in order (each case quantized after the previous case's output is "
                                    "complete); roofline: the chain launch's average duration over those K launches; "
                                    "e2e: K steps in one graph, one host-to-device and one device-to-host copy per "
                                    "step, double-buffered on two copy streams; per_launch: the same step as "
                                    "separate launches (cases: per-launch times with events around each GEMM)")
        line["config"]["path"] = "w4a8_chain (one persistent launch per step)"
    if world == 1 and not args.no_configs and not lut and args.act == "dynamic" and not args.cases:
        import torch
        dev = torch.device("cuda", local)
        int8_meas = int8_ceiling_tops(dev)
        with ClockSampler(dev) as clk2:
            configs, n_cfg_launches = run_configs(dev, peaks, int8_meas)
        configs["summary"]["clocks"] = clk2.summary()
        configs["summary"]["gpu_launches"] = n_cfg_launches
        line["configs"] = configs
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, sample, threads, t = cpu_oracle_run(args.workload, args.cpu_seconds, act_bits=ACT_BITS[args.act], lut=lut)
        line["cpu_baseline"] = {"value": round(v, 3), "unit": "GB/s", "cores": threads, "kind": "oracle",
                                "sample": f"{len(sample)} of {len(cases)} cases ({'; '.join(sample)}), "
                                          f"{t:.1f} s of oracle time"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main_reference(args, world, rank):
    """The CPU oracle as the reference arm (rank 0 only)."""
    if rank != 0:
        return
    cases = cases_of(args.workload)
    lut = lut_bits(args.weights)
    cpu_oracle_run(args.workload, 0.0, act_bits=ACT_BITS[args.act], lut=lut)  # untimed warm-up (one case)
    t0 = time.perf_counter()
    tot_bytes, tot_t, samples = 0.0, 0.0, []
    for _ in range(args.steps):
        v, sample, threads, t = cpu_oracle_run(args.workload, args.cpu_seconds / max(args.steps, 1),
                                               act_bits=ACT_BITS[args.act], lut=lut)
        tot_t += t
        tot_bytes += v * t * 1e9
        samples = sample
    value = tot_bytes / tot_t / 1e9
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(tot_t / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp16" if lut else "int8", "data": "synthetic",
        "config": {"workload": args.workload, "weights": args.weights, "cases": len(cases), "group": 128},
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": f"per step: {len(samples)} of {len(cases)} cases ({'; '.join(samples)})"},
        "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": round(time.perf_counter() - t0, 1),
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
