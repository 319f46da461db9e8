"""The benchmark's multi-rank plumbing on CPU: two gloo ranks (the N > 1
launch shape of `bench.py`, one process per GPU there) agree on the max of a
per-rank time and pass the barrier; the reference arm runs on rank 0 only."""
import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, _ = bench.dist_env()
        got = bench.max_over_ranks(1.5 + 3.0 * rank, w)
        bench.barrier(w)

        class Args:
            workload = "tiny"
            steps = 1
            cpu_seconds = 0.1
        ref = bench.main_reference(Args, w, r) if r != 0 else "skipped"
        out.put((r, w, got, ref))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_and_barrier():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [(r, w) for r, w, _, _ in res] == [(0, 2), (1, 2)]
    assert all(got == 4.5 for _, _, got, _ in res)  # max over ranks of 1.5, 4.5
    assert res[0][3] == "skipped" and res[1][3] is None  # rank 1 leaves the reference arm at once


def test_kv_reference_arm_prints_one_line():
    """`bench.py --workload kv-tiny --impl reference` (the CPU oracle as the
    reference arm of the KV-cache attention workload) prints one JSON line
    with the contract's keys; the GEMM lines are not involved."""
    import json
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--workload", "kv-tiny", "--impl",
                        "reference", "--steps", "2", "--warmup", "3", "--cpu-seconds", "0.2"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["config"]["workload"] == "kv-tiny"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
