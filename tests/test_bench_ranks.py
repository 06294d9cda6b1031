"""The benchmark's multi-rank plumbing on CPU (gloo, world size 2): every rank
times its own replica and the reported time is the maximum over ranks."""
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        assert bench.dist_env() == (rank, world, rank)
        dev = torch.device("cpu")
        bench.barrier(dev)
        t = bench.reduce_max(10.0 + 5.0 * rank, dev)
        q.put((rank, t))
        bench.barrier(dev)
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert got == [(0, 15.0), (1, 15.0)]


def test_reduce_max_without_process_group_is_identity():
    import bench
    assert bench.reduce_max(3.5, torch.device("cpu")) == 3.5


def test_decode_schedule_and_bytes():
    import bench
    from bit_asymmetric_kv_prefill_b200 import synth
    w = synth.WORKLOADS["llama2_7b_layer"]
    sched = bench.decode_schedule(w)
    assert sched[0] == (4096, 1) and sched[-1] == (4096, 64) and len(sched) == 64
    # 96 B per quantized (token, kv head) and 512 B per residual token at D=128, G=32
    assert bench.decode_bytes(w, 4096, 1) == 8 * 32 * (4096 * 96 + 512) + 8 * 32 * 128 * 6


def _run_bench(args, **env):
    import json
    import subprocess
    e = dict(os.environ, PYTHONPATH=ROOT, **env)
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True,
                       text=True, env=e, timeout=600, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    return [json.loads(ln) for ln in lines]


def test_reference_arm_runs_on_rank_0_only():
    """Under torchrun only rank 0 times the oracle and prints; other ranks exit
    0 without work."""
    args = ["--impl", "reference", "--workload", "tiny", "--decode-steps", "2", "--steps", "1",
            "--warmup", "3"]
    assert _run_bench(args, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1") == []
    (line,) = _run_bench(args, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0", KIVI_ORACLE_THREADS="2")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    # the oracle runs on the host's cores: here the two threads allowed
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 2
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
